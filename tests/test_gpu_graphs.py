"""Calls captured in a CUDA graph and replayed: the way a serving loop removes launch
overhead from many small GEMMs (the cost the GEMM-cost page, "为什么我们要死磕GEMM"
(kwkr.cn), section 3.3, attributes to small kernels). Every call type is captured on a
shape whose tiles are cut along K (the split fix-up and its arrival counters are the
state a replay must find reset), then replayed three times with new input values: each
replay must equal, bit for bit, an eager call of the library on the same inputs (both
are deterministic and run the same plan)."""
import numpy as np
import pytest
import torch

import sm_gemm_b200 as sg

pytestmark = pytest.mark.gpu


def _replays_match_eager(make_inputs, call, outputs, workspace):
    """make_inputs(seed) refills the input tensors in place; call(outs, ws) runs the
    library on them into the output set `outs` with workspace `ws`; outputs() allocates
    an output set and workspace() a workspace. The graph and the eager calls have
    separate workspaces, and every set of inputs is replayed twice in a row, so a replay
    finds only what the previous replay of the same graph left behind."""
    dev_out, eager_out = outputs(), outputs()
    dev_ws, eager_ws = workspace(), workspace()
    make_inputs(0)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        for _ in range(2):
            call(dev_out, dev_ws)
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        call(dev_out, dev_ws)
    for seed in (1, 2, 3):
        make_inputs(seed)
        call(eager_out, eager_ws)
        for rep in range(2):
            graph.replay()
            torch.cuda.synchronize()
            assert sg.check() == sg.OK
            for g, e in zip(dev_out, eager_out):
                assert torch.equal(g, e), f"replay {rep} of inputs {seed} differs from the eager call"
    del graph


def _fill(ts, seed, scale=1.0):
    gen = torch.Generator(device="cuda").manual_seed(1000 + seed)
    for t in ts:
        t.copy_((torch.randn(t.shape, generator=gen, device="cuda") * scale).to(t.dtype))


def test_graph_replay_bf16_split_tail(cuda_device):
    A = torch.empty(1024, 4096, dtype=torch.bfloat16, device="cuda")
    B = torch.empty(4096, 2048, dtype=torch.bfloat16, device="cuda")
    bias = torch.empty(2048, dtype=torch.bfloat16, device="cuda")
    nws = max(sg.workspace_size(1024, 2048, 4096), 16)
    _replays_match_eager(lambda s: _fill([A, B, bias], s, 0.1),
                         lambda o, ws: sg.gemm_bf16(A, B, bias=bias, act="gelu_tanh", out=o[0], workspace=ws),
                         lambda: [torch.empty(1024, 2048, dtype=torch.bfloat16, device="cuda")],
                         lambda: torch.empty(nws, dtype=torch.uint8, device="cuda"))
    assert "sk_iters=0" not in sg.last_config()


def test_graph_replay_skinny_stream_k(cuda_device):
    X = torch.empty(16, 8192, dtype=torch.bfloat16, device="cuda")
    W = torch.empty(8192, 1024, dtype=torch.bfloat16, device="cuda")
    nws = max(sg.workspace_size(16, 1024, 8192), 16)
    _replays_match_eager(lambda s: _fill([X, W], s, 0.1),
                         lambda o, ws: sg.gemm_bf16(X, W, out=o[0], workspace=ws),
                         lambda: [torch.empty(16, 1024, dtype=torch.float32, device="cuda")],
                         lambda: torch.empty(nws, dtype=torch.uint8, device="cuda"))
    assert "path=skinny" in sg.last_config() and "sk_iters=0" not in sg.last_config()


def test_graph_replay_fp8_quantise_fp8out_and_gemm(cuda_device):
    Xf = torch.empty(256, 4096, device="cuda")
    Wf = torch.empty(4096, 1024, device="cuda")
    X16 = torch.empty(256, 4096, dtype=torch.bfloat16, device="cuda")
    W16 = torch.empty(4096, 1024, dtype=torch.bfloat16, device="cuda")

    def outputs():
        return [torch.empty(256, 4096, dtype=torch.uint8, device="cuda"), torch.empty(32, 256, device="cuda"),
                torch.empty(1024, 4096, dtype=torch.uint8, device="cuda"), torch.empty(32, 8, device="cuda"),
                torch.empty(256, 1024, dtype=torch.bfloat16, device="cuda"),
                torch.empty(256, 1024, dtype=torch.uint8, device="cuda"), torch.empty(8, 256, device="cuda")]

    def call(o, ws):
        sg.quantize_fp8_blockwise(Xf, 1, Q=o[0], scales=o[1])
        sg.quantize_fp8_blockwise(Wf, 128, Q=o[2], scales=o[3])
        sg.gemm_fp8_blockscaled(o[0], o[1], o[2], o[3], out=o[4], workspace=ws[0])
        sg.gemm_bf16_fp8out(X16, W16, act="silu", Q=o[5], scales=o[6], workspace=ws[1])

    def inputs(s):
        _fill([Xf, Wf], s)
        _fill([X16, W16], s + 10, 0.1)

    # a workspace per GEMM, so that neither call's counters are touched by the other's
    _replays_match_eager(inputs, call, outputs,
                         lambda: [torch.empty(32 << 20, dtype=torch.uint8, device="cuda") for _ in range(2)])
    assert "sk_iters=0" not in sg.last_config()


def test_graph_replay_grouped_split_tail(cuda_device):
    sizes = [(384, 1024, 2048), (130, 512, 2048), (700, 256, 2048)]
    As = [torch.empty(m, k, dtype=torch.bfloat16, device="cuda") for m, n, k in sizes]
    Bs = [torch.empty(k, n, dtype=torch.bfloat16, device="cuda") for m, n, k in sizes]
    nws = int(sg.lib().smgemm_grouped_workspace_size(len(sizes)))
    _replays_match_eager(lambda s: _fill(As + Bs, s, 0.1),
                         lambda o, ws: sg.gemm_bf16_grouped(As, Bs, outs=o, workspace=ws),
                         lambda: [torch.empty(m, n, dtype=torch.bfloat16, device="cuda") for m, n, k in sizes],
                         lambda: torch.empty(nws, dtype=torch.uint8, device="cuda"))
    assert "splits=0" not in sg.last_config()


def test_graph_replay_lm_head_log_softmax(cuda_device):
    X = torch.empty(4, 4096, dtype=torch.bfloat16, device="cuda")
    W = torch.empty(4096, 4000, dtype=torch.bfloat16, device="cuda")
    nws = max(int(sg.lib().smgemm_logsoftmax_workspace_size(4, 4000, 4096)), 16)
    _replays_match_eager(lambda s: _fill([X, W], s, 0.1),
                         lambda o, ws: sg.gemm_bf16_logsoftmax(X, W, out=o[0], workspace=ws),
                         lambda: [torch.empty(4, 4000, dtype=torch.float32, device="cuda")],
                         lambda: torch.empty(nws, dtype=torch.uint8, device="cuda"))


def test_graph_replay_grouped_many_groups(cuda_device):
    """More groups than travel with the launch itself (16): the table is written into the
    workspace by kernels that carry it as parameters, which the graph replays."""
    rs = np.random.RandomState(5)
    sizes = [(int(rs.randint(1, 300)), 8 * int(rs.randint(1, 40)), 8 * int(rs.randint(1, 60))) for _ in range(40)]
    As = [torch.empty(m, k, dtype=torch.bfloat16, device="cuda") for m, n, k in sizes]
    Bs = [torch.empty(k, n, dtype=torch.bfloat16, device="cuda") for m, n, k in sizes]
    nws = int(sg.lib().smgemm_grouped_workspace_size(len(sizes)))
    _replays_match_eager(lambda s: _fill(As + Bs, s, 0.1),
                         lambda o, ws: sg.gemm_bf16_grouped(As, Bs, outs=o, workspace=ws),
                         lambda: [torch.empty(m, n, dtype=torch.bfloat16, device="cuda") for m, n, k in sizes],
                         lambda: torch.empty(nws, dtype=torch.uint8, device="cuda"))
