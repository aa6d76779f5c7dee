"""LM-head GEMM fused with the row log-softmax (gemm_bf16_logsoftmax; "为什么我们要死磕GEMM"
(kwkr.cn), section 7.2, scheme B), against the oracle: the FP64 GEMM, then the FP64 row
log-softmax.

Tolerance, from the GEMM contract: every logit z_n of a row is within
e_n = 1e-3 * sum_k |a_k||b_kn| + ulp_f32(z_n) of the exact one; the log-sum-exp is
1-Lipschitz in the max norm, so it is within max_n e_n, plus the FP32 evaluation of
exp/sum/log (a fixed-order tree of at most log2(N) additions: far below 1e-5 relative
to 1 + |lse|). Hence |out_n - ref_n| <= e_n + max_n' e_n' + 1e-5 (1 + |lse|)."""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import orc_view, to_dtype

pytestmark = pytest.mark.gpu


def _check(out, X, W, b, rows=None):
    xa, xd = orc_view(X)
    wa, wd = orc_view(W)
    kw = {} if b is None else dict(zip(("bias", "bias_dtype"), orc_view(b)))
    z, acc = oracle.gemm(xa, wa, a_dtype=xd, b_dtype=wd, out_dtype=oracle.F64, rows=rows, want_absacc=True, **kw)
    ref, lse = oracle.log_softmax_rows(z)
    got = out.cpu().numpy().astype(np.float64)
    if rows is not None:
        got = got[rows]
    e = 1e-3 * acc + np.spacing(np.abs(z).astype(np.float32)).astype(np.float64)
    bound = e + e.max(axis=1, keepdims=True) + 1e-5 * (1.0 + np.abs(lse))[:, None]
    err = np.abs(got - ref)
    assert np.isfinite(got).all()
    assert (err <= bound).all(), f"max err/bound {np.max(err / bound):.3g}"
    # the probabilities of every checked row sum to one
    assert np.allclose(np.exp(got).sum(axis=1), 1.0, atol=1e-4)


@pytest.mark.parametrize("M", [1, 5, 16, 64])
@pytest.mark.parametrize("N", [1000, 4096])
def test_logsoftmax_skinny(cuda_device, M, N):
    X = to_dtype(synth.normal(51, M, (M, 256)), torch.bfloat16)
    W = to_dtype(synth.normal(51, 100 + N, (256, N), 0.2), torch.bfloat16)
    b = to_dtype(synth.normal(51, 200, (N,), 0.5), torch.bfloat16)
    out = sg.gemm_bf16_logsoftmax(X.cuda(), W.cuda(), bias=b.cuda())
    assert sg.check() == sg.OK
    assert "path=skinny" in sg.last_config()
    _check(out, X, W, b)


@pytest.mark.parametrize("M,layout", [(200, "row"), (16, "col")])
def test_logsoftmax_large_path(cuda_device, M, layout):
    N = 1000
    X = to_dtype(synth.normal(52, M, (M, 264)), torch.bfloat16)
    W = to_dtype(synth.normal(52, 1, (264, N), 0.2), torch.bfloat16)
    Xd = X.cuda() if layout == "row" else X.t().contiguous().cuda().t()
    out = sg.gemm_bf16_logsoftmax(Xd, W.cuda())
    assert sg.check() == sg.OK
    assert "path=skinny" not in sg.last_config()
    _check(out, X, W, None)


def test_logsoftmax_lm_head_full_size(cuda_device):
    d = synth.lm_head(16)
    X = to_dtype(d["X"], torch.bfloat16)
    W = to_dtype(d["W"], torch.bfloat16)
    out = sg.gemm_bf16_logsoftmax(X.cuda(), W.cuda())
    assert sg.check() == sg.OK
    p = torch.exp(out.double()).sum(dim=1)
    assert torch.allclose(p, torch.ones_like(p), atol=1e-4)
    _check(out, X, W, None, rows=np.array([0, 15]))


@pytest.mark.parametrize("M,N", [(64, 20000), (3, 50000)])
def test_logsoftmax_cluster_merge_with_padding_ctas(cuda_device, M, N):
    """Wide rows whose column chunks run in clusters of 8 CTAs sharing the merge, with a
    chunk count that is not a multiple of 8 (10 and 49 chunks per row: the padding CTAs
    merge their share and subtract nothing), with bias, against the oracle on every row."""
    X = to_dtype(synth.normal(51, 0, (M, 256)), torch.bfloat16)
    W = to_dtype(synth.normal(51, 1, (256, N), 0.05), torch.bfloat16)
    b = to_dtype(synth.normal(51, 2, (N,), 0.5), torch.bfloat16)
    out = sg.gemm_bf16_logsoftmax(X.cuda(), W.cuda(), bias=b.cuda())
    assert sg.check() == sg.OK
    _check(out, X, W, b)


def test_logsoftmax_k0_is_log_softmax_of_bias(cuda_device):
    """K = 0: the logits are the bias alone, so every row is log_softmax(bias)."""
    M, N = 5, 1000
    b = to_dtype(synth.normal(53, 0, (N,), 2.0), torch.float32)
    X = torch.empty((M, 0), dtype=torch.bfloat16, device="cuda")
    W = torch.empty((0, N), dtype=torch.bfloat16, device="cuda")
    out = sg.gemm_bf16_logsoftmax(X, W, bias=b.cuda())
    assert sg.check() == sg.OK
    ref, _ = oracle.log_softmax_rows(np.tile(b.numpy().astype(np.float64), (M, 1)))
    assert np.allclose(out.cpu().numpy(), ref, rtol=0, atol=1e-5)


# ------------------------------------------------------------------ vocabulary split (two-step API)

@pytest.mark.parametrize("M,layout", [(5, "row"), (16, "row"), (64, "row"), (200, "row"), (16, "col")])
@pytest.mark.parametrize("slices", [1, 3])
def test_lse_partials_over_vocabulary_slices(cuda_device, M, layout, slices):
    """The vocabulary-parallel steps on one GPU: the columns of W are split into slices
    (tile-aligned, as the ranks of a vocabulary-parallel LM head hold them), each slice
    runs gemm_bf16_lse_partials on its own, the partials of all slices are stacked in
    slice order, and logsoftmax_apply_partials on each slice must give that slice of the
    whole row's log-softmax (same bound as the fused call). Rows M <= 64 with row-major X
    take the skinny kernel, whose epilogue forms the partials; the others the light pass
    over the logits."""
    from sm_gemm_b200 import vocab_parallel as vp
    N, K = 1000, 264
    X = to_dtype(synth.normal(54, M, (M, K)), torch.bfloat16)
    W = to_dtype(synth.normal(54, 1, (K, N), 0.2), torch.bfloat16)
    b = to_dtype(synth.normal(54, 2, (N,), 0.5), torch.float32)
    Xd = X.cuda() if layout == "row" else X.t().contiguous().cuda().t()
    outs, parts = [], []
    for r in range(slices):
        c0, c1 = vp.shard_columns(N, slices, r)
        Ws = W[:, c0:c1].contiguous().cuda()
        out = torch.empty((M, -(-(c1 - c0) // 4) * 4), dtype=torch.float32, device="cuda")[:, :c1 - c0]
        o, p = sg.gemm_bf16_lse_partials(Xd, Ws, bias=b[c0:c1].contiguous().cuda(), out=out)
        assert sg.check() == sg.OK
        outs.append((c0, c1, o))
        parts.append(p)
    every = torch.cat(parts, dim=0)
    full = torch.empty((M, N), dtype=torch.float32)
    lses = []
    for c0, c1, o in outs:
        lses.append(sg.logsoftmax_apply_partials(o, every).cpu())
        assert sg.check() == sg.OK
        full[:, c0:c1] = o.cpu()
    for l in lses[1:]:
        assert torch.equal(l, lses[0])
    _check(full, X, W, b)


def test_apply_partials_neutral_pairs_and_empty_slice(cuda_device):
    """Pairs (-inf, 0) (the padding of a short slice) change nothing, and a slice with no
    columns still receives the row's lse."""
    M, N, K = 4, 320, 128   # 2.5 tiles; W's row pitch (640 bytes) meets the 16-byte rule
    X = to_dtype(synth.normal(55, 0, (M, K)), torch.bfloat16).cuda()
    W = to_dtype(synth.normal(55, 1, (K, N), 0.2), torch.bfloat16).cuda()
    o, p = sg.gemm_bf16_lse_partials(X, W)
    pad = torch.zeros((2, M, 2), dtype=torch.float32, device="cuda")
    pad[:, :, 0] = float("-inf")
    ref = o.clone()
    lse_ref = sg.logsoftmax_apply_partials(ref, p)
    lse_pad = sg.logsoftmax_apply_partials(o, torch.cat([pad[:1], p, pad[1:]], dim=0))
    empty = torch.empty((M, 0), dtype=torch.float32, device="cuda")
    lse_empty = sg.logsoftmax_apply_partials(empty, p)
    assert sg.check() == sg.OK
    # neutral pairs change nothing but the pairing order of the merge tree (last-bit rounding)
    assert torch.allclose(lse_pad, lse_ref, rtol=0, atol=1e-5) and torch.allclose(o, ref, rtol=0, atol=1e-5)
    assert torch.equal(lse_empty, lse_ref)


def _ls_sweep(n=40, seed=909):
    rs = np.random.RandomState(seed)
    out = []
    for i in range(n):
        out.append(dict(M=int(rs.choice([int(rs.randint(1, 65)), int(rs.randint(65, 300))])),
                        N=8 * int(rs.randint(1, 400)), K=8 * int(rs.randint(1, 80)), bias=bool(rs.randint(2)),
                        sched=["auto", "dp", "sk"][rs.randint(3)], seed=700 + i))
    return out


@pytest.mark.parametrize("case", _ls_sweep(), ids=lambda c: "M{M}N{N}K{K}".format(**c))
def test_logsoftmax_seeded_random_sweep(cuda_device, monkeypatch, case):
    """Random rows (skinny and large-tile paths), vocabulary widths (not multiples of
    the 128-column tiles), depths, bias and schedules, within the bound above."""
    monkeypatch.setenv("SMGEMM_SCHED", case["sched"])
    M, N, K, s = case["M"], case["N"], case["K"], case["seed"]
    X = to_dtype(synth.normal(s, 0, (M, K)), torch.bfloat16)
    W = to_dtype(synth.normal(s, 1, (K, N), 0.2), torch.bfloat16)
    b = to_dtype(synth.normal(s, 2, (N,), 0.5), torch.bfloat16) if case["bias"] else None
    out = sg.gemm_bf16_logsoftmax(X.cuda(), W.cuda(), bias=None if b is None else b.cuda())
    assert sg.check() == sg.OK
    _check(out, X, W, b)
