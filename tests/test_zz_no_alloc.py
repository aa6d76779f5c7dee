"""gemm_bf16_noalloc: the entry point for callers that cannot allocate device memory
(a plugin or custom-op host given only its inputs and outputs, or a decode loop that
must not call cudaMalloc). It runs gemm_bf16's kernels with the library's own fixed
16 MiB device scratch array instead of a caller workspace.

Checks, through the C ABI: two calls in a row on a shape whose tiles are split along K
(so the partial tiles go through the scratch) give exactly gemm_bf16's output, bit for
bit (same kernels, same schedule, fixed reduction order), and sampled outputs meet the
GEMM contract against the CPU oracle; the LM head at M = 1, 4, 16 and 64 runs within the
array under both the default and the stream-K schedule and matches gemm_bf16 bit for
bit; a shape that would need more scratch than the array holds is rejected before
anything runs. This file is collected last so a
failure here never hides other tests; it passes alone in a fresh process as well as
after them.
"""
import ctypes as C
import os

import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import check_tolerance, orc_view, sample_indices

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _noalloc():
    f = sg.lib().gemm_bf16_noalloc
    I64, P, I = C.c_int64, C.c_void_p, C.c_int
    f.argtypes = [I64, I64, I64, P, I, I, I64, P, I, I64, P, I, I, P, I, I64, P]
    f.restype = I
    return f


def _call(f, A, B, C_out, stream):
    M, K = A.shape
    N = B.shape[1]
    return f(M, N, K, A.data_ptr(), sg.BF16, sg.ROW_MAJOR, A.stride(0), B.data_ptr(), sg.ROW_MAJOR, B.stride(0),
             None, 0, 0, C_out.data_ptr(), sg.F32, C_out.stride(0), C.c_void_p(stream.cuda_stream))


class _Sched:
    """Sets SMGEMM_SCHED for the calls inside the block (the library reads it per call)."""

    def __init__(self, mode):
        self.mode, self.old = mode, None

    def __enter__(self):
        self.old = os.environ.get("SMGEMM_SCHED")
        if self.mode is None:
            os.environ.pop("SMGEMM_SCHED", None)
        else:
            os.environ["SMGEMM_SCHED"] = self.mode

    def __exit__(self, *exc):
        if self.old is None:
            os.environ.pop("SMGEMM_SCHED", None)
        else:
            os.environ["SMGEMM_SCHED"] = self.old


def test_noalloc_matches_gemm_bf16_on_two_calls(cuda_device):
    M, N, K = 16, 8192, 8192                      # skinny shape whose tiles are split along K: uses scratch
    plan = sg.schedule_dump(M, N, K, 0, sg.ROW_MAJOR, torch.cuda.get_device_properties(0).multi_processor_count)
    assert (plan[:, 6] >= 0).any()                # some tiles are split: partials go through the scratch
    A = torch.from_numpy(synth.normal(95, 0, (M, K))).to(torch.bfloat16).cuda()
    B = torch.from_numpy(synth.normal(95, 1, (K, N), 0.02)).to(torch.bfloat16).cuda()
    ref = sg.gemm_bf16(A, B, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    f = _noalloc()
    stream = torch.cuda.current_stream()
    cols = sample_indices(N, 128, 3, seed=95)
    a_np, a_dt = orc_view(A)
    b_np, b_dt = orc_view(B)
    want, absacc = oracle.gemm(a_np, b_np, a_dtype=a_dt, b_dtype=b_dt, out_dtype=oracle.F32, cols=cols,
                               want_absacc=True)
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(f, A, B, out, stream) == sg.OK
        assert sg.check() == sg.OK
        assert torch.equal(out, ref), "noalloc output differs from gemm_bf16's"
        got = out.cpu().numpy()[:, cols]
        check_tolerance(got, want, absacc, torch.float32, what="noalloc vs oracle")


_W = {}


def _lm_head_weight():
    if "W" not in _W:
        _W["W"] = torch.from_numpy(synth.normal(96, 1000, (4096, 128256), 0.02)).to(torch.bfloat16).cuda()
    return _W["W"]


@pytest.mark.parametrize("sched", [None, "sk"])
@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_noalloc_lm_head_schedules(cuda_device, M, sched):
    """The LM head (N = 128256, K = 4096, row-major tokens: the skinny path) at every
    M <= 64 runs within the array under the default schedule and under the stream-K
    schedule (every tile's K range cut across CTAs, partials in the scratch), and gives
    gemm_bf16's output bit for bit."""
    N, K = 128256, 4096
    A = torch.from_numpy(synth.normal(96, M, (M, K))).to(torch.bfloat16).cuda()
    B = _lm_head_weight()
    with _Sched(sched):
        if sched == "sk":
            plan = sg.schedule_dump(M, N, K, 0, sg.ROW_MAJOR, torch.cuda.get_device_properties(0).multi_processor_count)
            assert (plan[:, 6] >= 0).any()
        ref = sg.gemm_bf16(A, B, out_dtype=torch.float32)
        assert sg.check() == sg.OK
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(_noalloc(), A, B, out, torch.cuda.current_stream()) == sg.OK
        assert sg.check() == sg.OK
    assert torch.equal(out, ref)


def test_noalloc_rejects_shapes_beyond_the_scratch(cuda_device):
    M = N = K = 4096                              # its stream-K partials need ~37 MiB > 16 MiB
    assert sg.workspace_size(M, N, K, 0) > SCRATCH_BYTES
    A = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((K, N), dtype=torch.bfloat16, device="cuda")
    out = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    assert _call(_noalloc(), A, B, out, torch.cuda.current_stream()) == sg.ERR_WORKSPACE
    assert sg.check() == sg.OK
    assert bool((out == 7.0).all())               # nothing was launched
