"""gemm_bf16_noalloc: the entry point for callers that cannot allocate device memory
(a plugin or custom-op host given only its inputs and outputs, or a decode loop that
must not call cudaMalloc). It runs gemm_bf16's kernels with the library's own fixed
16 MiB device scratch array instead of a caller workspace.

Checks, through the C ABI: two calls in a row on a stream-K shape (one that uses
scratch) agree with gemm_bf16 given an ordinary workspace, within the parity
tolerance the other tests use (in fact bit for bit, same kernels, fixed reduction
order); a shape that would need more scratch than the array holds is rejected before
anything runs. This file is collected last so a failure here never hides other tests;
it passes alone in a fresh process as well as after them.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import sm_gemm_b200 as sg
import synth
from _parity import check_tolerance

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


def test_noalloc_matches_gemm_bf16_on_two_calls(cuda_device):
    M, N, K = 16, 8192, 8192                      # skinny shape whose tiles are split along K: uses scratch
    plan = sg.schedule_dump(M, N, K, 0, sg.ROW_MAJOR, torch.cuda.get_device_properties(0).multi_processor_count)
    assert (plan[:, 6] >= 0).any()                # some tiles are split: partials go through the scratch
    A = torch.from_numpy(synth.normal(95, 0, (M, K))).to(torch.bfloat16).cuda()
    B = torch.from_numpy(synth.normal(95, 1, (K, N), 0.02)).to(torch.bfloat16).cuda()
    ref = sg.gemm_bf16(A, B, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    ref = ref.cpu().numpy().astype(np.float64)
    absacc = (A.abs().double() @ B.abs().double()).cpu().numpy()      # sum_k |a||b| for the bound
    f = _noalloc()
    stream = torch.cuda.current_stream()
    for _ in range(2):
        out = torch.full((M, N), float("nan"), dtype=torch.float32, device="cuda")
        assert _call(f, A, B, out, stream) == sg.OK
        assert sg.check() == sg.OK
        got = out.cpu().numpy().astype(np.float64)
        check_tolerance(got, ref, absacc, torch.float32, rel=1e-3, diag=1e-4, what="noalloc vs gemm_bf16")


def test_noalloc_rejects_shapes_beyond_the_scratch(cuda_device):
    M = N = K = 4096                              # its stream-K partials need ~37 MiB > 16 MiB
    assert sg.workspace_size(M, N, K, 0) > SCRATCH_BYTES
    A = torch.zeros((M, K), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((K, N), dtype=torch.bfloat16, device="cuda")
    out = torch.full((M, N), 7.0, dtype=torch.float32, device="cuda")
    assert _call(_noalloc(), A, B, out, torch.cuda.current_stream()) == sg.ERR_WORKSPACE
    assert sg.check() == sg.OK
    assert bool((out == 7.0).all())               # nothing was launched
