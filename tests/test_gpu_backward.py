"""Backward-pass GEMMs of a linear layer Y = X W through the layout flags alone (the
GEMM-backward derivation of "为什么我们要死磕GEMM" (kwkr.cn), section 3.2):
dX = dY W^T reads W as a column-major B operand, dW = X^T dY reads X as a
column-major A operand; no transposed copy is made. Checked against the oracle in
full on ragged shapes (and bit for bit on integer-valued inputs, where every partial
sum is exact), and on sampled outputs at the FFN layer's size (X[1024,4096],
W1[4096,16384], dH[1024,16384])."""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import check_tolerance, orc_view, sample_indices, to_dtype

pytestmark = pytest.mark.gpu


def _ref(A, B, rows=None, cols=None):
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    return oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.BF16, rows=rows, cols=cols,
                       want_absacc=True)


@pytest.mark.parametrize("M,K,N", [(200, 136, 264), (72, 56, 40), (384, 520, 1000)])
def test_backward_ragged(cuda_device, M, K, N):
    """Shapes ragged against the 256 x 256 tiles; every contiguous extent is a multiple
    of 8 elements (the 16-byte pitch the TMA descriptors need)."""
    X = to_dtype(synth.normal(31, 0, (M, K)), torch.bfloat16)
    W = to_dtype(synth.normal(31, 1, (K, N), 0.05), torch.bfloat16)
    dY = to_dtype(synth.normal(31, 2, (M, N)), torch.bfloat16)
    dX = sg.gemm_bf16(dY.cuda(), W.cuda().t(), out_dtype=torch.bfloat16)      # [M, K]
    dW = sg.gemm_bf16(X.cuda().t(), dY.cuda(), out_dtype=torch.bfloat16)      # [K, N]
    assert sg.check() == sg.OK
    ref, acc = _ref(dY, W.t())
    check_tolerance(dX.float().cpu().numpy(), ref, acc, torch.bfloat16, what="dX")
    ref, acc = _ref(X.t(), dY)
    check_tolerance(dW.float().cpu().numpy(), ref, acc, torch.bfloat16, what="dW")


def test_backward_integer_exact(cuda_device):
    """|values| <= 3, inner sizes <= 520: every partial sum is an exact integer below 2^13,
    so both sides must agree bit for bit after the one BF16 rounding."""
    M, K, N = 136, 264, 520
    X = torch.from_numpy(synth.integers(32, 0, (M, K), -3, 3).astype(np.float32)).to(torch.bfloat16)
    W = torch.from_numpy(synth.integers(32, 1, (K, N), -3, 3).astype(np.float32)).to(torch.bfloat16)
    dY = torch.from_numpy(synth.integers(32, 2, (M, N), -3, 3).astype(np.float32)).to(torch.bfloat16)
    dX = sg.gemm_bf16(dY.cuda(), W.cuda().t(), out_dtype=torch.float32)
    dW = sg.gemm_bf16(X.cuda().t(), dY.cuda(), out_dtype=torch.float32)
    assert sg.check() == sg.OK
    for got, (A, B) in ((dX, (dY, W.t())), (dW, (X.t(), dY))):
        a, ad = orc_view(A)
        b, bd = orc_view(B)
        ref = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32)
        assert np.array_equal(got.cpu().numpy(), ref.astype(np.float32))


def test_ffn_backward_full_size(cuda_device):
    d = synth.ffn_backward()
    X = to_dtype(d["X"], torch.bfloat16)
    W1 = to_dtype(d["W1"], torch.bfloat16)
    dH = to_dtype(d["dH"], torch.bfloat16)
    dX = sg.gemm_bf16(dH.cuda(), W1.cuda().t(), out_dtype=torch.bfloat16)     # 1024 x 4096, K = 16384
    dW1 = sg.gemm_bf16(X.cuda().t(), dH.cuda(), out_dtype=torch.bfloat16)     # 4096 x 16384, K = 1024
    assert sg.check() == sg.OK
    rows = sample_indices(1024, 128, 2, 7)
    cols = sample_indices(4096, 256, 1, 8)
    ref, acc = _ref(dH, W1.t(), rows, cols)
    check_tolerance(dX.float().cpu().numpy()[np.ix_(rows, cols)], ref, acc, torch.bfloat16, what="dX")
    rows = sample_indices(4096, 128, 1, 9)
    cols = sample_indices(16384, 256, 1, 10)
    ref, acc = _ref(X.t(), dH, rows, cols)
    check_tolerance(dW1.float().cpu().numpy()[np.ix_(rows, cols)], ref, acc, torch.bfloat16, what="dW1")
