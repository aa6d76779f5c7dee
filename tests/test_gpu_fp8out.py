"""GEMM with the FP8 output epilogue (gemm_bf16_fp8out): act(A B + bias) in FP32,
encoded per 1x128 row group exactly as the group quantiser does (DeepGEMM
kernel-library walkthrough, zwxr.cn, section 2.4), giving the A operand of the
block-scaled FP8 GEMM.

- Integer-valued inputs make every FP32 accumulator exact, so codes and scales must
  equal the oracle's quantisation of the exact product bit for bit (ragged N: a
  partial last group; ragged M).
- Real-valued inputs with bias and GeLU: every dequantised value code * s is within
  the GEMM contract (1e-3 sum|a||b|, times 1.2 for the slope of GeLU) plus one E4M3
  spacing at the value (the FP32 value may sit beside a rounding midpoint of the exact
  one), and every scale within the same relative bound of the exact amax / 448.
- Tiles split along K (split tail, stream-K range): the same exact codes and the same
  bounds.
- The output feeds gemm_fp8_blockscaled; that GEMM is checked against the oracle on
  the same codes and scales."""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import check_tolerance, orc_view, to_dtype

pytestmark = pytest.mark.gpu


def _e4m3_spacing(y):
    """Spacing of E4M3 at |y| (3 mantissa bits; subnormal spacing 2^-9 below 2^-6)."""
    a = np.maximum(np.abs(y), 2.0 ** -6)
    return 2.0 ** (np.floor(np.log2(a)) - 3)


@pytest.mark.parametrize("M,N,K", [(300, 520, 136), (256, 256, 64), (7, 136, 512)])
def test_fp8out_integer_exact(cuda_device, M, N, K):
    A = torch.from_numpy(synth.integers(61, 0, (M, K), -3, 3)).to(torch.bfloat16)
    B = torch.from_numpy(synth.integers(61, 1, (K, N), -3, 3)).to(torch.bfloat16)
    Q, S = sg.gemm_bf16_fp8out(A.cuda(), B.cuda())
    assert sg.check() == sg.OK
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    Z = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32).astype(np.float32)
    Qr, Sr = oracle.quant_1x128(Z)
    assert np.array_equal(S.cpu().numpy().view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q.cpu().numpy(), Qr)


@pytest.mark.parametrize("M,N,K,sched", [(512, 1024, 4096, "auto"), (300, 520, 1024, "sk"), (256, 256, 2048, "sk")])
def test_fp8out_split_tiles_integer_exact(cuda_device, monkeypatch, M, N, K, sched):
    """Tiles whose K range is cut over several CTAs: a ragged last wave split in 8 pieces
    (auto), or one stream-K range over all CTAs (sk). The reducer sums the pieces in K
    order with its own piece taken from TMEM, wherever it falls in that order, and keeps
    the activated values in TMEM between the two passes; integer inputs keep every
    partial sum exact, so codes and scales must still equal the oracle's bit for bit."""
    monkeypatch.setenv("SMGEMM_SCHED", sched)
    A = torch.from_numpy(synth.integers(65, 0, (M, K), -3, 3)).to(torch.bfloat16)
    B = torch.from_numpy(synth.integers(65, 1, (K, N), -3, 3)).to(torch.bfloat16)
    Q, S = sg.gemm_bf16_fp8out(A.cuda(), B.cuda())
    assert sg.check() == sg.OK
    plan = dict(kv.split("=") for kv in sg.last_config().split() if "=" in kv)
    assert int(plan["sk_iters"]) > 0, sg.last_config()
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    Z = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32).astype(np.float32)
    Qr, Sr = oracle.quant_1x128(Z)
    assert np.array_equal(S.cpu().numpy().view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q.cpu().numpy(), Qr)


@pytest.mark.parametrize("sched", ["auto", "sk"])
def test_fp8out_bias_gelu_tolerance(cuda_device, monkeypatch, sched):
    monkeypatch.setenv("SMGEMM_SCHED", sched)
    M, N, K = 384, 1000, 520
    A = to_dtype(synth.normal(62, 0, (M, K)), torch.bfloat16)
    B = to_dtype(synth.normal(62, 1, (K, N), 0.05), torch.bfloat16)
    bias = to_dtype(synth.normal(62, 2, (N,), 0.3), torch.bfloat16)
    Q, S = sg.gemm_bf16_fp8out(A.cuda(), B.cuda(), bias=bias.cuda(), act="gelu_tanh")
    assert sg.check() == sg.OK
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    bb, bbd = orc_view(bias)
    ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, bias=bb, bias_dtype=bbd, act=oracle.ACT_GELU_TANH,
                           out_dtype=oracle.F64, want_absacc=True)
    s = S.cpu().numpy().astype(np.float64)                       # [ceil(N/128), M]
    s_col = np.repeat(s.T, 128, axis=1)[:, :N]                   # scale of every element
    deq = oracle.e4m3_decode(Q.cpu().numpy()) * s_col
    gemm_err = 1.2e-3 * acc
    bound = gemm_err + s_col * _e4m3_spacing(ref / s_col) + 1e-12
    assert (np.abs(deq - ref) <= bound).all(), f"max err/bound {np.max(np.abs(deq - ref) / bound):.3g}"
    nb = s.shape[0]
    for g in range(nb):
        cols = slice(128 * g, min(N, 128 * g + 128))
        amax = np.abs(ref[:, cols]).max(axis=1)
        tol = 1.2e-3 * acc[:, cols].max(axis=1) / 448 + np.spacing(s[g].astype(np.float32))
        assert (np.abs(s[g] - amax / 448) <= tol).all()


def test_fp8out_feeds_fp8_gemm(cuda_device):
    M, D, F, N = 256, 512, 1024, 384
    X = to_dtype(synth.normal(63, 0, (M, D)), torch.bfloat16)
    W1 = to_dtype(synth.normal(63, 1, (D, F), 0.05), torch.bfloat16)
    W2 = synth.normal(63, 2, (F, N), 0.05)
    Hq, Hs = sg.gemm_bf16_fp8out(X.cuda(), W1.cuda(), act="gelu_tanh")
    W2q, W2s = sg.quantize_fp8_blockwise(torch.from_numpy(W2).cuda(), 128)
    Y = sg.gemm_fp8_blockscaled(Hq, Hs, W2q, W2s, out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    ref, acc = oracle.gemm_fp8(Hq.cpu().numpy(), Hs.cpu().numpy(), W2q.cpu().numpy(), W2s.cpu().numpy(),
                               out_dtype=oracle.BF16, want_absacc=True)
    check_tolerance(Y.float().cpu().numpy(), ref, acc, torch.bfloat16, what="FP8 GEMM on fused codes")


def test_fp8out_col_major_a_ragged_k_integer_exact(cuda_device):
    """Column-major A (the MN-major operand path) and K not a multiple of the 64-wide
    K-block: still exact on integer inputs."""
    M, N, K = 264, 384, 200
    A = torch.from_numpy(synth.integers(64, 0, (M, K), -3, 3)).to(torch.bfloat16)
    B = torch.from_numpy(synth.integers(64, 1, (K, N), -3, 3)).to(torch.bfloat16)
    Q, S = sg.gemm_bf16_fp8out(A.t().contiguous().cuda().t(), B.cuda())
    assert sg.check() == sg.OK
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    Z = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32).astype(np.float32)
    Qr, Sr = oracle.quant_1x128(Z)
    assert np.array_equal(S.cpu().numpy().view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q.cpu().numpy(), Qr)
