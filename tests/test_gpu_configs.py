"""The five workloads at full size, in the launch configuration the bench times,
checked on sampled outputs (every tile row and tile column is sampled, plus the
ragged tails) against the oracle computed one output at a time; the quantiser is
checked bit for bit over the whole FP8 workload.

Workloads (seeded, synthetic):
 1. tiny FP16 64^3, U[-1,1], seed 0, FP32 out (checked in full);
 2. square BF16 4096^3, A row-major, B column-major, N(0,1), BF16 out;
 3. FFN pair: X[1024,4096] N(0,1), W1[4096,16384] and W2[16384,4096] N(0,0.02)
    row-major, b1 N(0,0.01), GEMM1 + bias + GeLU(tanh) -> H bf16, then H @ W2
    (GEMM2 is checked on the GPU's own H, the same operands both sides see);
 4. FP8 block-scaled 2048x16384x4096 from N(0,1) inputs with 1% x50 outliers;
 5. LM head: X[M,4096] N(0,1) x W[4096,128256] N(0,0.02), FP32 logits, M in {1,4,16,64}.
"""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import check_tolerance, orc_view, sample_indices, to_dtype

pytestmark = pytest.mark.gpu


def _sampled_ref(A, B, rows, cols, **kw):
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    return oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, rows=rows, cols=cols, want_absacc=True, **kw)


def test_square_bf16_4096(cuda_device):
    d = synth.square_bf16()
    A = to_dtype(d["A"], torch.bfloat16)
    Bt = to_dtype(d["Bt"], torch.bfloat16)          # B column-major = B^T stored [N, K]
    out = sg.gemm_bf16(A.cuda(), Bt.cuda().t(), out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    rows = sample_indices(4096, 128, 2, 1)
    cols = sample_indices(4096, 256, 2, 2)
    ref, acc = _sampled_ref(A, Bt.t(), rows, cols, out_dtype=oracle.BF16)
    got = out.float().cpu().numpy()[np.ix_(rows, cols)]
    check_tolerance(got, ref, acc, torch.bfloat16, what="square bf16")


def test_ffn_pair(cuda_device):
    d = synth.ffn_pair()
    X = to_dtype(d["X"], torch.bfloat16)
    W1 = to_dtype(d["W1"], torch.bfloat16)
    W2 = to_dtype(d["W2"], torch.bfloat16)
    b1 = to_dtype(d["b1"], torch.bfloat16)
    H = sg.gemm_bf16(X.cuda(), W1.cuda(), bias=b1.cuda(), act="gelu_tanh", out_dtype=torch.bfloat16)
    Y = sg.gemm_bf16(H, W2.cuda(), out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    rows = sample_indices(1024, 128, 3, 3)
    cols1 = sample_indices(16384, 256, 1, 4)
    bb, bbd = orc_view(b1)
    ref1, acc1 = _sampled_ref(X, W1, rows, cols1, bias=bb, bias_dtype=bbd, act=oracle.ACT_GELU_TANH,
                              out_dtype=oracle.BF16)
    check_tolerance(H.float().cpu().numpy()[np.ix_(rows, cols1)], ref1, acc1, torch.bfloat16, what="FFN GEMM1")
    cols2 = sample_indices(4096, 256, 2, 5)
    Hc = H.cpu()
    ref2, acc2 = _sampled_ref(Hc, W2, rows, cols2, out_dtype=oracle.BF16)
    check_tolerance(Y.float().cpu().numpy()[np.ix_(rows, cols2)], ref2, acc2, torch.bfloat16, what="FFN GEMM2")


def test_fp8_blockscaled_2048x16384x4096(cuda_device):
    d = synth.fp8_blockscaled()
    A = torch.from_numpy(d["A"])
    B = torch.from_numpy(d["B"])
    qa, sa = sg.quantize_fp8_blockwise(A.cuda(), 1)
    qb, sb = sg.quantize_fp8_blockwise(B.cuda(), 128)
    out = sg.gemm_fp8_blockscaled(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    qa_r, sa_r = oracle.quant_1x128(d["A"])
    qb_r, sb_r = oracle.quant_128x128(d["B"])
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa_r.view(np.uint32))
    assert np.array_equal(sb.cpu().numpy().view(np.uint32), sb_r.view(np.uint32))
    assert np.array_equal(qa.cpu().numpy(), qa_r)
    assert np.array_equal(qb.cpu().numpy(), qb_r)
    rows = sample_indices(2048, 128, 2, 6)
    cols = sample_indices(16384, 128, 1, 7)
    ref, acc = oracle.gemm_fp8(qa_r, sa_r, qb_r, sb_r, rows=rows, cols=cols, out_dtype=oracle.BF16,
                               want_absacc=True)
    check_tolerance(out.float().cpu().numpy()[np.ix_(rows, cols)], ref, acc, torch.bfloat16, what="fp8 full")


@pytest.fixture(scope="module")
def lm_weight():
    W = to_dtype(synth.lm_head(m=1)["W"], torch.bfloat16)
    return W, W.cuda()


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_lm_head(cuda_device, lm_weight, M):
    W, Wd = lm_weight
    X = to_dtype(synth.lm_head(m=M, vocab=8)["X"], torch.bfloat16)
    out = sg.gemm_bf16(X.cuda(), Wd, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    assert "skinny" in sg.last_config()
    cols = sample_indices(128256, 128, 1, 8 + M)
    rows = np.arange(M)
    ref, acc = _sampled_ref(X, W, rows, cols, out_dtype=oracle.F32)
    check_tolerance(out.cpu().numpy()[np.ix_(rows, cols)], ref, acc, torch.float32, what=f"lm head M={M}")
