"""Pins for the oracle GEMM (FP64 triple loop + bias + activation + one RNE cast).

Each check is independent of the oracle's own code: exact rational arithmetic on
tiny shapes, closed forms (identity, permutation, rank-1, all-ones), integer-valued
inputs against numpy's int64 matmul, the activations against torch's float64
implementations, and the FLOP count of the worked example printed by the
DeepGEMM kernel-library walkthrough (zwxr.cn), section 3.4.
"""
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
import synth
from sm_gemm_b200 import metrics

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _bf16_bits(x: np.ndarray) -> np.ndarray:
    return torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.bfloat16) \
        .view(torch.int16).numpy().view(np.uint16)


def _bf16_values(bits: np.ndarray) -> np.ndarray:
    return torch.from_numpy(bits.view(np.int16)).view(torch.bfloat16).to(torch.float64).numpy()


def _exact_nearest(q: Fraction, prec: int, emin: int) -> float:
    if q == 0:
        return 0.0
    a = abs(q)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    e = max(e, emin)
    step = Fraction(2) ** (e - prec + 1)
    n = abs(q) / step
    lo = n.numerator // n.denominator
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    v = float(lo * step)
    return -v if q < 0 else v


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (3, 5, 7), (7, 9, 33), (4, 3, 130)])
@pytest.mark.parametrize("out", [oracle.F32, oracle.BF16])
def test_brute_force_rational(M, N, K, out):
    a = _bf16_bits(synth.normal(11, 0, (M, K)))
    b = _bf16_bits(synth.normal(11, 1, (K, N)))
    av, bv = _bf16_values(a), _bf16_values(b)
    got = oracle.gemm(a, b, a_dtype=oracle.BF16, b_dtype=oracle.BF16, out_dtype=out)
    prec, emin = (24, -126) if out == oracle.F32 else (8, -126)
    for i in range(M):
        for j in range(N):
            s = sum((Fraction(float(av[i, k])) * Fraction(float(bv[k, j])) for k in range(K)),
                    Fraction(0))
            assert got[i, j] == _exact_nearest(s, prec, emin)


def test_layouts_by_strides_agree():
    A = synth.normal(12, 0, (37, 53)).astype(np.float16)
    B = synth.normal(12, 1, (53, 29)).astype(np.float16)
    ref = oracle.gemm(A, B)
    assert (oracle.gemm(np.asfortranarray(A), B) == ref).all()
    assert (oracle.gemm(A, np.ascontiguousarray(B.T).T) == ref).all()      # B stored [N,K]
    assert (oracle.gemm(np.ascontiguousarray(A.T).T, np.ascontiguousarray(B.T).T) == ref).all()


def test_identity_and_permutation():
    A = synth.normal(13, 0, (40, 64)).astype(np.float16)
    I = np.eye(64, dtype=np.float16)
    assert (oracle.gemm(A, I) == A.astype(np.float64)).all()
    perm = np.random.RandomState(0).permutation(64)
    P = np.zeros((64, 64), dtype=np.float16)
    P[perm, np.arange(64)] = 1                       # (A @ P)[:, j] = A[:, perm[j]]
    assert (oracle.gemm(A, P) == A.astype(np.float64)[:, perm]).all()


def test_rank_one_closed_form():
    rs = np.random.RandomState(1)
    x = rs.randint(-4, 5, 23).astype(np.float64)
    u = rs.randint(-4, 5, 77).astype(np.float64)
    v = rs.randint(-4, 5, 77).astype(np.float64)
    z = rs.randint(-4, 5, 31).astype(np.float64)
    A = np.outer(x, u).astype(np.float16)            # |entries| <= 16: exact in fp16
    B = np.outer(v, z).astype(np.float16)
    want = np.outer(x, z) * float(u @ v)
    assert (oracle.gemm(A, B) == want).all()


def test_all_ones_gives_K():
    for K in (1, 64, 67, 4096):
        A = np.ones((5, K), dtype=np.float16)
        B = np.ones((K, 6), dtype=np.float16)
        assert (oracle.gemm(A, B) == K).all()


def test_integer_inputs_match_int64_matmul():
    A = synth.integers(14, 0, (70, 300), -4, 4)
    B = synth.integers(14, 1, (300, 90), -4, 4)
    want = A.astype(np.int64) @ B.astype(np.int64)
    got = oracle.gemm(_bf16_bits(A), _bf16_bits(B), a_dtype=oracle.BF16, b_dtype=oracle.BF16)
    assert (got == want).all()


def test_row_and_column_subsets():
    A = synth.normal(15, 0, (50, 40)).astype(np.float16)
    B = synth.normal(15, 1, (40, 60)).astype(np.float16)
    full = oracle.gemm(A, B)
    rows, cols = [3, 0, 49], [59, 7]
    assert (oracle.gemm(A, B, rows=rows, cols=cols) == full[np.ix_(rows, cols)]).all()


def test_activations_against_torch():
    x = np.linspace(-12, 12, 2001)
    g = np.array([oracle.act(v, oracle.ACT_GELU_TANH) for v in x])
    s = np.array([oracle.act(v, oracle.ACT_SILU) for v in x])
    tg = F.gelu(torch.from_numpy(x), approximate="tanh").numpy()
    ts = F.silu(torch.from_numpy(x)).numpy()
    np.testing.assert_allclose(g, tg, rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(s, ts, rtol=1e-13, atol=1e-15)
    # closed forms: act(0) = 0, SiLU(ln 3) = (3/4) ln 3, GeLU(x) -> x and SiLU(x) -> x for large x
    assert oracle.act(0.0, oracle.ACT_GELU_TANH) == 0.0 and oracle.act(0.0, oracle.ACT_SILU) == 0.0
    assert math.isclose(oracle.act(math.log(3), oracle.ACT_SILU), 0.75 * math.log(3), rel_tol=1e-15)
    assert oracle.act(40.0, oracle.ACT_GELU_TANH) == 40.0
    assert math.isclose(oracle.act(40.0, oracle.ACT_SILU), 40.0, rel_tol=1e-15)


def _gelu_tanh_decimal(x: float) -> "Decimal":
    """0.5 x (1 + tanh(u)), u = sqrt(2/pi)(x + 0.044715 x^3), in 200-digit decimal
    arithmetic with tanh(u) = (e^(2u) - 1) / (e^(2u) + 1): the definition as written,
    accurate even where 1 + tanh(u) is below 1e-100."""
    from decimal import Decimal, localcontext
    with localcontext() as ctx:
        ctx.prec, ctx.Emax, ctx.Emin = 200, 10 ** 9, -10 ** 9
        xd = Decimal(x)
        pi = Decimal("3.14159265358979323846264338327950288419716939937510582097494459230781640628620899863")
        c = (Decimal(2) / pi).sqrt()
        u = c * (xd + Decimal("0.044715") * xd * xd * xd)
        e = (2 * u).exp()
        return Decimal("0.5") * xd * (1 + (e - 1) / (e + 1))


def _silu_decimal(x: float) -> "Decimal":
    from decimal import Decimal, localcontext
    with localcontext() as ctx:
        ctx.prec, ctx.Emax, ctx.Emin = 200, 10 ** 9, -10 ** 9
        xd = Decimal(x)
        return xd / (1 + (-xd).exp())


def test_activations_against_high_precision():
    """GeLU (tanh form) and SiLU over [-15, 15] and a few large magnitudes, against the
    definitions evaluated in 200-digit decimal arithmetic: relative error at most 1e-13
    everywhere, including the negative tails where the values are tiny (GeLU(-12) is
    about 1e-53) and any cancellation in 1 + tanh(u) would show."""
    from decimal import Decimal
    xs = [float(v) for v in np.linspace(-15, 15, 1201)] + [-40.0, -80.0, -300.0, 1e-20, -1e-20, 37.5, 500.0]
    for x in xs:
        for which, ref_fn in ((oracle.ACT_GELU_TANH, _gelu_tanh_decimal), (oracle.ACT_SILU, _silu_decimal)):
            got = oracle.act(x, which)
            ref = ref_fn(x)
            if ref == 0:
                assert got == 0.0
                continue
            if abs(ref) < Decimal("1e-300"):        # below the normal double range: compare absolutely
                assert abs(Decimal(got) - ref) < Decimal("1e-310"), (which, x, got, ref)
                continue
            rel = abs((Decimal(got) - ref) / ref)
            assert rel < Decimal("1e-13"), (which, x, got, float(ref), float(rel))


def test_bias_then_activation_then_one_cast():
    K = 16
    A = np.zeros((3, K), dtype=np.float16)
    B = np.zeros((K, 4), dtype=np.float16)
    bias = np.array([0.5, -1.0, 2.0, 0.0], dtype=np.float32)
    got = oracle.gemm(A, B, bias=bias, act=oracle.ACT_SILU, out_dtype=oracle.F64)
    want = np.array([b / (1 + math.exp(-b)) for b in bias.astype(np.float64)])
    assert np.allclose(got, want[None, :], rtol=1e-15)
    # C = A B + bias: with A = e_0 row, B row 0 = ones, bias shifts every column
    A[0, 0] = 1
    B[0, :] = 1
    got = oracle.gemm(A, B, bias=bias, out_dtype=oracle.F64)
    assert (got[0] == 1 + bias.astype(np.float64)).all() and (got[1] == bias).all()


def test_absacc_is_sum_of_abs_products():
    A = np.array([[1, -2, 3]], dtype=np.float16)
    B = np.array([[-1], [4], [0.5]], dtype=np.float16)
    c, acc = oracle.gemm(A, B, want_absacc=True)
    assert c[0, 0] == -1 - 8 + 1.5 and acc[0, 0] == 1 + 8 + 1.5


def test_flop_count_worked_example():
    """The worked example of the walkthrough's section 3.4: a 4096^3 FP16 GEMM is
    2*4096^3 FLOPs (about 137 G); at 0.5 ms it runs at about 274 TFLOP/s, which is
    about 55% of a 500 TFLOP/s part."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "flop_worked_example.txt"))
            if l.strip() and not l.startswith("#")]
    hdr, vals = rows[0], rows[1]
    d = dict(zip(hdr, vals))
    M, N, K = int(d["M"]), int(d["N"]), int(d["K"])
    fl = metrics.gemm_flops(M, N, K)
    assert fl == 137438953472
    assert round(fl / 1e9) == int(d["gflop_approx"])
    tf = metrics.tflops(fl, float(d["time_ms"]) * 1e-3)
    assert round(tf) == int(d["tflops_approx"]) + 1 or round(tf) == int(d["tflops_approx"])
    assert round(100 * tf / float(d["peak_tflops"])) == int(d["util_pct_approx"])
