"""Pins for the oracle's FP8 E4M3 codec and its round-to-format casts.

The codec is checked against (a) the format's own fixed points (max finite 448,
smallest subnormal 2^-9, smallest normal 2^-6, NaN code), (b) torch's independent
float8_e4m3fn implementation, and (c) a brute-force nearest-value search over the
256-entry table with ties to the even code. The casts to bf16 / fp16 / fp32 are
checked against numpy's direct double->half/float conversions and against an exact
rational nearest search (Python fractions) for bf16, including the double-rounding
trap (a double that rounds differently when it goes through float first).
"""
from fractions import Fraction

import numpy as np
import pytest
import torch

import oracle


def _table():
    return oracle.e4m3_decode(np.arange(256, dtype=np.uint8))


def test_decode_fixed_points():
    d = _table()
    assert d[0x7E] == 448.0 and d[0xFE] == -448.0          # max finite
    assert d[0x01] == 2.0 ** -9                             # smallest subnormal
    assert d[0x08] == 2.0 ** -6                             # smallest normal
    assert d[0x38] == 1.0                                   # exponent field 7 = bias
    assert d[0x00] == 0.0 and np.signbit(d[0x80])
    assert np.isnan(d[0x7F]) and np.isnan(d[0xFF])
    assert np.isfinite(d[0x78]) and d[0x78] == 256.0        # S.1111.000 is finite (no inf)
    fin = d[np.isfinite(d)]
    assert fin.size == 254


def test_decode_matches_torch():
    codes = np.arange(256, dtype=np.uint8)
    t = torch.from_numpy(codes).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    d = _table()
    same = (d == t) | (np.isnan(d) & np.isnan(t))
    assert same.all()


def _structured_floats():
    """All 2^16 (sign, exponent, top-7-mantissa) patterns x low-bit patterns that hit
    every E4M3 rounding boundary (exact ties, one ulp either side) plus random low bits."""
    hi = np.arange(1 << 16, dtype=np.uint32) << 16
    lows = np.array([0, 1, 0x7FFF, 0x8000, 0x8001, 0xFFFF, 0x1234, 0xC0DE], dtype=np.uint32)
    bits = (hi[:, None] | lows[None, :]).ravel()
    rnd = np.random.RandomState(7).randint(0, 2 ** 32, size=1 << 20, dtype=np.uint64).astype(np.uint32)
    bits = np.concatenate([bits, rnd])
    y = bits.view(np.float32)
    return y[np.isfinite(y)]


def _brute_force_encode(y: np.ndarray) -> np.ndarray:
    """Nearest finite E4M3 value by exhaustive search, ties to the even code;
    saturate beyond 448; sign kept on zero."""
    d = _table()
    codes = np.array([c for c in range(128) if np.isfinite(d[c])], dtype=np.uint8)   # +0 .. 448
    vals = d[codes]
    a = np.abs(y.astype(np.float64))
    out = np.empty(y.shape, dtype=np.uint8)
    for s in range(0, a.size, 1 << 16):
        blk = a[s:s + (1 << 16)]
        dist = np.abs(blk[:, None] - vals[None, :])
        best = dist.min(axis=1, keepdims=True)
        cand = dist == best
        # among equally near codes take the one with an even mantissa (code & 1 == 0)
        even = cand & ((codes[None, :] & 1) == 0)
        pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
        out[s:s + blk.size] = codes[pick]
    out[a >= 448.0] = 0x7E
    out |= np.where(np.signbit(y), 0x80, 0).astype(np.uint8)
    return out


def test_nearest_search_agrees_with_brute_force():
    y = np.abs(_structured_floats())
    y = y[y <= 448.0]
    assert (_nearest_code_sorted(y.astype(np.float64)) == _brute_force_encode(y)).all()


def test_encode_brute_force_structured():
    y = _structured_floats()
    y = y[np.abs(y) < 1e6]
    got = oracle.e4m3_encode(y)
    want = _brute_force_encode(y)
    bad = np.nonzero(got != want)[0]
    assert bad.size == 0, (y[bad[:5]], got[bad[:5]], want[bad[:5]])


def test_encode_matches_torch_below_overflow():
    # torch rounds to nearest even and maps |y| >= 464 to NaN instead of saturating,
    # so compare only below that.
    y = _structured_floats()
    y = y[np.abs(y) < 464.0]
    got = oracle.e4m3_encode(y)
    t = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert (got == t).all()


def test_encode_saturation_sign_and_nan():
    y = np.array([448, 449, 463.99, 464, 1e30, np.inf, -1e30, -np.inf, -0.0, 0.0, -1e-30,
                  np.nan], dtype=np.float32)
    got = oracle.e4m3_encode(y)
    assert list(got[:8]) == [0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0x7E, 0xFE, 0xFE]
    assert list(got[8:11]) == [0x80, 0x00, 0x80]
    assert got[11] == 0x7F


def test_encode_ties_to_even_examples():
    # 1.0625 is halfway between 1.0 (0x38, even) and 1.125 (0x39): goes to 1.0.
    # 1.1875 is halfway between 1.125 (0x39) and 1.25 (0x3A, even): goes to 1.25.
    # 2^-10 is halfway between 0 and the smallest subnormal 2^-9: goes to 0.
    # 3*2^-10 is halfway between 2^-9 (0x01) and 2^-8 (0x02, even): goes to 2^-8.
    y = np.array([1.0625, 1.1875, 2.0 ** -10, 3 * 2.0 ** -10], dtype=np.float32)
    assert list(oracle.e4m3_encode(y)) == [0x38, 0x3A, 0x00, 0x02]


# ------------------------------------------------------------------ casts to output types

def test_round_f32_matches_numpy():
    x = np.random.RandomState(1).standard_normal(200000) * np.exp(np.random.RandomState(2).uniform(-60, 60, 200000))
    got = oracle.round_to(x, oracle.F32)
    assert (got == x.astype(np.float32).astype(np.float64)).all()


def test_round_f16_matches_numpy():
    rs = np.random.RandomState(3)
    x = rs.standard_normal(200000) * np.exp(rs.uniform(-25, 12, 200000))
    x = x[np.abs(x) < 65504]
    got = oracle.round_to(x, oracle.F16)
    assert (got == x.astype(np.float16).astype(np.float64)).all()


def _nearest_bf16_exact(x: float) -> float:
    """Exact rational nearest bf16 (8 significant bits, min normal 2^-126), ties to even."""
    fx = Fraction(x)
    if fx == 0:
        return x
    a = abs(fx)
    e = 0
    while a >= 2:
        a /= 2
        e += 1
    while a < 1:
        a *= 2
        e -= 1
    e = max(e, -126)
    q = Fraction(2) ** (e - 7)
    n = abs(fx) / q
    lo = n.numerator // n.denominator
    rem = n - lo
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and lo % 2 == 1):
        lo += 1
    v = float(lo * q)
    return -v if fx < 0 else v


def test_round_bf16_exact_nearest():
    rs = np.random.RandomState(4)
    x = rs.standard_normal(3000) * np.exp(rs.uniform(-30, 30, 3000))
    got = oracle.round_to(x, oracle.BF16)
    want = np.array([_nearest_bf16_exact(float(v)) for v in x])
    assert (got == want).all()


def test_round_bf16_ties_and_double_rounding_trap():
    x = np.array([1 + 2.0 ** -8,                 # tie -> 1.0 (even)
                  1 + 3 * 2.0 ** -8,             # tie -> 1 + 2^-6 (even)
                  1 + 2.0 ** -8 + 2.0 ** -30,    # just above the tie -> 1 + 2^-7
                  -(1 + 2.0 ** -8 + 2.0 ** -30)])
    got = oracle.round_to(x, oracle.BF16)
    assert list(got) == [1.0, 1 + 2.0 ** -6, 1 + 2.0 ** -7, -(1 + 2.0 ** -7)]
    # going through float first would give 1.0 for the third value (it rounds to the
    # tie 1 + 2^-8 first), which is exactly what a one-step cast must avoid
    via_float = torch.tensor(np.float32(x[2])).to(torch.bfloat16).item()
    assert via_float == 1.0


def test_load_fp16_and_bf16_decoding():
    h = np.random.RandomState(5).standard_normal(1000).astype(np.float16)
    h[:3] = [np.float16(6e-8), np.float16(-0.0), np.float16(65504)]
    for i in range(h.size):
        assert oracle.load_elem(h, oracle.F16, i) == float(h[i])
    b = torch.randn(1000, dtype=torch.float32).to(torch.bfloat16)
    bits = b.view(torch.int16).numpy().view(np.uint16)
    ref = b.to(torch.float64).numpy()
    for i in range(0, 1000, 7):
        assert oracle.load_elem(bits, oracle.BF16, i) == ref[i]


def _nearest_code_sorted(a: np.ndarray) -> np.ndarray:
    """Code of the E4M3 value nearest to each magnitude a in [0, 448], ties to the even
    code, by bisection over the 127 ascending non-negative finite values (the same
    definition as _brute_force_encode, fast enough for a billion inputs)."""
    vals = _table()[:127]
    i = np.minimum(np.searchsorted(vals, a, side="left"), 126)   # vals[i - 1] < a <= vals[i]
    lo = np.maximum(i - 1, 0)
    d_lo, d_hi = a - vals[lo], vals[i] - a                       # exact in double
    return np.where(d_hi < d_lo, i, np.where(d_lo < d_hi, lo, np.where(i % 2 == 0, i, lo))).astype(np.uint8)


def test_encode_exhaustive_against_torch():
    """Every non-negative FP32 value up to 448 (all 1,138,753,537 bit patterns from +0 to
    448.0), encoded by the oracle, by torch's independent float8_e4m3fn cast (RNE) and by
    a nearest-value search with ties to even; plus the sign-flipped patterns of a
    strided subset."""
    top = int(np.array(448.0, dtype=np.float32).view(np.uint32))
    step = 1 << 24
    for lo in range(0, top + 1, step):
        bits = np.arange(lo, min(lo + step, top + 1), dtype=np.uint32)
        y = bits.view(np.float32)
        ref = torch.from_numpy(y).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
        got = oracle.e4m3_encode(y)
        bad = np.flatnonzero(got != ref)
        assert bad.size == 0, f"{bad.size} mismatches from {y[bad[0]]!r}: {got[bad[0]]:#x} vs {ref[bad[0]]:#x}"
        near = _nearest_code_sorted(y.astype(np.float64))
        bad = np.flatnonzero(got != near)
        assert bad.size == 0, f"{bad.size} off the nearest code from {y[bad[0]]!r}: {got[bad[0]]:#x} vs {near[bad[0]]:#x}"
    neg = -(np.arange(0, top + 1, 997, dtype=np.uint32).view(np.float32))
    ref = torch.from_numpy(neg).to(torch.float8_e4m3fn).view(torch.uint8).numpy()
    assert np.array_equal(oracle.e4m3_encode(neg), ref)
