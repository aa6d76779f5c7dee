"""Pins for the oracle's group-scaled FP8 quantiser and its block-scaled FP8 GEMM.

Group scaling follows the DeepGEMM kernel-library walkthrough (zwxr.cn),
section 2.4: one FP32 scale per 1x128 row group (activations) or per 128x128
block (weights), scale = amax/448, codes = E4M3(x/scale); the GEMM accumulates the
code products in high precision and rescales per K-block.

Checks: each code equals an independent brute-force nearest search applied to
numpy's IEEE float32 division x/scale; per-group invariants (the largest code is
+-448 unless the group is all zero, signs are kept, the dequantisation error is at
most half a code spacing); closed forms (constant groups, powers of two, all-zero
groups); the transposed code layout of the weight mode; and the FP8 GEMM against
numpy int64 matmul (unit scales, integer codes) and power-of-two scales.
"""
import numpy as np
import pytest

import oracle
import synth

DEC = oracle.e4m3_decode(np.arange(256, dtype=np.uint8))
FIN_CODES = np.array([c for c in range(128) if np.isfinite(DEC[c])], dtype=np.uint8)
FIN_VALS = DEC[FIN_CODES]


def _nearest_codes(y: np.ndarray) -> np.ndarray:
    a = np.abs(y.astype(np.float64)).ravel()
    dist = np.abs(a[:, None] - FIN_VALS[None, :])
    best = dist.min(axis=1, keepdims=True)
    cand = dist == best
    even = cand & ((FIN_CODES[None, :] & 1) == 0)
    pick = np.where(even.any(axis=1), even.argmax(axis=1), cand.argmax(axis=1))
    out = FIN_CODES[pick]
    out[a >= 448.0] = 0x7E
    out |= np.where(np.signbit(y.ravel()), 0x80, 0).astype(np.uint8)
    return out.reshape(y.shape)


def _check_groups_1x128(X, Q, S):
    rows, cols = X.shape
    for kb in range((cols + 127) // 128):
        c0, c1 = kb * 128, min(cols, kb * 128 + 128)
        g = X[:, c0:c1]
        amax = np.abs(g).max(axis=1)
        s_want = np.where(amax == 0, np.float32(1.0), amax / np.float32(448.0)).astype(np.float32)
        assert (S[kb] == s_want).all()
        y = (g / S[kb][:, None]).astype(np.float32)            # numpy: IEEE float32 division
        assert (Q[:, c0:c1] == _nearest_codes(y)).all()


def test_quant_1x128_brute_force_and_scales():
    X = synth.normal_with_outliers(21, 0, (37, 300))           # ragged last group (44 wide)
    Q, S = oracle.quant_1x128(X)
    assert Q.shape == (37, 300) and S.shape == (3, 37)
    _check_groups_1x128(X, Q, S)


def test_quant_1x128_column_major_input_same_result():
    X = synth.normal(22, 0, (19, 260))
    Q, S = oracle.quant_1x128(X)
    Qf, Sf = oracle.quant_1x128(np.asfortranarray(X))
    assert (Q == Qf).all() and (S == Sf).all()


def test_quant_invariants():
    X = synth.normal_with_outliers(23, 0, (64, 512))
    Q, S = oracle.quant_1x128(X)
    dq = DEC[Q].reshape(Q.shape)
    for kb in range(4):
        blk = dq[:, kb * 128:(kb + 1) * 128]
        assert (np.abs(blk).max(axis=1) == 448.0).all()         # amax maps onto 448 exactly
    xs = X.astype(np.float64)
    # signs kept (zero codes carry the input's sign bit)
    assert (np.signbit(dq) == np.signbit(xs)).all()
    # |x/s - dec(q)| <= half the code spacing at dec(q)
    y = xs / np.repeat(S.T.astype(np.float64), 128, axis=1)
    spacing = np.where(np.abs(dq) < 2.0 ** -6, 2.0 ** -9,
                       2.0 ** (np.floor(np.log2(np.maximum(np.abs(dq), 2.0 ** -6))) - 3))
    assert (np.abs(y - dq) <= spacing / 2 * (1 + 1e-6)).all()


def test_quant_closed_forms():
    X = np.zeros((3, 256), dtype=np.float32)
    X[0, :128] = -2.5                                  # constant group -> all -448, s = 2.5/448
    # powers of two with amax = 448 * 2^-2: the scale is exactly 2^-2, every x/s is a power
    # of two inside the normal E4M3 range, so the round trip dec(q) * s is exact
    X[1, :128] = 2.0 ** (np.arange(128) % 11 - 5)
    X[1, 7] = 112.0
    # row 2 and the second group of row 0 stay all zero -> scale 1, codes 0
    Q, S = oracle.quant_1x128(X)
    assert (Q[0, :128] == 0xFE).all() and S[0, 0] == np.float32(2.5) / np.float32(448)
    assert S[0, 1] == 0.25                             # S is [group, row]
    assert (DEC[Q[1, :128]] * 0.25 == X[1, :128]).all()
    assert DEC[Q[1, 7]] == 448.0
    assert S[1, 0] == 1.0 and S[0, 2] == 1.0 and (Q[2] == 0).all() and (Q[0, 128:] == 0).all()


def test_quant_128x128_layout_and_brute_force():
    K, N = 300, 200                                    # ragged in both directions
    X = synth.normal_with_outliers(24, 0, (K, N))
    Q, S = oracle.quant_128x128(X)
    assert Q.shape == (N, K) and S.shape == (3, 2)
    for kb in range(3):
        for nb in range(2):
            blk = X[kb * 128:(kb + 1) * 128, nb * 128:(nb + 1) * 128]
            amax = np.abs(blk).max()
            s = np.float32(amax) / np.float32(448.0)
            assert S[kb, nb] == s
            y = (blk / s).astype(np.float32)
            q = _nearest_codes(y)                      # [k, n]
            assert (Q[nb * 128:nb * 128 + blk.shape[1], kb * 128:kb * 128 + blk.shape[0]] == q.T).all()


def test_quant_128x128_column_major_input_same_result():
    X = synth.normal(25, 0, (256, 130))
    Q, S = oracle.quant_128x128(X)
    Qf, Sf = oracle.quant_128x128(np.asfortranarray(X))
    assert (Q == Qf).all() and (S == Sf).all()


# ------------------------------------------------------------------ block-scaled FP8 GEMM

def _int_codes(rs, shape, lo=-8, hi=8):
    """Codes whose decoded values are the integers lo..hi (all exact in E4M3)."""
    v = rs.randint(lo, hi + 1, size=shape).astype(np.float32)
    return oracle.e4m3_encode(v), v.astype(np.int64)


@pytest.mark.parametrize("M,N,K", [(5, 7, 128), (33, 130, 300), (1, 256, 1)])
def test_fp8_gemm_unit_scales_is_integer_matmul(M, N, K):
    rs = np.random.RandomState(M + N + K)
    qa, a = _int_codes(rs, (M, K))
    qb, b = _int_codes(rs, (N, K))
    sa = np.ones(((K + 127) // 128, M), np.float32)
    sb = np.ones(((K + 127) // 128, (N + 127) // 128), np.float32)
    got = oracle.gemm_fp8(qa, sa, qb, sb)
    assert (got == a @ b.T).all()


def test_fp8_gemm_power_of_two_scales_exact():
    rs = np.random.RandomState(9)
    M, N, K = 20, 300, 384
    qa, a = _int_codes(rs, (M, K))
    qb, b = _int_codes(rs, (N, K))
    KB, NB = 3, 3
    ea = rs.randint(-6, 7, size=(KB, M))
    eb = rs.randint(-6, 7, size=(KB, NB))
    sa = (2.0 ** ea).astype(np.float32)
    sb = (2.0 ** eb).astype(np.float32)
    want = np.zeros((M, N))
    for kb in range(KB):
        part = a[:, kb * 128:(kb + 1) * 128] @ b[:, kb * 128:(kb + 1) * 128].T
        want += part * (2.0 ** ea[kb])[:, None] * (2.0 ** eb[kb][np.arange(N) // 128])[None, :]
    got = oracle.gemm_fp8(qa, sa, qb, sb, out_dtype=oracle.F64)
    assert (got == want).all()


def test_fp8_gemm_matches_dequantised_fp64_gemm():
    A = synth.normal_with_outliers(26, 0, (40, 384))
    B = synth.normal_with_outliers(26, 1, (384, 260))
    qa, sa = oracle.quant_1x128(A)
    qb, sb = oracle.quant_128x128(B)
    a_hat = DEC[qa] * np.repeat(sa.T.astype(np.float64), 128, axis=1)[:, :384]
    nb = np.arange(260) // 128
    b_hat = (DEC[qb] * np.repeat(sb.astype(np.float64)[:, nb].T, 128, axis=1)[:, :384]).T
    got, acc = oracle.gemm_fp8(qa, sa, qb, sb, out_dtype=oracle.F64, want_absacc=True)
    want = oracle.gemm(a_hat, b_hat, out_dtype=oracle.F64)
    assert np.all(np.abs(got - want) <= 1e-12 * acc)
    # the dequantised product is close to the unquantised one (FP8 error only)
    full = A.astype(np.float64) @ B.astype(np.float64)
    assert np.abs(got - full).max() / np.abs(full).max() < 0.1
