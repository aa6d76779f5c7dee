"""The FP8 quantiser's division x / s (an FMA sequence after Markstein, "IA-64 and
Elementary Functions", chapter 8) against IEEE single-precision division, on the CPU.

The quantiser computes each code from x / s, where the DeepGEMM kernel-library
walkthrough (zwxr.cn), section 2.4 fixes s = amax / 448 per group and the reading of
the pages is an IEEE division. On the GPU it uses the sequence r = RN(1/s),
y = RN(x r), e = x - y s, q = RN(y + e r) whenever the scale's significand is not all
ones and 2^-90 <= s (otherwise an IEEE division). The claim checked here: under those
conditions q equals the IEEE quotient bit for bit for every quotient E4M3 can tell from
zero (|x / s| > 2^-11), and smaller quotients keep the sign of x and stay at or below
2^-10, so the codes agree. The check runs a plain C restatement of the sequence
(tests/markstein_check.c, libm fmaf) over
  - every significand of x, both signs, in the binades that give quotients near 2^-11,
    near 1 and near 448, for scales with structured significands (one ulp above and
    below a power of two, repeating patterns, one short of all ones);
  - every scale exponent from -90 to 119 with structured significands, and
    pseudo-random x in every quotient binade from 2^-12 to 2^9;
  - the low end s ~ 2^-90 exhaustively in the smallest quotient binades.
It also shows the check can fail: the same sweep finds disagreements for scales
below the 2^-90 limit and for the reciprocal product alone (no residual step).
"""
import ctypes as C
import subprocess

import numpy as np
import pytest

SRC = __file__.replace("test_markstein_division.py", "markstein_check.c")

# Significands (23-bit fields) of the scales: powers of two, one ulp above / below, repeating
# patterns, one short of all ones (all ones itself is excluded by the quantiser).
SIGNIFICANDS = [0x000000, 0x000001, 0x000002, 0x7FFFFE, 0x7FFFFD, 0x400000, 0x555555, 0x2AAAAB, 0x3FFFFF,
                0x7FFF00, 0x00FFFF, 0x123457]


@pytest.fixture(scope="module")
def mk(tmp_path_factory):
    so = tmp_path_factory.mktemp("markstein") / "mk.so"
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-shared", "-fPIC", SRC, "-o", str(so), "-lm"],
                   check=True)
    L = C.CDLL(str(so))
    L.mk_binade.argtypes = [C.c_float, C.c_int, C.c_int, C.POINTER(C.c_uint32)]
    L.mk_binade.restype = C.c_int64
    L.mk_scales.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_uint64]
    L.mk_scales.restype = C.c_int64
    return L


def _scale(exp: int, sig: int) -> float:
    return float(np.array([((exp + 127) << 23) | sig], dtype=np.uint32).view(np.float32)[0])


def _binade_bad(mk, s: float, qexps, mode=0) -> int:
    e = int(np.floor(np.log2(s)))
    first = C.c_uint32()
    return sum(mk.mk_binade(s, e + q, mode, C.byref(first)) for q in qexps)


def test_exhaustive_significands_of_x(mk):
    """Every x significand in the quotient binades 2^-12 .. 2^-10, 2^-1 .. 2^0 and 2^7 .. 2^8
    (quotients up to 448), for each structured scale significand at exponent 0."""
    for sig in SIGNIFICANDS:
        s = _scale(0, sig)
        assert _binade_bad(mk, s, (-12, -11, -10, -1, 0, 7, 8)) == 0, hex(sig)


def test_every_scale_exponent(mk):
    """Scale exponents -90 .. 119 (s * 448 stays finite) with every structured significand,
    2000 pseudo-random x per quotient binade 2^-12 .. 2^9 and both signs."""
    scales = np.array([_scale(e, sig) for e in range(-90, 120) for sig in SIGNIFICANDS], dtype=np.float32)
    assert mk.mk_scales(scales.ctypes.data, scales.size, 2000, 12345) == 0


def test_low_end_of_the_scale_range(mk):
    """s at 2^-90 .. 2^-89 exhaustively in the smallest quotient binades, where the
    residual x - y s is closest to the subnormal range."""
    for sig in SIGNIFICANDS:
        for e in (-90, -89):
            assert _binade_bad(mk, _scale(e, sig), (-12, -11, -10, -9)) == 0, (e, hex(sig))


def test_the_check_detects_wrong_quotients(mk):
    """The same sweeps find disagreements where the sequence is not used: scales below
    2^-90 (the residual underflows), and the reciprocal product without the residual."""
    assert _binade_bad(mk, _scale(-100, 0x266666), (-12, -11, -10, -9)) > 0
    assert _binade_bad(mk, _scale(0, 0x266666), (-1, 0), mode=1) > 0
