"""Python face of the CPU oracle (``oracle.c``). TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package. It never imports the GPU library, and the
GPU library never imports it. Inputs are numpy arrays (bf16 data is passed as its
raw uint16 bits); outputs are float64 arrays holding values that are exactly
representable in the requested output type.

Every function states the passage of the pages it follows in ``oracle.c``.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_LIB = os.path.join(_HERE, "_oracle.so")
_lock = threading.Lock()
_lib = None

F32, BF16, F16, E4M3, F64 = 0, 1, 2, 3, 4
ACT_NONE, ACT_GELU_TANH, ACT_SILU = 0, 1, 2


def build(force: bool = False) -> str:
    """Compile oracle.c into _oracle.so (gcc, OpenMP, no fast-math, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-shared", "-fPIC", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            P, I64, I = C.c_void_p, C.c_int64, C.c_int
            lib.orc_gemm.argtypes = [I64, I64, I64, P, I, I64, I64, P, I, I64, I64, P, I, I, I,
                                     P, I64, P, I64, P, P]
            lib.orc_gemm.restype = I
            lib.orc_gemm_fp8.argtypes = [I64, I64, I64, P, P, P, P, P, I, I, I, P, I64, P, I64, P, P]
            lib.orc_gemm_fp8.restype = I
            lib.orc_quant_1x128.argtypes = [P, I64, I64, I64, I64, P, P]
            lib.orc_quant_128x128.argtypes = [P, I64, I64, I64, I64, P, P]
            lib.orc_e4m3_encode_array.argtypes = [P, I64, P]
            lib.orc_e4m3_decode_array.argtypes = [P, I64, P]
            lib.orc_round_array.argtypes = [P, I64, I, P]
            lib.orc_act.argtypes = [C.c_double, I]
            lib.orc_act.restype = C.c_double
            lib.orc_load.argtypes = [P, I, I64]
            lib.orc_load.restype = C.c_double
            _lib = lib
    return _lib


def _ptr(a):
    return None if a is None else a.ctypes.data_as(C.c_void_p)


def _dtype_code(a: np.ndarray, declared):
    if declared is not None:
        return declared
    return {np.dtype(np.float32): F32, np.dtype(np.float16): F16,
            np.dtype(np.float64): F64}[a.dtype]


def _elem_strides(a: np.ndarray):
    return tuple(s // a.itemsize for s in a.strides)


def _index_list(idx, n):
    if idx is None:
        return np.arange(n, dtype=np.int64)
    return np.ascontiguousarray(np.asarray(idx, dtype=np.int64))


def gemm(A, B, *, bias=None, act=ACT_NONE, out_dtype=F32, a_dtype=None, b_dtype=None,
         bias_dtype=None, rows=None, cols=None, want_absacc=False):
    """C[rows, cols] of act(A @ B + bias), FP64 accumulation, one RNE cast to out_dtype.

    A is the logical [M, K] matrix and B the logical [K, N] matrix, as numpy arrays in
    any strides (pass ``X.T`` for a column-major operand). bf16 operands are uint16
    arrays of raw bits with ``a_dtype/b_dtype/bias_dtype = BF16``.
    """
    lib = _load()
    M, K = A.shape
    K2, N = B.shape
    assert K == K2
    r = _index_list(rows, M)
    c = _index_list(cols, N)
    out = np.empty((r.size, c.size), dtype=np.float64)
    acc = np.empty_like(out) if want_absacc else None
    ars, acs = _elem_strides(A)
    brs, bcs = _elem_strides(B)
    bd = None
    if bias is not None:
        bias = np.ascontiguousarray(bias)
        bd = _dtype_code(bias, bias_dtype)
    rc = lib.orc_gemm(M, N, K, _ptr(A), _dtype_code(A, a_dtype), ars, acs,
                      _ptr(B), _dtype_code(B, b_dtype), brs, bcs,
                      _ptr(bias), 0 if bd is None else bd, act, out_dtype,
                      _ptr(r), r.size, _ptr(c), c.size, _ptr(out), _ptr(acc))
    if rc != 0:
        raise MemoryError("oracle scratch allocation failed")
    return (out, acc) if want_absacc else out


def gemm_fp8(qa, sa, qb, sb, *, bias=None, bias_dtype=None, act=ACT_NONE, out_dtype=F32,
             rows=None, cols=None, want_absacc=False):
    """Block-scaled FP8 GEMM from codes qa[M,K], qb[N,K] (uint8, K contiguous) and
    scales sa[KB, M], sb[KB, NB] (float32)."""
    lib = _load()
    qa = np.ascontiguousarray(qa, dtype=np.uint8)
    qb = np.ascontiguousarray(qb, dtype=np.uint8)
    sa = np.ascontiguousarray(sa, dtype=np.float32)
    sb = np.ascontiguousarray(sb, dtype=np.float32)
    M, K = qa.shape
    N, K2 = qb.shape
    assert K == K2
    r = _index_list(rows, M)
    c = _index_list(cols, N)
    out = np.empty((r.size, c.size), dtype=np.float64)
    acc = np.empty_like(out) if want_absacc else None
    bd = None
    if bias is not None:
        bias = np.ascontiguousarray(bias)
        bd = _dtype_code(bias, bias_dtype)
    lib.orc_gemm_fp8(M, N, K, _ptr(qa), _ptr(sa), _ptr(qb), _ptr(sb), _ptr(bias),
                     0 if bd is None else bd, act, out_dtype, _ptr(r), r.size, _ptr(c), c.size,
                     _ptr(out), _ptr(acc))
    return (out, acc) if want_absacc else out


def quant_1x128(X):
    """Activations X[rows, cols] (float32, any strides) -> (Q[rows, cols] uint8, S[KB, rows])."""
    lib = _load()
    X = np.asarray(X, dtype=np.float32)
    rows, cols = X.shape
    rs, cs = _elem_strides(X)
    Q = np.empty((rows, cols), dtype=np.uint8)
    S = np.empty(((cols + 127) // 128, rows), dtype=np.float32)
    lib.orc_quant_1x128(_ptr(X), rows, cols, rs, cs, _ptr(Q), _ptr(S))
    return Q, S


def quant_128x128(X):
    """Weights X[K, N] (float32, any strides) -> (Q[N, K] uint8, S[KB, NB])."""
    lib = _load()
    X = np.asarray(X, dtype=np.float32)
    K, N = X.shape
    rs, cs = _elem_strides(X)
    Q = np.empty((N, K), dtype=np.uint8)
    S = np.empty(((K + 127) // 128, (N + 127) // 128), dtype=np.float32)
    lib.orc_quant_128x128(_ptr(X), K, N, rs, cs, _ptr(Q), _ptr(S))
    return Q, S


def e4m3_encode(y):
    lib = _load()
    y = np.ascontiguousarray(y, dtype=np.float32)
    out = np.empty(y.shape, dtype=np.uint8)
    lib.orc_e4m3_encode_array(_ptr(y), y.size, _ptr(out))
    return out


def e4m3_decode(c):
    lib = _load()
    c = np.ascontiguousarray(c, dtype=np.uint8)
    out = np.empty(c.shape, dtype=np.float64)
    lib.orc_e4m3_decode_array(_ptr(c), c.size, _ptr(out))
    return out


def round_to(x, dtype):
    lib = _load()
    x = np.ascontiguousarray(x, dtype=np.float64)
    out = np.empty_like(x)
    lib.orc_round_array(_ptr(x), x.size, dtype, _ptr(out))
    return out


def act(x: float, which: int) -> float:
    return _load().orc_act(float(x), which)


def load_elem(a: np.ndarray, dtype: int, idx: int) -> float:
    return _load().orc_load(_ptr(np.ascontiguousarray(a)), dtype, idx)


def log_softmax_rows(z):
    """out[m, n] = z[m, n] - lse_m, lse_m = mx_m + log(sum_n exp(z[m, n] - mx_m)),
    mx_m = max_n z[m, n], in FP64: the plain row log-softmax that follows the LM-head
    GEMM ("为什么我们要死磕GEMM", section 7.2). Returns (out, lse)."""
    z = np.asarray(z, dtype=np.float64)
    mx = z.max(axis=1, keepdims=True)
    lse = mx + np.log(np.exp(z - mx).sum(axis=1, keepdims=True))
    return z - lse, lse[:, 0]
