"""Seeded synthetic inputs for the GEMM workloads.

This module is shared by the tests, ``bench.py`` and the oracle checks. It holds
no GEMM, quantisation or epilogue arithmetic: only a counter-based random stream
(splitmix64 -> uniform double in [0, 1) -> Box-Muller normals) and the shapes and
value distributions of the workloads. Every value is a pure function of
``(seed, tensor_id, element index)``, so any sub-block can be regenerated alone.

Workload shapes follow the pages: the 7B-style FFN (d_model 4096, d_ff 16384,
batch 1 x seq 1024) of "从一次深夜的算力账单说起：为什么我们要死磕GEMM" (kwkr.cn),
section 2.1, the thin-and-tall LM head of the same page, section 7.2, and the
4096^3 square GEMM of the DeepGEMM kernel-library walkthrough (zwxr.cn), section 3.4.
"""
from __future__ import annotations

import math
import os
from concurrent.futures import ThreadPoolExecutor

import numpy as np

_GOLDEN = np.uint64(0x9E3779B97F4A7C15)
_M1 = np.uint64(0xBF58476D1CE4E5B9)
_M2 = np.uint64(0x94D049BB133111EB)
_CHUNK = 1 << 22


def _mix(z: np.ndarray) -> np.ndarray:
    """The splitmix64 finaliser (Steele, Lea, Flood 2014), on uint64 arrays (wraps mod 2^64)."""
    z = (z ^ (z >> np.uint64(30))) * _M1
    z = (z ^ (z >> np.uint64(27))) * _M2
    return z ^ (z >> np.uint64(31))


def stream_key(seed: int, tensor_id: int) -> int:
    """64-bit key of the sub-stream for one tensor of one workload."""
    with np.errstate(over="ignore"):
        z = np.array([(seed * 0x100000001B3 + tensor_id * 0xD1B54A32D192ED03 + 1) & (2**64 - 1)],
                     dtype=np.uint64)
        return int(_mix(z + _GOLDEN)[0])


def _bits(key: int, start: int, count: int) -> np.ndarray:
    """splitmix64 outputs for counters start .. start+count-1 of stream ``key``."""
    with np.errstate(over="ignore"):
        ctr = np.arange(start, start + count, dtype=np.uint64)
        return _mix(np.uint64(key) + (ctr + np.uint64(1)) * _GOLDEN)


def _uniform(key: int, start: int, count: int) -> np.ndarray:
    """Doubles in [0, 1) with 53 random bits."""
    return (_bits(key, start, count) >> np.uint64(11)).astype(np.float64) * (2.0 ** -53)


def _normal_chunk(key: int, start: int, count: int) -> np.ndarray:
    """Standard normals for element indices start .. start+count-1 (Box-Muller on pairs)."""
    p0 = start // 2
    p1 = (start + count + 1) // 2
    u = _uniform(key, 2 * p0, 2 * (p1 - p0)).reshape(-1, 2)
    r = np.sqrt(-2.0 * np.log1p(-u[:, 0]))
    t = 2.0 * math.pi * u[:, 1]
    z = np.empty((p1 - p0) * 2, dtype=np.float64)
    z[0::2] = r * np.cos(t)
    z[1::2] = r * np.sin(t)
    off = start - 2 * p0
    return z[off:off + count]


def _parallel_fill(n: int, fn) -> np.ndarray:
    out = np.empty(n, dtype=np.float32)
    starts = list(range(0, n, _CHUNK))

    def work(s):
        c = min(_CHUNK, n - s)
        out[s:s + c] = fn(s, c)

    if len(starts) <= 1:
        for s in starts:
            work(s)
    else:
        with ThreadPoolExecutor(max_workers=min(len(starts), os.cpu_count() or 1)) as ex:
            list(ex.map(work, starts))
    return out


def normal(seed: int, tensor_id: int, shape, std: float = 1.0) -> np.ndarray:
    """float32 array of N(0, std^2) values (std is the standard deviation)."""
    n = int(np.prod(shape))
    key = stream_key(seed, tensor_id)
    return _parallel_fill(n, lambda s, c: (std * _normal_chunk(key, s, c))).reshape(shape)


def uniform(seed: int, tensor_id: int, shape, lo: float = -1.0, hi: float = 1.0) -> np.ndarray:
    """float32 array of U[lo, hi) values."""
    n = int(np.prod(shape))
    key = stream_key(seed, tensor_id)
    return _parallel_fill(n, lambda s, c: lo + (hi - lo) * _uniform(key, s, c)).reshape(shape)


def normal_with_outliers(seed: int, tensor_id: int, shape, frac: float = 0.01,
                         factor: float = 50.0) -> np.ndarray:
    """N(0,1) values where an independent Bernoulli(frac) draw per entry scales it by ``factor``.

    The Bernoulli draws come from the sub-stream ``tensor_id + 1000``.
    """
    n = int(np.prod(shape))
    key = stream_key(seed, tensor_id)
    okey = stream_key(seed, tensor_id + 1000)

    def fn(s, c):
        z = _normal_chunk(key, s, c)
        hit = _uniform(okey, s, c) < frac
        return np.where(hit, z * factor, z)

    return _parallel_fill(n, fn).reshape(shape)


def integers(seed: int, tensor_id: int, shape, lo: int, hi: int) -> np.ndarray:
    """float32 array of integers uniform in [lo, hi] (exact in every input dtype used here)."""
    u = uniform(seed, tensor_id, shape, 0.0, 1.0).astype(np.float64)
    return (lo + np.floor(u * (hi - lo + 1))).clip(lo, hi).astype(np.float32)


# --------------------------------------------------------------------------------------
# Workload recipes. Each returns float32 numpy arrays in their STORAGE orientation;
# the caller casts them to the input dtype (round to nearest even) where needed.
# --------------------------------------------------------------------------------------

SEEDS = {"tiny_fp16": 0, "square_bf16": 1, "ffn_pair": 2, "fp8_blockscaled": 3, "lm_head": 4, "grouped": 5}


def tiny_fp16():
    """A[64,64], B[64,64] row-major, U[-1,1], seed 0."""
    s = SEEDS["tiny_fp16"]
    return {"A": uniform(s, 0, (64, 64)), "B": uniform(s, 1, (64, 64))}


def square_bf16(n: int = 4096):
    """A[n,n] row-major; B column-major, stored as Bt[N,K] (K contiguous); N(0,1)."""
    s = SEEDS["square_bf16"]
    return {"A": normal(s, 0, (n, n)), "Bt": normal(s, 1, (n, n))}


def ffn_pair(tokens: int = 1024, d_model: int = 4096, d_ff: int = 16384):
    """X[tokens,d_model] N(0,1); W1[d_model,d_ff], W2[d_ff,d_model] N(0,0.02), row-major
    as written; b1[d_ff] N(0,0.01)."""
    s = SEEDS["ffn_pair"]
    return {"X": normal(s, 0, (tokens, d_model)),
            "W1": normal(s, 1, (d_model, d_ff), 0.02),
            "b1": normal(s, 2, (d_ff,), 0.01),
            "W2": normal(s, 3, (d_ff, d_model), 0.02)}


def ffn_backward(tokens: int = 1024, d_model: int = 4096, d_ff: int = 16384):
    """The FFN layer's X and W1 (same streams as ffn_pair) and an upstream gradient
    dH[tokens,d_ff] N(0,1): dX = dH W1^T and dW1 = X^T dH."""
    s = SEEDS["ffn_pair"]
    return {"X": normal(s, 0, (tokens, d_model)),
            "W1": normal(s, 1, (d_model, d_ff), 0.02),
            "dH": normal(s, 4, (tokens, d_ff))}


def grouped_experts(tokens=(128, 256, 384, 512, 640, 768, 896, 1024), d_model: int = 4096, d_out: int = 4096):
    """One small GEMM per group g: X_g[tokens[g], d_model] N(0,1) times W_g[d_model, d_out]
    N(0,0.02) row-major (the shape of routing tokens to several weight matrices)."""
    s = SEEDS["grouped"]
    return {"X": [normal(s, g, (m, d_model)) for g, m in enumerate(tokens)],
            "W": [normal(s, 100 + g, (d_model, d_out), 0.02) for g in range(len(tokens))]}


def fp8_blockscaled(m: int = 2048, k: int = 4096, n: int = 16384):
    """A[m,k] and B[k,n] fp32, N(0,1) with 1% of entries scaled x50."""
    s = SEEDS["fp8_blockscaled"]
    return {"A": normal_with_outliers(s, 0, (m, k)), "B": normal_with_outliers(s, 1, (k, n))}


def lm_head(m: int = 16, d_model: int = 4096, vocab: int = 128256):
    """X[m,d_model] N(0,1); W[d_model,vocab] N(0,0.02) row-major as written.

    W does not depend on m (its own sub-stream), so every M shares one weight.
    """
    s = SEEDS["lm_head"]
    return {"X": normal(s, 10 + m, (m, d_model)), "W": normal(s, 1, (d_model, vocab), 0.02)}
