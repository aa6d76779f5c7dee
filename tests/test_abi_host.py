"""Host-side tests of the C-ABI library (no GPU needed).

The library must load without a GPU driver and export every function that
include/smgemm.h declares. Argument errors are reported before any CUDA call, so
they are exercised here with fake device addresses. The persistent schedule
(data-parallel tiles + stream-K ranges) is checked through smgemm_schedule_dump:
every (tile, K-block) pair is computed exactly once, segments of one tile are
contiguous in K, and partial tiles use the slots the kernels' fix-up expects.
"""
import ctypes as C
import os
import re
import subprocess

import numpy as np
import pytest
import torch

import sm_gemm_b200 as sg

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "smgemm.h")

# A fake, 16-byte aligned device address: these tests only reach host-side validation.
FAKE = 0x7F0000001000


def _declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"^[A-Za-z_][\w\s\*]*?\b(\w+)\s*\(", text, flags=re.M)) - {"if"})


def test_header_declares_the_abi():
    names = _declared_functions()
    for want in ("gemm_bf16", "gemm_fp8_blockscaled", "quantize_fp8_blockwise", "smgemm_workspace_size",
                 "smgemm_status_string", "smgemm_check"):
        assert want in names


def test_library_exports_every_declared_symbol():
    out = subprocess.run(["nm", "-D", "--defined-only", sg.LIB_PATH], capture_output=True, text=True,
                         check=True).stdout
    exported = {l.split()[-1] for l in out.splitlines() if " T " in l}
    missing = [n for n in _declared_functions() if n not in exported]
    assert not missing, missing
    L = sg.lib()
    for n in _declared_functions():
        assert hasattr(L, n)


def test_library_has_no_driver_dependency():
    out = subprocess.run(["ldd", sg.LIB_PATH], capture_output=True, text=True).stdout
    assert "libcuda.so" not in out


def test_status_strings():
    for s in range(7):
        assert len(sg.status_string(s)) > 0
    assert sg.status_string(99) == "unknown status"


needs_cpu = pytest.mark.skipif(torch.cuda.is_available(),
                               reason="fake-pointer validation tests run only where no GPU can be reached")


def _gemm(M=256, N=256, K=256, A=FAKE, ab=sg.BF16, la=sg.ROW_MAJOR, lda=None, B=FAKE, lb=sg.COL_MAJOR,
          ldb=None, bias=None, bias_dt=sg.F32, act=0, Cp=FAKE, c_dt=sg.BF16, ldc=None, ws=None, wsb=0):
    lda = lda if lda is not None else (K if la == sg.ROW_MAJOR else M)
    ldb = ldb if ldb is not None else (N if lb == sg.ROW_MAJOR else K)
    ldc = ldc if ldc is not None else N
    return sg.lib().gemm_bf16(M, N, K, A, ab, la, lda, B, lb, ldb, bias, bias_dt, act, Cp, c_dt, ldc, ws, wsb,
                              None)


@needs_cpu
def test_gemm_bf16_argument_errors():
    assert _gemm(M=-1) == sg.ERR_INVALID_ARG
    assert _gemm(K=1 << 31) == sg.ERR_INVALID_ARG
    assert _gemm(ab=sg.F32) == sg.ERR_UNSUPPORTED
    assert _gemm(ab=sg.E4M3) == sg.ERR_UNSUPPORTED
    assert _gemm(la=7) == sg.ERR_INVALID_ARG
    assert _gemm(act=9) == sg.ERR_INVALID_ARG
    assert _gemm(c_dt=sg.E4M3) == sg.ERR_INVALID_ARG
    assert _gemm(A=None) == sg.ERR_INVALID_ARG
    assert _gemm(Cp=None) == sg.ERR_INVALID_ARG
    assert _gemm(lda=100) == sg.ERR_INVALID_ARG              # lda < K
    assert _gemm(ldc=100) == sg.ERR_INVALID_ARG              # ldc < N
    assert _gemm(A=FAKE + 2) == sg.ERR_ALIGNMENT
    assert _gemm(lda=260) == sg.ERR_ALIGNMENT                # 520 bytes: not a multiple of 16
    assert _gemm(Cp=FAKE + 8) == sg.ERR_ALIGNMENT
    assert _gemm(N=250, ldc=250) == sg.ERR_ALIGNMENT         # 500 bytes
    assert _gemm(bias=FAKE + 2, bias_dt=sg.F32) == sg.ERR_ALIGNMENT
    assert _gemm(bias=FAKE, bias_dt=9) == sg.ERR_INVALID_ARG


@needs_cpu
def test_empty_shapes_are_noops_and_valid_calls_need_a_device():
    assert _gemm(M=0) == sg.OK
    assert _gemm(N=0, Cp=None) == sg.OK
    # a valid call with no reachable sm_100 device fails cleanly
    assert _gemm() == sg.ERR_CUDA
    assert _gemm(K=0) == sg.ERR_CUDA
    assert sg.lib().smgemm_check(None) == sg.ERR_CUDA
    assert sg.lib().smgemm_selftest_wait_timeout(1000, None) == sg.ERR_CUDA
    assert sg.workspace_size(4096, 4096, 4096) == 0          # unknown device -> 0


@needs_cpu
def test_fp8_and_quant_argument_errors():
    L = sg.lib()
    def fp8(M=256, N=256, K=256, Aq=FAKE, sa=FAKE, Bq=FAKE, sb=FAKE, Cp=FAKE, ldc=256, c_dt=sg.BF16):
        return L.gemm_fp8_blockscaled(M, N, K, Aq, sa, Bq, sb, None, 0, 0, Cp, c_dt, ldc, None, 0, None)
    assert fp8(K=200) == sg.ERR_ALIGNMENT                     # K must be a multiple of 16
    assert fp8(sa=None) == sg.ERR_INVALID_ARG
    assert fp8(Aq=FAKE + 1) == sg.ERR_ALIGNMENT
    assert fp8(sb=FAKE + 2) == sg.ERR_ALIGNMENT
    assert fp8(M=0) == sg.OK
    assert fp8() == sg.ERR_CUDA
    def q(rows=256, cols=256, layout=sg.ROW_MAJOR, ldx=256, g=1, X=FAKE, Q=FAKE, S=FAKE):
        return L.quantize_fp8_blockwise(X, rows, cols, layout, ldx, g, Q, S, None)
    assert q(g=64) == sg.ERR_INVALID_ARG
    assert q(ldx=100) == sg.ERR_INVALID_ARG
    assert q(ldx=258) == sg.ERR_ALIGNMENT
    assert q(X=FAKE + 4) == sg.ERR_ALIGNMENT
    assert q(Q=FAKE + 1) == sg.ERR_ALIGNMENT
    assert q(rows=0) == sg.OK
    assert q() == sg.ERR_CUDA


@needs_cpu
def test_fp8out_and_logsoftmax_argument_errors():
    L = sg.lib()
    def f8(M=256, N=256, K=256, Cq=FAKE, ldc=256, S=FAKE, act=0):
        return L.gemm_bf16_fp8out(M, N, K, FAKE, sg.BF16, sg.ROW_MAJOR, K, FAKE, sg.ROW_MAJOR, N, None, 0, act,
                                  Cq, ldc, S, None, 0, None)
    assert f8(S=None) == sg.ERR_INVALID_ARG
    assert f8(ldc=200) == sg.ERR_INVALID_ARG                  # ldc < N
    assert f8(ldc=264) == sg.ERR_ALIGNMENT                    # not a multiple of 16 codes
    assert f8(Cq=FAKE + 8) == sg.ERR_ALIGNMENT
    assert f8(S=FAKE + 2) == sg.ERR_ALIGNMENT
    assert f8(K=0) == sg.ERR_UNSUPPORTED
    assert f8(act=9) == sg.ERR_INVALID_ARG
    assert f8(M=0) == sg.OK
    assert f8() == sg.ERR_CUDA
    def ls(M=16, N=1000, K=256, ws=FAKE, wsb=1 << 30):
        return L.gemm_bf16_logsoftmax(M, N, K, FAKE, sg.BF16, sg.ROW_MAJOR, K, FAKE, sg.ROW_MAJOR, N, None, 0,
                                      FAKE, N, ws, wsb, None)
    assert ls(M=0) == sg.OK
    assert ls() == sg.ERR_CUDA                                # workspace size needs a device
    assert L.smgemm_logsoftmax_workspace_size(0, 10, 10) == 0


def _grouped(shapes, ab=sg.BF16, la=sg.ROW_MAJOR, lb=sg.ROW_MAJOR, ptr=FAKE, ws=FAKE, wsb=None, act=0,
             c_dt=sg.BF16, ld_pad=0):
    import ctypes as C
    G = len(shapes)
    arr = lambda xs: (C.c_int64 * max(G, 1))(*xs)
    ptrs = lambda: (C.c_void_p * max(G, 1))(*([ptr] * G))
    Ms, Ns, Ks = [s[0] for s in shapes], [s[1] for s in shapes], [s[2] for s in shapes]
    lda = [(k if la == sg.ROW_MAJOR else m) + ld_pad for m, n, k in shapes]
    ldb = [(n if lb == sg.ROW_MAJOR else k) for m, n, k in shapes]
    wsb = sg.lib().smgemm_grouped_workspace_size(G) if wsb is None else wsb
    return sg.lib().gemm_bf16_grouped(G, arr(Ms), arr(Ns), arr(Ks), ptrs(), ab, la, arr(lda), ptrs(), lb, arr(ldb),
                                      None, 0, act, ptrs(), c_dt, arr(Ns), ws, wsb, None)


def test_grouped_workspace_size():
    """Room for one 320-byte record per group (64-byte aligned), plus, where the device
    is known, the partial tiles of a split last wave."""
    L = sg.lib()
    assert L.smgemm_grouped_workspace_size(0) == 0
    sizes = [L.smgemm_grouped_workspace_size(g) for g in (1, 2, 8, 100)]
    for g, n in zip((1, 2, 8, 100), sizes):
        assert n >= g * 320 + 64
    assert sizes == sorted(sizes)


@needs_cpu
def test_grouped_argument_errors():
    good = [(256, 256, 256), (128, 512, 64)]
    assert _grouped([]) == sg.OK
    assert _grouped(good, ab=sg.F32) == sg.ERR_UNSUPPORTED
    assert _grouped(good, act=9) == sg.ERR_INVALID_ARG
    assert _grouped([(256, 256, 256), (-1, 8, 8)]) == sg.ERR_INVALID_ARG
    assert _grouped(good, ld_pad=4) == sg.ERR_ALIGNMENT        # lda * 2 bytes not a multiple of 16
    assert _grouped(good, ptr=FAKE + 2) == sg.ERR_ALIGNMENT
    assert _grouped(good, wsb=16) == sg.ERR_WORKSPACE
    assert _grouped(good, ws=None) == sg.ERR_WORKSPACE
    assert _grouped(good, ws=FAKE + 4) == sg.ERR_ALIGNMENT       # split partials are float4
    assert _grouped(good, ws=FAKE + 8) == sg.ERR_ALIGNMENT
    assert _grouped([(0, 256, 256), (256, 0, 64)]) == sg.ERR_CUDA  # valid: needs a device
    assert _grouped(good) == sg.ERR_CUDA


# ------------------------------------------------------------------ persistent schedule

def _check_schedule(M, N, K, kind=0, layout_a=sg.ROW_MAJOR, sms=148, bk=None):
    d = sg.schedule_dump(M, N, K, kind, layout_a, sms)
    assert d.shape[0] > 0
    ctas = d[:, 0]
    assert ctas.min() == 0 and ctas.max() < sms
    # every (tile, K-block) exactly once
    if bk is None:
        bk = 128 if kind == 1 else (128 if (M <= 64 and layout_a == sg.ROW_MAJOR) else 64)
    kb_total = -(-K // bk)
    seen = {}
    for c, t, mt, nt, k0, k1, slot in d:
        assert 0 <= k0 < k1 <= kb_total
        for kb in range(k0, k1):
            assert (t, kb) not in seen
            seen[(t, kb)] = c
    tiles = sorted({int(t) for t in d[:, 1]})
    assert tiles == list(range(len(tiles)))
    assert len(seen) == len(tiles) * kb_total
    # tile -> (mt, nt) is a bijection onto the tile grid
    coords = {(int(t), int(mt), int(nt)) for _, t, mt, nt, *_ in d}
    assert len({(m, n) for _, m, n in coords}) == len(tiles)
    # a split tile's contributors are consecutive CTAs in K order, and each partial
    # segment's slot is 0 iff it is the first segment of that CTA
    first_seg, seen_dp = {}, set()
    for i, (c, t, mt, nt, k0, k1, slot) in enumerate(d):
        if slot >= 0:
            assert int(c) not in seen_dp                   # a CTA's stream-K range comes first
            first_seg.setdefault(int(c), i)
        else:
            assert k0 == 0 and k1 == kb_total
            seen_dp.add(int(c))
    by_tile = {}
    for i, (c, t, mt, nt, k0, k1, slot) in enumerate(d):
        by_tile.setdefault(int(t), []).append((int(k0), int(c), int(slot), i))
    for t, segs in by_tile.items():
        segs.sort()
        if len(segs) > 1:
            cs = [c for _, c, _, _ in segs]
            assert cs == sorted(cs) and len(set(cs)) == len(cs)
            for k0, c, slot, i in segs:
                assert slot == (0 if first_seg[c] == i else 1)
    # stream-K / split work is balanced: per-CTA K-block counts differ by at most one
    sk = d[d[:, 6] >= 0]
    if sk.size:
        per = np.bincount(sk[:, 0], weights=sk[:, 5] - sk[:, 4])
        per = per[per > 0]
        assert per.max() - per.min() <= 1
    return d


def test_split_tail_plan_square():
    """4096^3 on 74 CTA pairs: 3 whole waves of 256x256 tiles, the 34 tiles of the
    ragged fourth wave split in two K halves over 68 pairs."""
    d = sg.schedule_dump(4096, 4096, 4096, 0, sg.ROW_MAJOR, 148)
    dp = d[d[:, 6] < 0]
    sk = d[d[:, 6] >= 0]
    assert len(dp) == 3 * 74 and len(sk) == 68
    assert set((sk[:, 5] - sk[:, 4]).tolist()) == {32}
    assert sorted(set(sk[:, 4].tolist())) == [0, 32]


@pytest.mark.parametrize("M,N,K", [(4096, 4096, 4096), (1024, 16384, 4096), (1024, 4096, 16384),
                                   (300, 600, 500), (64, 64, 64), (128, 256, 4096), (67, 50, 33)])
def test_schedule_large_covers_each_kblock_once(M, N, K):
    _check_schedule(M, N, K, layout_a=sg.COL_MAJOR if M <= 64 else sg.ROW_MAJOR)


@pytest.mark.parametrize("M", [1, 4, 16, 64])
def test_schedule_skinny_lm_head(M):
    d = _check_schedule(M, 128256, 4096)
    # all 148 SMs get work and no SM has more than one tile (32 K-blocks) above another
    per_cta = np.bincount(d[:, 0], weights=d[:, 5] - d[:, 4], minlength=148)
    assert per_cta.min() > 0 and per_cta.max() - per_cta.min() <= 32


@pytest.mark.parametrize("M,N,K", [(2048, 16384, 4096), (256, 384, 1024), (130, 260, 128)])
def test_schedule_fp8(M, N, K):
    _check_schedule(M, N, K, kind=1)


def test_schedule_small_grid_override(monkeypatch):
    monkeypatch.setenv("SMGEMM_GRID", "3")
    d = _check_schedule(1000, 1000, 1000)
    assert d[:, 0].max() == 2
    monkeypatch.setenv("SMGEMM_SCHED", "sk")
    _check_schedule(300, 300, 3000)
    monkeypatch.setenv("SMGEMM_SCHED", "dp")
    d = _check_schedule(300, 300, 3000)
    assert (d[:, 4] == 0).all()


def test_splitk_override(monkeypatch):
    """SMGEMM_SPLITK=1 keeps every tile whole; SMGEMM_SPLITK=s cuts each tile's K range
    into about s pieces spread over min(P, s T) CTAs, still covering every K-block once."""
    monkeypatch.setenv("SMGEMM_SPLITK", "1")
    d = _check_schedule(1024, 1024, 4096)                 # 4 x 4 pair tiles: a ragged wave otherwise split
    assert (d[:, 6] == -1).all()
    monkeypatch.setenv("SMGEMM_SPLITK", "3")
    d = _check_schedule(512, 512, 4096)                   # 2 x 2 pair tiles -> 12 CTAs
    assert len(set(d[:, 0].tolist())) == 12 and (d[:, 6] >= 0).all()


def test_force_config_override(monkeypatch):
    """SMGEMM_FORCE_CONFIG=single runs M = 16 on one-SM 128 x 256 tiles instead of the
    swap-AB skinny path; =pair puts it on CTA pairs (256 x 256)."""
    M, N, K = 16, 4096, 1024
    skinny = sg.schedule_dump(M, N, K)
    assert len(set(skinny[:, 1].tolist())) == N // 128      # swap-AB: 128 weight columns per tile
    monkeypatch.setenv("SMGEMM_FORCE_CONFIG", "single")
    single = _check_schedule(M, N, K, bk=64)
    assert len(set(single[:, 1].tolist())) == N // 256
    monkeypatch.setenv("SMGEMM_FORCE_CONFIG", "pair")
    pair = _check_schedule(M, N, K, bk=64, sms=74)
    assert len(set(pair[:, 1].tolist())) == N // 256
