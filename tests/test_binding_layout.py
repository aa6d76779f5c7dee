"""Host-side logic of the Python binding: the (layout, leading dimension) it hands the
C ABI for strided torch views, including the single-row/column operands that grouped
calls read in the groups' shared layout. CPU tensors only (no library call)."""
import pytest
import torch

import sm_gemm_b200 as sg


def test_layout_of_plain_and_transposed_views():
    a = torch.zeros(64, 40)
    assert sg._layout(a, "a") == (sg.ROW_MAJOR, 40)
    assert sg._layout(a.t(), "a") == (sg.COL_MAJOR, 40)
    padded = torch.zeros(64, 48)[:, :40]                       # row pitch 48
    assert sg._layout(padded, "a") == (sg.ROW_MAJOR, 48)
    assert sg._layout(padded.t(), "a") == (sg.COL_MAJOR, 48)


def test_layout_rejects_non_unit_strides():
    with pytest.raises(ValueError):
        sg._layout(torch.zeros(8, 8)[::2, ::2], "a")
    with pytest.raises(ValueError):
        sg._layout(torch.zeros(2, 3, 4), "a")


def test_layout_as_reads_single_rows_and_columns_in_either_layout():
    row = torch.zeros(1, 64)                                   # one row, contiguous
    assert sg._layout_as(row, "r", sg.ROW_MAJOR) == 64
    # read as column-major its column pitch is real (1 element); the C ABI rejects that
    # pitch (not 16 bytes), so the binding passes it on rather than inventing another
    assert sg._layout_as(row, "r", sg.COL_MAJOR) == 1
    padded_row = torch.zeros(64, 8)[:, :1].t()                 # one row, column pitch 8
    assert sg._layout_as(padded_row, "r", sg.COL_MAJOR) == 8
    col = torch.zeros(64, 8)[:, :1]                            # one column of a pitch-8 buffer
    assert sg._layout_as(col, "c", sg.ROW_MAJOR) == 8
    with pytest.raises(ValueError):                            # its 64 elements are 8 apart
        sg._layout_as(col, "c", sg.COL_MAJOR)
    dense_col = torch.zeros(64, 1)                             # 64 consecutive elements
    assert sg._layout_as(dense_col, "c", sg.COL_MAJOR) == 64  # unused pitch: >= rows
    with pytest.raises(ValueError):
        sg._layout_as(torch.zeros(4, 8), "x", sg.COL_MAJOR)    # a true row-major matrix


class _RecordingLib:
    """Stands in for the C library: records the arguments of gemm_bf16_grouped."""

    def __init__(self):
        self.calls = []

    def smgemm_grouped_workspace_size(self, G):
        return 4096

    def gemm_bf16_grouped(self, *args):
        # The host arrays are only valid during the call (as for the library, which
        # copies what it needs before returning): decode them now.
        (G, Ms, Ns, Ks, pA, adt, lay_a, ldas, pB, lay_b, ldbs, pbias, bdt, act, pC, cdt, ldcs, ws, wsb, st) = args
        as_list = lambda arr: [arr[i] for i in range(G)]
        self.calls.append(dict(G=G, M=as_list(Ms), N=as_list(Ns), K=as_list(Ks), A=as_list(pA), adt=adt,
                               lay_a=lay_a, lda=as_list(ldas), B=as_list(pB), lay_b=lay_b, ldb=as_list(ldbs),
                               bias=None if pbias is None else as_list(pbias), bdt=bdt, act=act, C=as_list(pC),
                               cdt=cdt, ldc=as_list(ldcs), ws=ws, wsb=wsb))
        return sg.OK


def _host_only(monkeypatch, rec):
    """Route the binding to a stand-in library and accept CPU tensors (the device check
    is tested on its own below)."""
    monkeypatch.setattr(sg, "_lib", rec)
    monkeypatch.setattr(sg, "_stream", lambda s: 0)
    monkeypatch.setattr(sg, "_device", lambda *ts: None)
    monkeypatch.setattr(sg, "_current_device", lambda: None)


def _grouped_args(monkeypatch, *a, **kw):
    rec = _RecordingLib()
    _host_only(monkeypatch, rec)
    res = sg.gemm_bf16_grouped(*a, **kw)
    (d,) = rec.calls
    return res, d


def test_grouped_marshalling_padded_views(monkeypatch):
    """Sizes, pitches, pointers, dtypes and the shared layouts handed to the C ABI."""
    bf = torch.bfloat16
    As = [torch.zeros(3, 72, dtype=bf)[:, :64], torch.zeros(5, 136, dtype=bf)[:, :128]]   # row-major, padded
    Bs = [torch.zeros(40, 64, dtype=bf)[:, :64].t()[:, :24], torch.zeros(16, 136, dtype=bf)[:, :128].t()]  # col
    biases = [torch.zeros(24, dtype=torch.float32), None]
    outs = [torch.zeros(3, 32, dtype=torch.float32)[:, :24], torch.zeros(5, 16, dtype=torch.float32)]
    ws = torch.zeros(8192, dtype=torch.uint8)
    res, d = _grouped_args(monkeypatch, As, Bs, biases=biases, act="silu", outs=outs, workspace=ws)
    assert res == outs
    assert (d["G"], d["M"], d["N"], d["K"]) == (2, [3, 5], [24, 16], [64, 128])
    assert (d["lay_a"], d["lda"]) == (sg.ROW_MAJOR, [72, 136])
    assert (d["lay_b"], d["ldb"]) == (sg.COL_MAJOR, [64, 136])
    assert d["ldc"] == [32, 16]
    assert d["A"] == [t.data_ptr() for t in As] and d["B"] == [t.data_ptr() for t in Bs]
    assert d["C"] == [t.data_ptr() for t in outs]
    assert d["bias"] == [biases[0].data_ptr(), None] and d["bdt"] == sg.F32
    assert (d["adt"], d["cdt"], d["act"]) == (sg.BF16, sg.F32, sg.ACTS["silu"])
    assert (d["ws"], d["wsb"]) == (ws.data_ptr(), 8192)


def test_grouped_marshalling_single_rows_and_allocated_outputs(monkeypatch):
    """A one-row A takes the layout of the other groups (column-major here); outputs
    are allocated with the requested type when not given; no biases."""
    h = torch.float16
    a0 = torch.zeros(64, 8, dtype=h)[:, :1].t()            # one row [1, 64], column pitch 8
    a1 = torch.zeros(96, 48, dtype=h)[:, :40].t()          # [40, 96] column-major, pitch 48
    As = [a0, a1]
    Bs = [torch.zeros(64, 8, dtype=h), torch.zeros(96, 16, dtype=h)]
    with pytest.raises(ValueError):                        # K of group 1 does not match its B
        _grouped_args(monkeypatch, [a0, torch.zeros(48, 40, dtype=h)], Bs)
    res, d = _grouped_args(monkeypatch, As, Bs, out_dtype=torch.bfloat16, workspace=torch.zeros(16, dtype=torch.uint8))
    assert [tuple(r.shape) for r in res] == [(1, 8), (40, 16)] and all(r.dtype == torch.bfloat16 for r in res)
    assert d["lay_a"] == sg.COL_MAJOR and d["lda"] == [8, 48]
    assert d["lay_b"] == sg.ROW_MAJOR and d["ldb"] == [8, 16]
    assert d["bias"] is None and d["bdt"] == 0 and d["cdt"] == sg.BF16 and d["adt"] == sg.F16
    assert d["K"] == [64, 96] and d["M"] == [1, 40] and d["N"] == [8, 16]


def test_workspace_cache_per_stream_and_growth(monkeypatch):
    """Cached workspaces: shared by calls on one stream, distinct per stream (calls on
    different streams may overlap), and an outgrown one is kept alive, not freed."""
    import ctypes
    monkeypatch.setattr(sg, "_ws_cache", {})
    monkeypatch.setattr(sg, "_ws_retired", [])
    dev = torch.device("cpu", 0)
    assert sg._workspace(0, dev, 0) == (None, 0)
    w1, n1 = sg._workspace(1000, dev, 0)
    assert n1 == w1.numel() >= 1 << 20
    assert sg._workspace(5000, dev, 0)[0] is w1                 # same stream: reused
    w2, _ = sg._workspace(1000, dev, 0x1234)                      # another stream: its own
    assert w2 is not w1
    assert sg._workspace(1000, dev, ctypes.c_void_p(0x1234))[0] is w2
    w3, n3 = sg._workspace(n1 + 1, dev, 0)                        # outgrown: at least doubled
    assert w3 is not w1 and n3 >= 2 * n1 and sg._ws_retired == [w1]


class _FakeTensor:
    def __init__(self, cuda, dev):
        self.is_cuda, self._dev = cuda, dev

    def get_device(self):
        return self._dev


def test_device_check():
    """Pointers of host tensors or of another GPU's tensors would be dereferenced by the
    kernels: the binding refuses them before calling the library."""
    a, b, other = _FakeTensor(True, 0), _FakeTensor(True, 0), _FakeTensor(True, 1)
    assert sg._device(a, None, b) == 0
    assert sg._device(None) is None
    with pytest.raises(ValueError):
        sg._device(a, _FakeTensor(False, -1))
    with pytest.raises(ValueError):
        sg._device(a, other)
    with pytest.raises(ValueError):
        sg._device(torch.zeros(2, 2))                       # a real host tensor


class _CountingLib:
    """Stand-in library that counts calls; the size queries return a small workspace."""

    def __init__(self):
        self.calls = 0

    def __getattr__(self, name):
        if name.endswith("workspace_size"):
            return lambda *a: 0
        def call(*a):
            self.calls += 1
            return sg.OK
        return call


def test_shape_and_dtype_checks_refuse_before_the_library(monkeypatch):
    """Tensors smaller than the sizes say, or of the wrong type, never reach the library
    (the kernels would read or write past them)."""
    rec = _CountingLib()
    _host_only(monkeypatch, rec)
    bf = torch.bfloat16
    A, B = torch.zeros(8, 16, dtype=bf), torch.zeros(16, 24, dtype=bf)
    bad_calls = [
        lambda: sg.gemm_bf16(A, B, bias=torch.zeros(23, dtype=bf)),                       # bias too short
        lambda: sg.gemm_bf16(A, B, bias=torch.zeros(48, dtype=bf)[::2]),                  # bias strided
        lambda: sg.gemm_bf16(A, B, out=torch.zeros(8, 23, dtype=bf)),                     # out too small
        lambda: sg.gemm_bf16(A, B, out=torch.zeros(8, 24, dtype=torch.int32)),            # out type
        lambda: sg.gemm_bf16(A, B, bias=torch.zeros(24, dtype=torch.int64)),              # bias type
        lambda: sg.gemm_bf16_fp8out(A, B, scales=torch.zeros(1, 7)),                      # scales shape
        lambda: sg.gemm_bf16_fp8out(A, B, Q=torch.zeros(8, 24)),                          # codes type
        lambda: sg.gemm_bf16_logsoftmax(A, B, out=torch.zeros(8, 24, dtype=bf)),          # not float32
        lambda: sg.quantize_fp8_blockwise(torch.zeros(4, 256, dtype=bf)),                 # X type
        lambda: sg.quantize_fp8_blockwise(torch.zeros(4, 256), Q=torch.zeros(4, 255, dtype=torch.uint8)),
        lambda: sg.quantize_fp8_blockwise(torch.zeros(4, 256), scales=torch.zeros(2, 3)),
        lambda: sg.gemm_fp8_blockscaled(torch.zeros(8, 256, dtype=torch.uint8), torch.zeros(1, 8),
                                        torch.zeros(24, 256, dtype=torch.uint8), torch.zeros(2, 1)),  # sa shape
        lambda: sg.gemm_fp8_blockscaled(torch.zeros(8, 256, dtype=torch.uint8), torch.zeros(2, 8, dtype=bf),
                                        torch.zeros(24, 256, dtype=torch.uint8), torch.zeros(2, 1)),  # sa type
        lambda: sg.gemm_bf16_grouped([A], [B], outs=[torch.zeros(8, 20, dtype=bf)]),       # group output
        lambda: sg.gemm_bf16_grouped([A, A], [B, B], biases=[torch.zeros(24), torch.zeros(24, dtype=bf)]),
    ]
    for i, f in enumerate(bad_calls):
        with pytest.raises(ValueError):
            f()
        assert rec.calls == 0, f"call {i} reached the library"
    # the well-formed versions do reach it
    sg.gemm_bf16(A, B, bias=torch.zeros(24, dtype=bf), out=torch.zeros(8, 24))
    sg.gemm_bf16_fp8out(A, B)
    sg.gemm_bf16_logsoftmax(A, B)
    sg.quantize_fp8_blockwise(torch.zeros(4, 256))
    sg.quantize_fp8_blockwise(torch.zeros(256, 4), 128)
    sg.gemm_fp8_blockscaled(torch.zeros(8, 256, dtype=torch.uint8), torch.zeros(2, 8),
                            torch.zeros(24, 256, dtype=torch.uint8), torch.zeros(2, 1))
    sg.gemm_bf16_grouped([A, A], [B, B], biases=[torch.zeros(24), None])
    assert rec.calls == 7


def test_single_row_output_pitch_is_rounded(monkeypatch):
    """A one-row output's pitch addresses nothing, so an odd width (a one-token LM head
    over an odd vocabulary) gets a 16-element pitch instead of an alignment error;
    outputs of several rows keep their real pitch."""
    seen = []

    class Lib(_CountingLib):
        def gemm_bf16(self, *a):
            seen.append(a[15])
            return sg.OK

    _host_only(monkeypatch, Lib())
    bf = torch.bfloat16
    sg.gemm_bf16(torch.zeros(1, 16, dtype=bf), torch.zeros(16, 50257, dtype=bf), out_dtype=torch.float32)
    sg.gemm_bf16(torch.zeros(2, 16, dtype=bf), torch.zeros(16, 24, dtype=bf))
    assert seen == [50272, 24]


def test_prepared_grouped_call_marshals_once(monkeypatch):
    """GroupedGemm builds the same arguments as gemm_bf16_grouped and each call passes
    them unchanged (only the stream handle is refreshed)."""
    rec = _RecordingLib()
    _host_only(monkeypatch, rec)
    bf = torch.bfloat16
    As = [torch.zeros(16 * (g + 1), 32, dtype=bf) for g in range(3)]
    Bs = [torch.zeros(32, 24, dtype=bf) for _ in range(3)]
    outs = [torch.zeros(16 * (g + 1), 24, dtype=bf) for g in range(3)]
    ws = torch.zeros(64, dtype=torch.uint8)
    sg.gemm_bf16_grouped(As, Bs, outs=outs, workspace=ws, act="gelu_tanh")
    pg = sg.GroupedGemm(As, Bs, outs=outs, workspace=ws, act="gelu_tanh")
    assert pg() is pg.outs and pg() is pg.outs
    one_shot, *prepared = rec.calls
    assert len(prepared) == 2
    for d in prepared:
        assert d == one_shot


def test_layout_accepts_empty_operands_of_any_strides():
    """An empty operand (M = 0 or K = 0; numpy gives such arrays zero strides) is read
    by nothing, so it fits either layout, with a 16-byte leading dimension."""
    import numpy as np
    e = torch.from_numpy(np.zeros((0, 456), dtype=np.float32)[:, :])
    z = torch.from_numpy(np.ones((6, 1), dtype=np.float32)[:, :0])
    for t in (e, z, torch.zeros(0, 0)):
        lay, ld = sg._layout(t, "t")
        assert lay == sg.ROW_MAJOR and ld % 8 == 0 and ld >= max(t.shape[1], 1)
        assert sg._layout_as(t, "t", sg.ROW_MAJOR) % 8 == 0
        assert sg._layout_as(t, "t", sg.COL_MAJOR) % 8 == 0
