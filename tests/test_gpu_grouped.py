"""Grouped GEMM (gemm_bf16_grouped): several independent GEMMs in one launch (the
batching remedy of "为什么我们要死磕GEMM" (kwkr.cn), section 5.3). Every group is checked
against the oracle: in full on ragged shapes in every layout pair (with empty groups,
a K = 0 group and per-group bias), bit for bit on integer-valued inputs, and on sampled
outputs for eight 4096-wide groups of 128..1024 rows."""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import check_tolerance, orc_view, sample_indices, to_dtype

pytestmark = pytest.mark.gpu

SHAPES = [(300, 520, 136), (1, 64, 64), (256, 256, 1024), (0, 128, 64), (77, 40, 0), (640, 1000, 200),
          (129, 8, 72)]


def _operand(x, layout):
    """bf16 CUDA tensor holding x in the given layout: row-major as is; column-major as
    the transposed view of a [cols, ld] buffer whose ld is rows rounded up to 8 (the
    16-byte pitch TMA needs)."""
    t = to_dtype(x, torch.bfloat16)
    if layout == "row":
        return t.cuda()
    rows, cols = t.shape
    ld = max(8, -(-rows // 8) * 8)
    buf = torch.zeros((cols, ld), dtype=torch.bfloat16)
    buf[:, :rows] = t.t()
    return buf.cuda()[:, :rows].t()


@pytest.mark.parametrize("transpose", ["1", "0"])
@pytest.mark.parametrize("la,lb", [("row", "row"), ("row", "col"), ("col", "row"), ("col", "col")])
def test_grouped_ragged_all_layouts(cuda_device, monkeypatch, la, lb, transpose):
    """Ragged groups in every layout pair, with a group's last row of tiles (<= 128 rows)
    run transposed (the default) or padded to 256 rows."""
    monkeypatch.setenv("SMGEMM_GROUPED_TRANSPOSE", transpose)
    As, Bs, bs, Ah, Bh, bh = [], [], [], [], [], []
    for g, (M, N, K) in enumerate(SHAPES):
        a = synth.normal(41, 3 * g, (M, K))
        b = synth.normal(41, 3 * g + 1, (K, N), 0.1)
        As.append(_operand(a, la))
        Bs.append(_operand(b, lb))
        Ah.append(to_dtype(a, torch.bfloat16))
        Bh.append(to_dtype(b, torch.bfloat16))
        bias = to_dtype(synth.normal(41, 3 * g + 2, (N,), 0.5), torch.bfloat16) if g % 2 == 0 else None
        bs.append(None if bias is None else bias.cuda())
        bh.append(bias)
    outs = sg.gemm_bf16_grouped(As, Bs, biases=bs, act="gelu_tanh", out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    for g, (M, N, K) in enumerate(SHAPES):
        if M == 0 or N == 0:
            assert outs[g].numel() == 0
            continue
        a, ad = orc_view(Ah[g])
        b, bd = orc_view(Bh[g])
        kw = {} if bh[g] is None else dict(zip(("bias", "bias_dtype"), orc_view(bh[g])))
        ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, act=oracle.ACT_GELU_TANH, out_dtype=oracle.BF16,
                               want_absacc=True, **kw)
        check_tolerance(outs[g].float().cpu().numpy(), ref, acc, torch.bfloat16, what=f"group {g} {M}x{N}x{K}")


@pytest.mark.parametrize("transpose", ["1", "0"])
def test_grouped_integer_exact_and_deterministic(cuda_device, monkeypatch, transpose):
    monkeypatch.setenv("SMGEMM_GROUPED_TRANSPOSE", transpose)
    shapes = [(200, 136, 264), (512, 384, 128), (33, 520, 64), (384, 264, 200)]
    As, Bs, refs = [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = torch.from_numpy(synth.integers(42, 2 * g, (M, K), -3, 3)).to(torch.bfloat16)
        b = torch.from_numpy(synth.integers(42, 2 * g + 1, (K, N), -3, 3)).to(torch.bfloat16)
        As.append(a.cuda())
        Bs.append(b.cuda())
        av, ad = orc_view(a)
        bv, bd = orc_view(b)
        refs.append(oracle.gemm(av, bv, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32))
    o1 = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    o2 = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    for g in range(len(shapes)):
        assert np.array_equal(o1[g].cpu().numpy(), refs[g].astype(np.float32))
        assert torch.equal(o1[g], o2[g])


def test_grouped_experts_full_size(cuda_device):
    d = synth.grouped_experts()
    Xs = [to_dtype(x, torch.bfloat16) for x in d["X"]]
    Ws = [to_dtype(w, torch.bfloat16) for w in d["W"]]
    outs = sg.gemm_bf16_grouped([x.cuda() for x in Xs], [w.cuda() for w in Ws], out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    assert "path=grouped" in sg.last_config()
    for g, (X, W) in enumerate(zip(Xs, Ws)):
        rows = sample_indices(X.shape[0], 128, 1, 20 + g)
        cols = sample_indices(4096, 256, 1, 40 + g)
        a, ad = orc_view(X)
        b, bd = orc_view(W)
        ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.BF16, rows=rows, cols=cols,
                               want_absacc=True)
        check_tolerance(outs[g].float().cpu().numpy()[np.ix_(rows, cols)], ref, acc, torch.bfloat16,
                        what=f"expert {g}")


def test_grouped_many_small_groups(cuda_device):
    """40 groups of assorted small shapes (many below one tile, some empty): every tile
    of every group must land in its own group's output."""
    rng = np.random.RandomState(7)
    shapes = [(int(rng.choice([0, 1, 8, 64, 136, 256, 300])), int(rng.choice([8, 40, 128, 264])),
               int(rng.choice([16, 64, 200]))) for _ in range(40)]
    As, Bs, Ah, Bh = [], [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = to_dtype(synth.normal(43, 2 * g, (M, K)), torch.bfloat16)
        b = to_dtype(synth.normal(43, 2 * g + 1, (K, N), 0.1), torch.bfloat16)
        Ah.append(a); Bh.append(b); As.append(a.cuda()); Bs.append(b.cuda())
    outs = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    for g, (M, N, K) in enumerate(shapes):
        if M == 0:
            continue
        a, ad = orc_view(Ah[g])
        b, bd = orc_view(Bh[g])
        ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32, want_absacc=True)
        check_tolerance(outs[g].cpu().numpy(), ref, acc, torch.float32, what=f"group {g} {M}x{N}x{K}")


def test_grouped_split_tail_few_tiles(cuda_device):
    """Three single-tile groups with K = 4096 leave most clusters idle, so each tile is
    split along K into pieces summed in fixed order: checked against the oracle and
    bit-identical across calls."""
    shapes = [(256, 256, 4096), (200, 136, 4096), (64, 256, 4096)]
    As, Bs, Ah, Bh = [], [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = to_dtype(synth.normal(44, 2 * g, (M, K)), torch.bfloat16)
        b = to_dtype(synth.normal(44, 2 * g + 1, (K, N), 0.02), torch.bfloat16)
        Ah.append(a); Bh.append(b); As.append(a.cuda()); Bs.append(b.cuda())
    o1 = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    cfg = sg.last_config()
    o2 = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    assert "splits=" in cfg and "splits=0" not in cfg, cfg
    for g in range(len(shapes)):
        a, ad = orc_view(Ah[g])
        b, bd = orc_view(Bh[g])
        ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32, want_absacc=True)
        check_tolerance(o1[g].cpu().numpy(), ref, acc, torch.float32, what=f"group {g}")
        assert torch.equal(o1[g], o2[g])


def test_grouped_misaligned_workspace_is_rejected_before_any_launch(cuda_device):
    """A workspace that is not 16-byte aligned is refused with SMGEMM_ERR_ALIGNMENT before
    anything is enqueued: neither the GEMM groups nor a K = 0 group (filled with act(bias)
    on valid calls) touch their outputs."""
    shapes = [(256, 256, 1024), (64, 128, 0)]
    As = [torch.ones((M, K), dtype=torch.bfloat16, device="cuda") for M, N, K in shapes]
    Bs = [torch.ones((K, N), dtype=torch.bfloat16, device="cuda") for M, N, K in shapes]
    outs = [torch.full((M, N), 7.0, dtype=torch.float32, device="cuda") for M, N, K in shapes]
    nbytes = int(sg.lib().smgemm_grouped_workspace_size(len(shapes)))
    ws = torch.zeros(nbytes + 64, dtype=torch.uint8, device="cuda")[4:]
    assert ws.data_ptr() % 16 == 4
    with pytest.raises(sg.SmgemmError) as ei:
        sg.gemm_bf16_grouped(As, Bs, outs=outs, workspace=ws)
    assert ei.value.status == sg.ERR_ALIGNMENT
    assert sg.check() == sg.OK
    for o in outs:
        assert bool((o == 7.0).all())
    sg.gemm_bf16_grouped(As, Bs, outs=outs, workspace=torch.zeros(nbytes, dtype=torch.uint8, device="cuda"))
    assert sg.check() == sg.OK
    assert bool((outs[0] == 1024.0).all()) and bool((outs[1] == 0.0).all())


def test_prepared_grouped_gemm_matches_one_shot_calls(cuda_device):
    """GroupedGemm checks and marshals once; each call only launches. Two calls, with the
    inputs' contents changed in between, equal gemm_bf16_grouped on the same tensors bit
    for bit (the kernel reads the tensors at launch time)."""
    shapes = [(128 * (g + 1), 512, 256) for g in range(8)]
    As = [to_dtype(synth.normal(42, g, (M, K)), torch.bfloat16).cuda() for g, (M, N, K) in enumerate(shapes)]
    Bs = [to_dtype(synth.normal(42, 100 + g, (K, N), 0.1), torch.bfloat16).cuda() for g, (M, N, K) in enumerate(shapes)]
    prepared = sg.GroupedGemm(As, Bs, act="silu", out_dtype=torch.bfloat16)
    for step in range(2):
        got = [o.clone() for o in prepared()]
        want = sg.gemm_bf16_grouped(As, Bs, act="silu", out_dtype=torch.bfloat16)
        assert sg.check() == sg.OK
        for g in range(len(shapes)):
            assert torch.equal(got[g], want[g]), f"step {step} group {g}"
        for A in As:
            A.mul_(-0.5)                       # new contents, same storage


def _grouped_sweep(n=40, seed=77):
    rs = np.random.RandomState(seed)
    cases = []
    for i in range(n):
        G = int(rs.randint(1, 13))
        shapes = [(int(rs.choice([0, int(rs.randint(1, 65)), int(rs.randint(65, 600))], p=[0.1, 0.3, 0.6])),
                   8 * int(rs.randint(1, 66)), 8 * int(rs.randint(0, 80))) for _ in range(G)]
        cases.append(dict(shapes=shapes, la=["row", "col"][rs.randint(2)], lb=["row", "col"][rs.randint(2)],
                          integer=bool(rs.randint(2)), act=["none", "gelu_tanh", "silu"][rs.randint(3)],
                          sched_split=["1", "0"][rs.randint(2)], seed=300 + i,
                          transpose="0" if i % 4 == 3 else "1"))
    return cases


@pytest.mark.parametrize("case", _grouped_sweep(), ids=lambda c: "G{}".format(len(c["shapes"])))
def test_grouped_seeded_random_sweep(cuda_device, monkeypatch, case):
    """Random group counts and shapes (empty groups, K = 0, one-row groups, ragged tails),
    layouts, activations, with and without the split tail: integer inputs without an
    activation are exact in FP32; real inputs with bias and activation meet the contract."""
    monkeypatch.setenv("SMGEMM_SCHED_GROUPED_SPLIT", case["sched_split"])
    monkeypatch.setenv("SMGEMM_GROUPED_TRANSPOSE", case["transpose"])
    exact = case["integer"]
    act = "none" if exact else case["act"]
    As, Bs, bs, Ah, Bh, bh = [], [], [], [], [], []
    for g, (M, N, K) in enumerate(case["shapes"]):
        s = case["seed"]
        if exact:
            a = synth.integers(s, 3 * g, (M, K), -3, 3)
            b = synth.integers(s, 3 * g + 1, (K, N), -3, 3)
        else:
            a = synth.normal(s, 3 * g, (M, K))
            b = synth.normal(s, 3 * g + 1, (K, N), 0.1)
        As.append(_operand(a, case["la"]))
        Bs.append(_operand(b, case["lb"]))
        Ah.append(to_dtype(a, torch.bfloat16))
        Bh.append(to_dtype(b, torch.bfloat16))
        bias = None if exact or g % 3 == 1 else to_dtype(synth.normal(s, 3 * g + 2, (N,), 0.5), torch.bfloat16)
        bs.append(None if bias is None else bias.cuda())
        bh.append(bias)
    out_dt = torch.float32 if exact else torch.bfloat16
    outs = sg.gemm_bf16_grouped(As, Bs, biases=bs, act=act, out_dtype=out_dt)
    assert sg.check() == sg.OK
    orc_act = {"none": oracle.ACT_NONE, "gelu_tanh": oracle.ACT_GELU_TANH, "silu": oracle.ACT_SILU}[act]
    for g, (M, N, K) in enumerate(case["shapes"]):
        if M == 0 or N == 0:
            assert outs[g].numel() == 0
            continue
        a, ad = orc_view(Ah[g])
        b, bd = orc_view(Bh[g])
        kw = {} if bh[g] is None else dict(zip(("bias", "bias_dtype"), orc_view(bh[g])))
        ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, act=orc_act,
                               out_dtype=oracle.F32 if exact else oracle.BF16, want_absacc=True, **kw)
        got = outs[g].float().cpu().numpy()
        if exact:
            assert np.array_equal(got, ref.astype(np.float32)), f"group {g} {M}x{N}x{K}"
        else:
            check_tolerance(got, ref, acc, out_dt, what=f"group {g} {M}x{N}x{K}")


@pytest.mark.parametrize("la,lb", [("row", "row"), ("row", "col"), ("col", "row"), ("col", "col")])
def test_grouped_transposed_remainder_tiles(cuda_device, monkeypatch, la, lb):
    """Groups whose last row of tiles holds 1..128 rows run that row transposed (C^T =
    B^T A^T, the rows of A as the MMA's N): on integer inputs the result equals the padded
    tiles' and the oracle's bit for bit, also where those tiles are split along K; with
    bias and activation into FP32 and FP16 outputs it meets the contract."""
    shapes = [(1, 264, 136), (128, 256, 64), (129, 520, 200), (300, 40, 72), (384, 256, 4096), (640, 136, 64)]
    As, Bs, Ah, Bh, refs = [], [], [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = synth.integers(45, 2 * g, (M, K), -3, 3)
        b = synth.integers(45, 2 * g + 1, (K, N), -3, 3)
        As.append(_operand(a, la)); Bs.append(_operand(b, lb))
        Ah.append(to_dtype(a, torch.bfloat16)); Bh.append(to_dtype(b, torch.bfloat16))
        av, ad = orc_view(Ah[g]); bv, bd = orc_view(Bh[g])
        refs.append(oracle.gemm(av, bv, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32))
    got = {}
    for t in ("1", "0"):
        monkeypatch.setenv("SMGEMM_GROUPED_TRANSPOSE", t)
        got[t] = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
        cfg = sg.last_config()
        assert sg.check() == sg.OK
        assert ("transposed_tiles=0" in cfg) == (t == "0"), cfg
    for g in range(len(shapes)):
        assert np.array_equal(got["1"][g].cpu().numpy(), refs[g].astype(np.float32)), f"group {g}"
        assert torch.equal(got["1"][g], got["0"][g])
    monkeypatch.setenv("SMGEMM_GROUPED_TRANSPOSE", "1")
    for out_dt, act, bias_dt in ((torch.float32, "silu", torch.float32), (torch.float16, "gelu_tanh", torch.float16)):
        reals_a, reals_b, biases, hb = [], [], [], []
        for g, (M, N, K) in enumerate(shapes):
            a = to_dtype(synth.normal(46, 3 * g, (M, K)), torch.bfloat16)
            b = to_dtype(synth.normal(46, 3 * g + 1, (K, N), 0.05), torch.bfloat16)
            bias = to_dtype(synth.normal(46, 3 * g + 2, (N,), 0.5), bias_dt)
            reals_a.append(a); reals_b.append(b); hb.append(bias)
            biases.append(bias.cuda())
        outs = sg.gemm_bf16_grouped([_operand(a.float().numpy(), la) for a in reals_a],
                                    [_operand(b.float().numpy(), lb) for b in reals_b],
                                    biases=biases, act=act, out_dtype=out_dt)
        assert sg.check() == sg.OK
        orc_act = oracle.ACT_SILU if act == "silu" else oracle.ACT_GELU_TANH
        orc_out = oracle.F32 if out_dt == torch.float32 else oracle.F16
        for g, (M, N, K) in enumerate(shapes):
            av, ad = orc_view(reals_a[g]); bv, bd = orc_view(reals_b[g])
            kw = dict(zip(("bias", "bias_dtype"), orc_view(hb[g])))
            ref, acc = oracle.gemm(av, bv, a_dtype=ad, b_dtype=bd, act=orc_act, out_dtype=orc_out, want_absacc=True,
                                   **kw)
            check_tolerance(outs[g].float().cpu().numpy(), ref, acc, out_dt, what=f"{out_dt} group {g} {M}x{N}x{K}")


@pytest.mark.parametrize("order", ["0", "1", "2"])
def test_grouped_table_orders_give_identical_results(cuda_device, monkeypatch, order):
    """The groups' order inside the launch (given, largest work first, or alternating
    largest and smallest) changes only which cluster computes which tile: integer inputs
    give the oracle's values bit for bit under every order, including a K = 0 group, an
    empty group and a split last wave."""
    monkeypatch.setenv("SMGEMM_GROUPED_ORDER", order)
    shapes = [(128, 512, 256), (700, 264, 4096), (0, 64, 64), (33, 1000, 200), (300, 136, 0), (512, 256, 1024),
              (1, 8, 16)]
    As, Bs, refs = [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = torch.from_numpy(synth.integers(47, 2 * g, (M, K), -3, 3)).to(torch.bfloat16)
        b = torch.from_numpy(synth.integers(47, 2 * g + 1, (K, N), -3, 3)).to(torch.bfloat16)
        As.append(a.cuda()); Bs.append(b.cuda())
        av, ad = orc_view(a); bv, bd = orc_view(b)
        refs.append(oracle.gemm(av, bv, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32))
    outs = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    for g, (M, N, K) in enumerate(shapes):
        if M == 0:
            assert outs[g].numel() == 0
            continue
        assert np.array_equal(outs[g].cpu().numpy(), refs[g].astype(np.float32)), f"group {g} {M}x{N}x{K}"


@pytest.mark.parametrize("la,lb", [("row", "row"), ("col", "col")])
def test_grouped_fp16_inputs(cuda_device, la, lb):
    """FP16 operands (the instruction descriptors' other input format) through normal and
    transposed tiles: integer inputs exact in FP32; real inputs with an FP16 bias and SiLU
    into FP16 outputs within the contract."""
    shapes = [(100, 264, 136), (384, 512, 200), (1, 40, 64), (520, 128, 72)]

    def op16(x, layout):
        t = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).to(torch.float16)
        if layout == "row":
            return t.cuda()
        rows, cols = t.shape
        ld = max(8, -(-rows // 8) * 8)
        buf = torch.zeros((cols, ld), dtype=torch.float16)
        buf[:, :rows] = t.t()
        return buf.cuda()[:, :rows].t()

    As, Bs, refs = [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = synth.integers(48, 2 * g, (M, K), -3, 3)
        b = synth.integers(48, 2 * g + 1, (K, N), -3, 3)
        As.append(op16(a, la)); Bs.append(op16(b, lb))
        refs.append(oracle.gemm(a.astype(np.float16), b.astype(np.float16), a_dtype=oracle.F16, b_dtype=oracle.F16,
                                out_dtype=oracle.F32))
    outs = sg.gemm_bf16_grouped(As, Bs, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    for g in range(len(shapes)):
        assert np.array_equal(outs[g].cpu().numpy(), refs[g].astype(np.float32)), f"group {g}"
    As, Bs, bs, hs = [], [], [], []
    for g, (M, N, K) in enumerate(shapes):
        a = synth.normal(49, 3 * g, (M, K)).astype(np.float16)
        b = (synth.normal(49, 3 * g + 1, (K, N)) * 0.1).astype(np.float16)
        bias = synth.normal(49, 3 * g + 2, (N,)).astype(np.float16)
        As.append(op16(a, la)); Bs.append(op16(b, lb)); bs.append(torch.from_numpy(bias).cuda())
        hs.append((a, b, bias))
    outs = sg.gemm_bf16_grouped(As, Bs, biases=bs, act="silu", out_dtype=torch.float16)
    assert sg.check() == sg.OK
    for g, (M, N, K) in enumerate(shapes):
        a, b, bias = hs[g]
        ref, acc = oracle.gemm(a, b, a_dtype=oracle.F16, b_dtype=oracle.F16, bias=bias, bias_dtype=oracle.F16,
                               act=oracle.ACT_SILU, out_dtype=oracle.F16, want_absacc=True)
        check_tolerance(outs[g].float().cpu().numpy(), ref, acc, torch.float16, what=f"group {g} {M}x{N}x{K}")
