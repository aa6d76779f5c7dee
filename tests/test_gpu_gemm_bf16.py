"""GPU parity of gemm_bf16 against the CPU oracle, through the C-ABI.

Sizes span several tiles and ragged tails in M, N and K; every layout pair, epilogue,
bias type and output type is covered; integer-valued inputs must match bit for bit
(every partial sum is exact in FP32); random inputs must meet the contract
|C - C_ref| <= 1e-3 * sum_k |a||b| + ulp(C_ref). Also: the p2 section 4.4 checklist of
the DeepGEMM kernel-library walkthrough (32x32, 64x64, non-aligned 67x50, all-ones,
sentinel-filled outputs), degenerate shapes, the skinny path and stream-K schedules,
and run-to-run determinism.
"""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import TORCH_TO_ORC, check_tolerance, orc_view, to_dtype

pytestmark = pytest.mark.gpu

SENT16 = 0x7BAD          # sentinel bit pattern for 16-bit outputs
SENT32 = 0x7FBADBAD      # sentinel bit pattern for fp32 outputs (a NaN)
ORC_ACT = {"none": oracle.ACT_NONE, "gelu_tanh": oracle.ACT_GELU_TANH, "silu": oracle.ACT_SILU}


def place(t: torch.Tensor, layout: str, pad: int = 8) -> torch.Tensor:
    """Copy a CPU [R, C] tensor to the GPU as a row- or column-major view whose leading
    dimension is padded to a multiple of `pad` elements (16 bytes for 16-bit types)."""
    R, Cn = t.shape
    if layout == "row":
        ld = -(-Cn // pad) * pad
        buf = torch.zeros((R, ld), dtype=t.dtype, device="cuda")
        buf[:, :Cn] = t.cuda()
        return buf[:, :Cn]
    ld = -(-R // pad) * pad
    buf = torch.zeros((Cn, ld), dtype=t.dtype, device="cuda")
    buf[:, :R] = t.t().cuda()
    return buf[:, :R].t()


def sentinel_out(M, N, dt, extra_rows=3):
    """Output view [M, N] inside a larger buffer filled with a sentinel pattern."""
    ld = -(-(N + 5) // 8) * 8
    full = torch.empty((M + extra_rows, ld), dtype=dt, device="cuda")
    if dt == torch.float32:
        full.view(torch.int32).fill_(SENT32)
    else:
        full.view(torch.int16).fill_(SENT16)
    return full, full[:M, :N]


def assert_sentinel_intact(full, M, N):
    bits = full.view(torch.int32 if full.dtype == torch.float32 else torch.int16).cpu().numpy()
    s = SENT32 if full.dtype == torch.float32 else np.int16(np.uint16(SENT16).view(np.int16))
    assert (bits[M:, :] == s).all(), "rows below M were written"
    assert (bits[:, N:] == s).all(), "columns right of N were written"


def run_case(M, N, K, *, ab=torch.bfloat16, la="row", lb="col", bias_dt=None, act="none",
             out_dt=torch.bfloat16, seed=0, integer=False):
    if integer:
        A = to_dtype(synth.integers(seed, 0, (M, K), -4, 4), ab)
        B = to_dtype(synth.integers(seed, 1, (K, N), -4, 4), ab)
    else:
        A = to_dtype(synth.normal(seed, 0, (M, K)), ab)
        B = to_dtype(synth.normal(seed, 1, (K, N)), ab)
    bias = None if bias_dt is None else to_dtype(synth.normal(seed, 2, (N,), 0.5), bias_dt)
    full, out = sentinel_out(M, N, out_dt)
    sg.gemm_bf16(place(A, la), place(B, lb), bias=None if bias is None else bias.cuda(), act=act, out=out)
    assert sg.check() == sg.OK
    got = out.float().cpu().numpy().astype(np.float64) if out_dt != torch.float32 else \
        out.cpu().numpy().astype(np.float64)
    assert_sentinel_intact(full, M, N)
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    kw = {}
    if bias is not None:
        bb, bbd = orc_view(bias)
        kw = dict(bias=bb, bias_dtype=bbd)
    ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, act=ORC_ACT[act],
                           out_dtype={torch.float32: oracle.F32, torch.bfloat16: oracle.BF16,
                                      torch.float16: oracle.F16}[out_dt], want_absacc=True, **kw)
    return got, ref, acc


# ------------------------------------------------------------------ configuration 1

def test_tiny_fp16_64cube_fp32_out(cuda_device):
    """64x64x64 fp16, U[-1,1] from seed 0, row-major A and B, FP32 out, no bias."""
    t = synth.tiny_fp16()
    A = to_dtype(t["A"], torch.float16)
    B = to_dtype(t["B"], torch.float16)
    out = sg.gemm_bf16(A.cuda(), B.cuda(), out_dtype=torch.float32)
    assert sg.check() == sg.OK
    a, ad = orc_view(A)
    b, bd = orc_view(B)
    ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bd, out_dtype=oracle.F32, want_absacc=True)
    check_tolerance(out.cpu().numpy(), ref, acc, torch.float32, what="tiny fp16")


# ------------------------------------------------------------------ exactness / layouts

@pytest.mark.parametrize("la", ["row", "col"])
@pytest.mark.parametrize("lb", ["row", "col"])
@pytest.mark.parametrize("sched", ["auto", "dp", "sk"])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_integer_inputs_bit_exact_all_layouts(cuda_device, monkeypatch, la, lb, sched, pair):
    """pair=1: 256x256 tiles on CTA pairs (cta_group::2); pair=0: 128x256 one-SM tiles."""
    monkeypatch.setenv("SMGEMM_SCHED", sched)
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    got, ref, _ = run_case(300, 600, 520, la=la, lb=lb, out_dt=torch.float32, integer=True, seed=3)
    assert ("path=pair" in sg.last_config()) == (pair == "1")
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float16])
def test_integer_inputs_bit_exact_16bit_out(cuda_device, out_dt):
    got, ref, _ = run_case(257, 513, 777, out_dt=out_dt, integer=True, seed=4)
    assert np.array_equal(got, ref)


def test_all_ones_gives_K(cuda_device):
    """The walkthrough's all-ones check: every output equals K."""
    for K in (64, 67, 1000):
        A = torch.ones((130, K), dtype=torch.bfloat16)
        B = torch.ones((K, 270), dtype=torch.bfloat16)
        full, out = sentinel_out(130, 270, torch.float32)
        sg.gemm_bf16(place(A, "row"), place(B, "row"), out=out)
        assert sg.check() == sg.OK
        assert (out.cpu() == K).all()
        assert_sentinel_intact(full, 130, 270)


def test_identity_and_permutation(cuda_device):
    A = to_dtype(synth.normal(5, 0, (200, 192)), torch.bfloat16)
    I = torch.eye(192, dtype=torch.bfloat16)
    out = sg.gemm_bf16(A.cuda(), I.cuda(), out_dtype=torch.float32)
    assert torch.equal(out.cpu(), A.float())
    perm = torch.from_numpy(np.random.RandomState(1).permutation(192))
    P = torch.zeros((192, 192), dtype=torch.bfloat16)
    P[perm, torch.arange(192)] = 1
    out = sg.gemm_bf16(A.cuda(), place(P, "col"), out_dtype=torch.bfloat16)
    assert torch.equal(out.cpu(), A[:, perm])


# ------------------------------------------------------------------ tolerance, epilogues

@pytest.mark.parametrize("M,N,K", [(32, 32, 32), (64, 64, 64), (67, 50, 33), (300, 700, 1000),
                                   (129, 257, 4096)])
@pytest.mark.parametrize("la,lb", [("row", "col"), ("row", "row"), ("col", "col")])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_random_within_tolerance(cuda_device, monkeypatch, M, N, K, la, lb, pair):
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    got, ref, acc = run_case(M, N, K, la=la, lb=lb, seed=M + N + K)
    check_tolerance(got, ref, acc, torch.bfloat16, what=f"{M}x{N}x{K} {la}/{lb}")


@pytest.mark.parametrize("act", ["none", "gelu_tanh", "silu"])
@pytest.mark.parametrize("bias_dt", [None, torch.bfloat16, torch.float32, torch.float16])
@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float16, torch.float32])
def test_epilogue_matrix(cuda_device, act, bias_dt, out_dt):
    got, ref, acc = run_case(200, 300, 256, bias_dt=bias_dt, act=act, out_dt=out_dt, seed=9)
    check_tolerance(got, ref, acc, out_dt, what=f"{act}/{bias_dt}/{out_dt}")


def test_fp16_inputs(cuda_device):
    got, ref, acc = run_case(333, 444, 555, ab=torch.float16, lb="row", bias_dt=torch.float16,
                             act="silu", out_dt=torch.float16, seed=11)
    check_tolerance(got, ref, acc, torch.float16, what="fp16 inputs")


# ------------------------------------------------------------------ skinny path

@pytest.mark.parametrize("M", [1, 4, 16, 17, 33, 64])
@pytest.mark.parametrize("lb", ["row", "col"])
def test_skinny_path(cuda_device, M, lb):
    got, ref, acc = run_case(M, 1000, 700, lb=lb, out_dt=torch.float32, seed=20 + M)
    assert "skinny" in sg.last_config()
    check_tolerance(got, ref, acc, torch.float32, what=f"skinny M={M} {lb}")


@pytest.mark.parametrize("M", [1, 16, 64])
def test_skinny_integer_exact_with_bias_act(cuda_device, M):
    got, ref, _ = run_case(M, 777, 1300, lb="row", out_dt=torch.float32, integer=True, seed=30 + M)
    assert np.array_equal(got, ref)
    got, ref, acc = run_case(M, 777, 300, lb="row", bias_dt=torch.bfloat16, act="gelu_tanh",
                             out_dt=torch.bfloat16, seed=31)
    check_tolerance(got, ref, acc, torch.bfloat16, what="skinny epilogue")


# ------------------------------------------------------------------ activation accuracy

def _act_points(n=8192):
    """n FP32 activation inputs: a dense sweep of [-20, 20] (it crosses the region near
    x = -10 where the GeLU value enters the subnormal range) plus zeros, tiny and large
    magnitudes (where exp overflows and tanh saturates)."""
    special = np.float32([0.0, -0.0, 1e-30, -1e-30, 1e-6, -1e-6, 0.5, -0.5, 1.0, -1.0, 40.0, -40.0,
                          60.0, -60.0, -87.0, -89.0, 100.0, -100.0, -10.3, -10.45, -10.6, -103.0, -104.0])
    sweep = np.linspace(-20.0, 20.0, n - special.size, dtype=np.float32)
    return np.concatenate([special, sweep]).astype(np.float32)


def _act_run(path, act, out_dt, x, offset):
    """Runs one GEMM whose products are all zero (A = 0, or K = 0), so every output is
    act(bias[n]) with bias = x; returns the first output row as float64."""
    N = x.size
    buf = torch.zeros(N + 4, dtype=torch.float32, device="cuda")  # 256-byte aligned start
    buf[offset:offset + N] = torch.from_numpy(x).cuda()
    bias = buf[offset:offset + N]
    M = 16 if path == "skinny" else 128
    if path in ("skinny", "tile"):
        A = torch.zeros((M, 64), dtype=torch.bfloat16, device="cuda")
        B = torch.zeros((N, 64), dtype=torch.bfloat16, device="cuda").t()
        out = sg.gemm_bf16(A, B, bias=bias, act=act, out_dtype=out_dt)
    elif path == "grouped":
        A = torch.zeros((M, 64), dtype=torch.bfloat16, device="cuda")
        B = torch.zeros((64, N), dtype=torch.bfloat16, device="cuda")
        out = sg.gemm_bf16_grouped([A], [B], biases=[bias], act=act, out_dtype=out_dt)[0]
    elif path == "fp8":
        K = 256
        qa = torch.zeros((M, K), dtype=torch.uint8, device="cuda")
        qb = torch.zeros((N, K), dtype=torch.uint8, device="cuda")
        sa = torch.ones((K // 128, M), dtype=torch.float32, device="cuda")
        sb = torch.ones((K // 128, -(-N // 128)), dtype=torch.float32, device="cuda")
        out = sg.gemm_fp8_blockscaled(qa, sa, qb, sb, bias=bias, act=act, out_dtype=out_dt)
    else:  # K = 0: the fill kernel writes act(bias)
        ldc = -(-N // 8) * 8
        out = torch.empty((M, ldc), dtype=out_dt, device="cuda")[:, :N]
        codes = {torch.float32: sg.F32, torch.bfloat16: sg.BF16, torch.float16: sg.F16}
        st = sg.lib().gemm_bf16(M, N, 0, None, sg.BF16, sg.ROW_MAJOR, 8, None, sg.ROW_MAJOR, ldc,
                                bias.data_ptr(), sg.F32, {"gelu_tanh": 1, "silu": 2}[act], out.data_ptr(),
                                codes[out_dt], ldc, None, 0, None)
        assert st == sg.OK
    assert sg.check() == sg.OK
    got = out.float().cpu()
    assert bool((got == got[0]).all() | (got.isnan() & got[0].isnan()).all()), "rows differ"
    return got[0].numpy().astype(np.float64)


@pytest.mark.parametrize("act", ["gelu_tanh", "silu"])
@pytest.mark.parametrize("out_dt", [torch.float32, torch.bfloat16, torch.float16])
@pytest.mark.parametrize("path,offset", [("skinny", 0), ("skinny", 1), ("tile", 0), ("tile", 1), ("grouped", 0),
                                         ("fp8", 0), ("fill", 0)])
def test_epilogue_activation_accuracy(cuda_device, act, out_dt, path, offset):
    """The contract |C - C_ref| <= 1e-3 sum_k |a||b| + ulp_out(C_ref) where it is
    tightest: A = 0 (or K = 0), so sum_k |a||b| = 0 and every output act(bias[n]) must be
    within one ulp of the output type of the oracle's value, for 8192 FP32 inputs and
    every activation, output type and epilogue (swap-AB skinny, CTA-pair tile, grouped,
    FP8 block-scaled, the K = 0 fill). offset = 1 misaligns the bias so the scalar bias
    loads run instead of the 16-byte ones."""
    x = _act_points()
    got = _act_run(path, act, out_dt, x, offset)
    ref = oracle.round_to(np.array([oracle.act(float(v), ORC_ACT[act]) for v in x]), TORCH_TO_ORC[out_dt])
    check_tolerance(got, ref, np.zeros_like(ref), out_dt, what=f"{act} {path} -> {out_dt}")


# ------------------------------------------------------------------ degenerate shapes

def test_k_zero_writes_activation_of_bias(cuda_device):
    bias = to_dtype(np.linspace(-3, 3, 70, dtype=np.float32), torch.float32)
    A = torch.zeros((5, 8), dtype=torch.bfloat16, device="cuda")[:, :0]
    B = torch.zeros((8, 70), dtype=torch.bfloat16, device="cuda")[:0, :]
    out = torch.empty((5, 72), dtype=torch.float32, device="cuda")[:, :70]
    sg.lib()  # fail loudly if missing
    st = sg.lib().gemm_bf16(5, 70, 0, A.data_ptr(), sg.BF16, sg.ROW_MAJOR, 8, B.data_ptr(), sg.ROW_MAJOR, 72,
                            bias.cuda().data_ptr(), sg.F32, 2, out.data_ptr(), sg.F32, 72, None, 0, None)
    assert st == sg.OK and sg.check() == sg.OK
    want = np.array([oracle.act(float(b), oracle.ACT_SILU) for b in bias.numpy()])
    np.testing.assert_allclose(out.cpu().numpy(), np.tile(want, (5, 1)), rtol=1e-6, atol=1e-7)


def test_empty_m_or_n_is_noop(cuda_device):
    A = torch.zeros((0, 64), dtype=torch.bfloat16, device="cuda")
    B = torch.zeros((64, 64), dtype=torch.bfloat16, device="cuda")
    out = sg.gemm_bf16(A, B)
    assert out.shape == (0, 64) and sg.check() == sg.OK


@pytest.mark.parametrize("M,N,K", [(1, 1, 1), (1, 8, 1), (200, 1, 3), (5, 3, 200)])
def test_tiny_ragged(cuda_device, M, N, K):
    got, ref, acc = run_case(M, N, K, la="row", lb="col", out_dt=torch.float32, seed=40 + M + N + K)
    check_tolerance(got, ref, acc, torch.float32, what=f"{M}x{N}x{K}")


def test_misaligned_leading_dimension_is_rejected(cuda_device):
    A = torch.zeros((64, 50), dtype=torch.bfloat16, device="cuda")   # lda*2 = 100 bytes
    B = torch.zeros((50, 64), dtype=torch.bfloat16, device="cuda")
    with pytest.raises(sg.SmgemmError) as e:
        sg.gemm_bf16(A, B)
    assert e.value.status == sg.ERR_ALIGNMENT


# ------------------------------------------------------------------ stream-K, determinism

def test_stream_k_split_across_many_ctas(cuda_device, monkeypatch):
    """Few tiles, long K: stream-K splits every tile over several CTAs."""
    monkeypatch.setenv("SMGEMM_SCHED", "sk")
    got, ref, acc = run_case(256, 512, 8192, seed=50, out_dt=torch.float32)
    assert "sk_iters=" in sg.last_config() and "sk_iters=0" not in sg.last_config()
    check_tolerance(got, ref, acc, torch.float32, what="stream-K")


@pytest.mark.parametrize("pair", ["1", "0"])
def test_persistent_multi_tile_per_cta(cuda_device, monkeypatch, pair):
    monkeypatch.setenv("SMGEMM_GRID", "3")
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    got, ref, _ = run_case(700, 1100, 300, integer=True, out_dt=torch.float32, seed=51)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("pair", ["1", "0"])
def test_stream_k_hybrid_many_tiles(cuda_device, monkeypatch, pair):
    """More tiles than CTAs, not a multiple: data-parallel waves + a stream-K tail."""
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    monkeypatch.setenv("SMGEMM_GRID", "5")
    got, ref, _ = run_case(1500, 1300, 1024, integer=True, out_dt=torch.float32, seed=52)
    cfg = sg.last_config()
    assert "sk_iters=0" not in cfg and "dp_tiles=0" not in cfg, cfg
    assert np.array_equal(got, ref)


def test_deterministic_run_to_run(cuda_device):
    A = to_dtype(synth.normal(60, 0, (1024, 4096)), torch.bfloat16).cuda()
    B = to_dtype(synth.normal(60, 1, (4096, 1024)), torch.bfloat16).cuda()
    c1 = sg.gemm_bf16(A, B, out_dtype=torch.float32).clone()
    c2 = sg.gemm_bf16(A, B, out_dtype=torch.float32)
    assert sg.check() == sg.OK
    assert torch.equal(c1, c2)


# ------------------------------------------------------------------ TMA-store epilogue

@pytest.mark.parametrize("out_dt", [torch.bfloat16, torch.float16, torch.float32])
@pytest.mark.parametrize("M,N,K,act", [(300, 520, 136, "gelu_tanh"), (1024, 1024, 512, "none"), (257, 200, 64, "silu"),
                                       (4096, 4096, 256, "none"), (200, 304, 96, "none"), (200, 300, 64, "silu")])
def test_tma_store_epilogue_matches_direct_stores(cuda_device, monkeypatch, out_dt, M, N, K, act):
    """The pair kernel writes C through shared memory and TMA tile stores (boxes clipped
    at the matrix edge); SMGEMM_EPI_STORE=direct selects 16-byte stores from registers.
    The values are computed the same way in both, so the outputs must agree bit for bit,
    and with the oracle within the contract. Rows and columns past M and N
    (sentinel-filled padding) stay untouched. A row of C that is not a whole number of
    16-byte units (N = 300 in 16-bit) keeps the register stores."""
    A = to_dtype(synth.normal(97, M, (M, K)), torch.bfloat16)
    B = to_dtype(synth.normal(97, N, (K, N), 0.2), torch.bfloat16)
    bias = to_dtype(synth.normal(97, 1, (N,), 0.5), torch.bfloat16)
    Ad, Bd, bd = A.cuda(), B.t().contiguous().cuda().t(), bias.cuda()
    outs = {}
    for mode in ("direct", "tma"):
        if mode == "direct":
            monkeypatch.setenv("SMGEMM_EPI_STORE", "direct")
        else:
            monkeypatch.delenv("SMGEMM_EPI_STORE", raising=False)
        full, view = sentinel_out(M, N, out_dt)
        sg.gemm_bf16(Ad, Bd, bias=bd, act=act, out=view)
        assert sg.check() == sg.OK
        assert ("tmastore" in sg.last_config()) == (mode == "tma" and (N * view.element_size()) % 16 == 0)
        assert_sentinel_intact(full, M, N)
        outs[mode] = view.clone()
    assert torch.equal(outs["direct"], outs["tma"])
    if M * N <= 600_000:
        a, ad = orc_view(A)
        b, bdt = orc_view(B)
        bb, bbd = orc_view(bias)
        ref, acc = oracle.gemm(a, b, a_dtype=ad, b_dtype=bdt, bias=bb, bias_dtype=bbd, act=ORC_ACT[act],
                               out_dtype=TORCH_TO_ORC[out_dt], want_absacc=True)
        check_tolerance(outs["tma"].float().cpu().numpy(), ref, acc, out_dt, what=f"tma store {M}x{N}x{K}")


# ------------------------------------------------------------------ split-tile counters need no zeroing

@pytest.mark.parametrize("fill", ["zeros", "garbage", "ones"])
def test_split_counters_need_no_zeroed_workspace(cuda_device, fill):
    """The split tail's arrival counters carry a per-call generation, so the workspace is
    used as found: zeros, random bytes or all-ones bytes, and the words the previous call
    left, all give the same bits as a fresh call (4096^3 splits its ragged last wave)."""
    M = N = K = 4096
    A = torch.from_numpy(synth.integers(98, 0, (M, K), -3, 3)).to(torch.bfloat16).cuda()
    B = torch.from_numpy(synth.integers(98, 1, (K, N), -3, 3)).to(torch.bfloat16).cuda()
    plan = sg.schedule_dump(M, N, K, 0, sg.ROW_MAJOR, torch.cuda.get_device_properties(0).multi_processor_count)
    assert (plan[:, 6] >= 0).any()
    nbytes = sg.workspace_size(M, N, K, 0)
    ref = sg.gemm_bf16(A, B, out_dtype=torch.float32)
    if fill == "zeros":
        ws = torch.zeros(nbytes, dtype=torch.uint8, device="cuda")
    elif fill == "ones":
        ws = torch.full((nbytes,), 0xFF, dtype=torch.uint8, device="cuda")
    else:
        ws = torch.randint(0, 256, (nbytes,), dtype=torch.uint8, device="cuda")
    for _ in range(3):
        out = sg.gemm_bf16(A, B, out_dtype=torch.float32, workspace=ws)
        assert sg.check() == sg.OK
        assert torch.equal(out, ref)
    # integer inputs: every partial sum is exact, so the split result is the exact product
    exact = (A.double() @ B.double()).float()
    assert torch.equal(ref, exact)


# ------------------------------------------------------------------ seeded random sweep

def _sweep_cases(n=400, seed=2024):
    rs = np.random.RandomState(seed)
    cases = []
    for i in range(n):
        M = int(rs.choice([int(rs.randint(1, 65)), int(rs.randint(65, 700))]))
        N = int(rs.randint(1, 700))
        K = int(rs.randint(1, 900))
        cases.append(dict(
            M=M, N=N, K=K, ab=[torch.bfloat16, torch.float16][rs.randint(2)],
            la=["row", "col"][rs.randint(2)], lb=["row", "col"][rs.randint(2)],
            out_dt=[torch.float32, torch.bfloat16, torch.float16][rs.randint(3)],
            bias_dt=[None, torch.float32, torch.bfloat16, torch.float16][rs.randint(4)],
            act=["none", "gelu_tanh", "silu"][rs.randint(3)],
            integer=bool(rs.randint(2)), sched=["auto", "dp", "sk"][rs.randint(3)],
            pair=["1", "0"][rs.randint(2)], seed=100 + i))
    return cases


@pytest.mark.parametrize("case", _sweep_cases(), ids=lambda c: "M{M}N{N}K{K}".format(**c))
def test_seeded_random_sweep(cuda_device, monkeypatch, case):
    """Random shapes (tiny to several tiles, ragged in M, N and K), operand types,
    layouts, bias types, activations, output types and schedules: integer inputs without
    an activation match the oracle bit for bit; everything else meets the contract."""
    c = dict(case)
    monkeypatch.setenv("SMGEMM_SCHED", c.pop("sched"))
    monkeypatch.setenv("SMGEMM_PAIR", c.pop("pair"))
    M, N, K = c.pop("M"), c.pop("N"), c.pop("K")
    got, ref, acc = run_case(M, N, K, **c)
    if c["integer"] and c["act"] == "none" and c["bias_dt"] is None:
        assert np.array_equal(got, ref), sg.last_config()
    else:
        check_tolerance(got, ref, acc, c["out_dt"], what=sg.last_config())
