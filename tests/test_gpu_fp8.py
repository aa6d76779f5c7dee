"""GPU parity of quantize_fp8_blockwise (bit-exact) and gemm_fp8_blockscaled
(tolerance; exact on integer codes) against the CPU oracle, through the C-ABI.

Group scaling follows the DeepGEMM kernel-library walkthrough (zwxr.cn), section 2.4.
The quantiser must reproduce the oracle's scales and codes bit for bit, including
ragged groups, all-zero groups, signed zeros and saturation; the GEMM must meet the
contract computed from the same quantised operands.
"""
import numpy as np
import pytest
import torch

import oracle
import sm_gemm_b200 as sg
import synth
from _parity import TORCH_TO_ORC, check_tolerance, orc_view

pytestmark = pytest.mark.gpu


def _gpu_quant(X: np.ndarray, group_rows: int, layout: str = "row"):
    t = torch.from_numpy(np.ascontiguousarray(X))
    if layout == "row":
        R, Cn = X.shape
        ld = -(-Cn // 4) * 4
        buf = torch.zeros((R, ld), dtype=torch.float32, device="cuda")
        buf[:, :Cn] = t.cuda()
        Xd = buf[:, :Cn]
    else:
        R, Cn = X.shape
        ld = -(-R // 4) * 4
        buf = torch.zeros((Cn, ld), dtype=torch.float32, device="cuda")
        buf[:, :R] = t.t().cuda()
        Xd = buf[:, :R].t()
    Q, S = sg.quantize_fp8_blockwise(Xd, group_rows)
    assert sg.check() == sg.OK
    return Q.cpu().numpy(), S.cpu().numpy()


@pytest.mark.parametrize("shape", [(37, 300), (128, 128), (1, 1), (5, 1000), (2048, 4096)])
@pytest.mark.parametrize("layout", ["row", "col"])
def test_quant_1x128_bit_exact(cuda_device, shape, layout):
    X = synth.normal_with_outliers(70, 0, shape)
    Q, S = _gpu_quant(X, 1, layout)
    Qr, Sr = oracle.quant_1x128(X)
    assert np.array_equal(S.view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q, Qr)


@pytest.mark.parametrize("shape", [(300, 200), (128, 128), (1, 1), (4096, 1024), (257, 130)])
@pytest.mark.parametrize("layout", ["row", "col"])
def test_quant_128x128_bit_exact(cuda_device, shape, layout):
    X = synth.normal_with_outliers(71, 0, shape)
    Q, S = _gpu_quant(X, 128, layout)
    Qr, Sr = oracle.quant_128x128(X)
    assert np.array_equal(S.view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q, Qr)


def test_quant_special_values(cuda_device):
    """Signed zeros, tiny values that round to zero, all-zero groups, a constant group,
    exact ties and values at the saturation edge."""
    X = np.zeros((4, 256), dtype=np.float32)
    X[0, :8] = [-0.0, 0.0, -1e-30, 1e-30, 448.0, -448.0, 1.0, -1.0]
    X[1, :128] = -3.0
    X[2, :128] = np.float32(1.0) + np.arange(128, dtype=np.float32) * np.float32(2.0 ** -7)
    X[3, 128:] = 2.0 ** (np.arange(128) % 20 - 10)
    for g in (1, 128):
        Q, S = _gpu_quant(X if g == 1 else np.ascontiguousarray(X.T), g)
        Qr, Sr = (oracle.quant_1x128(X) if g == 1 else oracle.quant_128x128(np.ascontiguousarray(X.T)))
        assert np.array_equal(S.view(np.uint32), Sr.view(np.uint32))
        assert np.array_equal(Q, Qr)


def _scale_hitting(target: np.float32):
    """An amax whose group scale RN(amax / 448) is exactly `target`, or None."""
    a = np.float32(target * np.float32(448.0))
    for _ in range(16):
        s = np.float32(a / np.float32(448.0))
        if s == target:
            return a
        a = np.nextafter(a, np.float32(np.inf) if s < target else np.float32(0.0), dtype=np.float32)
    return None


def _edge_scales():
    """Scales that stress the division by the group scale: significands of all ones
    (where a reciprocal-based quotient needs special care), powers of two, scales
    near 2^-90 and near the largest finite amax, and ordinary random ones."""
    f = np.float32
    out = []
    for e in (-120, -95, -91, -90, -89, -60, -20, -7, -1, 0, 1, 7, 40, 110, 119):
        out += [f(2.0 ** e), f(np.nextafter(f(2.0 ** (e + 1)), f(0))),   # 1.0 and all-ones significands
                f(1.5 * 2.0 ** e), f(np.nextafter(f(2.0 ** e), f(np.inf)))]
    rng = np.random.default_rng(5)
    out += list((rng.uniform(1, 2, 24) * 2.0 ** rng.integers(-40, 40, 24)).astype(np.float32))
    with np.errstate(over="ignore"):
        return [s for s in out if np.isfinite(s) and np.isfinite(f(s * f(448.0)))]


def _tie_group(amax: np.float32, s: np.float32, n: int, rng) -> np.ndarray:
    """n values whose quotients by s sit on and next to the E4M3 rounding midpoints
    (where one ulp of the FP32 quotient decides the code), plus +-amax."""
    vals = oracle.e4m3_decode(np.arange(0, 127, dtype=np.uint8)).astype(np.float64)
    mids = (vals[:-1] + vals[1:]) / 2.0
    m = rng.choice(mids, n)
    x = (m * np.float64(s)).astype(np.float32)
    step = rng.integers(-1, 2, n)
    x = np.where(step > 0, np.nextafter(x, np.float32(np.inf)), np.where(step < 0, np.nextafter(x, np.float32(0)), x))
    x = np.minimum(np.abs(x), amax).astype(np.float32) * rng.choice(np.float32([-1, 1]), n)
    x[0], x[1] = amax, -amax
    return x.astype(np.float32)


def test_quant_division_edge_scales(cuda_device):
    """Bit-exact codes for groups whose scales stress the quotient x / s: elements on
    and one FP32 ulp beside the E4M3 rounding midpoints, under each edge scale."""
    rng = np.random.default_rng(11)
    groups, blocks = [], []
    for s in _edge_scales():
        amax = _scale_hitting(s)
        if amax is None:
            continue
        groups.append(_tie_group(amax, s, 128, rng))
        blocks.append(_tie_group(amax, s, 128 * 128, rng).reshape(128, 128))
    assert len(groups) >= 60
    X1 = np.stack(groups)
    Q, S = _gpu_quant(X1, 1)
    Qr, Sr = oracle.quant_1x128(X1)
    assert np.array_equal(S.view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q, Qr)
    X2 = np.concatenate(blocks, axis=1)  # [K = 128, N = 128 * blocks]
    Q, S = _gpu_quant(X2, 128)
    Qr, Sr = oracle.quant_128x128(X2)
    assert np.array_equal(S.view(np.uint32), Sr.view(np.uint32))
    assert np.array_equal(Q, Qr)


def test_quant_encoder_every_fp32_value_up_to_448(cuda_device):
    """The device E4M3 encoder on every FP32 bit pattern of magnitude <= 448, both signs
    (2,277,507,074 values). Each 1x128 group holds 448 in its first slot, so its scale is
    448 / 448 = 1 exactly, x / s = x, and every code must be the oracle's encoding of x
    itself. Inputs are an enumeration of bit patterns built on the device; the codes come
    back in chunks of 127 * 2^20 values and are checked against the oracle's encoder."""
    assert oracle.quant_1x128(np.float32([[448.0, 1.0]]))[1][0, 0] == np.float32(1.0)
    top = int(np.array(448.0, dtype=np.float32).view(np.uint32))
    rows = 1 << 20
    per = rows * 127
    X = torch.empty((rows, 128), dtype=torch.float32, device="cuda")
    body = torch.empty(per, dtype=torch.float32, device="cuda")
    for sign in (0, 1):
        for lo in range(0, top + 1, per):
            n = min(per, top + 1 - lo)
            bits = torch.arange(lo, lo + n, dtype=torch.int64, device="cuda")
            if sign:
                bits -= 1 << 31  # the int32 of the pattern with the sign bit set
            body.zero_()
            body[:n] = bits.to(torch.int32).view(torch.float32)
            X[:, 0] = 448.0
            X[:, 1:] = body.view(rows, 127)
            Q, S = sg.quantize_fp8_blockwise(X, 1)
            assert sg.check() == sg.OK
            assert bool((S == 1.0).all()) and bool((Q[:, 0] == 0x7E).all())
            got = Q[:, 1:].reshape(-1)[:n].cpu().numpy()
            y = np.arange(lo, lo + n, dtype=np.uint32)
            if sign:
                y |= np.uint32(1 << 31)
            ref = oracle.e4m3_encode(y.view(np.float32))
            bad = np.flatnonzero(got != ref)
            assert bad.size == 0, f"{bad.size} codes differ, first for bits {y[bad[0]]:#010x}: " \
                f"{got[bad[0]]:#04x} vs {ref[bad[0]]:#04x}"


def _quantised_problem(M, N, K, seed):
    A = synth.normal_with_outliers(seed, 0, (M, K))
    B = synth.normal_with_outliers(seed, 1, (K, N))
    qa, sa = oracle.quant_1x128(A)
    qb, sb = oracle.quant_128x128(B)
    return qa, sa, qb, sb


def _run_fp8(qa, sa, qb, sb, out_dt=torch.bfloat16, bias=None, act="none"):
    M, N = qa.shape[0], qb.shape[0]
    out = torch.empty((M, -(-N // 8) * 8), dtype=out_dt, device="cuda")[:, :N]
    sg.gemm_fp8_blockscaled(torch.from_numpy(qa).cuda(), torch.from_numpy(sa).cuda(),
                            torch.from_numpy(qb).cuda(), torch.from_numpy(sb).cuda(),
                            bias=None if bias is None else bias.cuda(), act=act, out=out)
    assert sg.check() == sg.OK
    return out.float().cpu().numpy().astype(np.float64)


@pytest.mark.parametrize("M,N,K", [(128, 128, 128), (300, 260, 384), (64, 1000, 1024), (257, 129, 2048)])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_fp8_gemm_within_tolerance(cuda_device, monkeypatch, M, N, K, pair):
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    qa, sa, qb, sb = _quantised_problem(M, N, K, seed=M + N + K)
    got = _run_fp8(qa, sa, qb, sb)
    ref, acc = oracle.gemm_fp8(qa, sa, qb, sb, out_dtype=oracle.BF16, want_absacc=True)
    check_tolerance(got, ref, acc, torch.bfloat16, what=f"fp8 {M}x{N}x{K}")


@pytest.mark.parametrize("sched", ["dp", "sk", "auto"])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_fp8_gemm_integer_codes_unit_scales_exact(cuda_device, monkeypatch, sched, pair):
    """pair=1: 256x256 tiles on CTA pairs; pair=0: 128x128 one-SM tiles."""
    monkeypatch.setenv("SMGEMM_SCHED", sched)
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    rs = np.random.RandomState(5)
    M, N, K = 300, 400, 1024
    qa = oracle.e4m3_encode(rs.randint(-8, 9, (M, K)).astype(np.float32))
    qb = oracle.e4m3_encode(rs.randint(-8, 9, (N, K)).astype(np.float32))
    sa = np.ones((K // 128, M), np.float32)
    sb = np.ones((K // 128, -(-N // 128)), np.float32)
    got = _run_fp8(qa, sa, qb, sb, out_dt=torch.float32)
    ref = oracle.gemm_fp8(qa, sa, qb, sb, out_dtype=oracle.F32)
    assert np.array_equal(got, ref)


def test_fp8_gemm_power_of_two_scales_exact(cuda_device):
    rs = np.random.RandomState(6)
    M, N, K = 200, 300, 512
    qa = oracle.e4m3_encode(rs.randint(-8, 9, (M, K)).astype(np.float32))
    qb = oracle.e4m3_encode(rs.randint(-8, 9, (N, K)).astype(np.float32))
    # scale products in 2^[-4, 4] keep every FP32 partial sum exact (<= 24 significant bits)
    sa = (2.0 ** rs.randint(-2, 3, (K // 128, M))).astype(np.float32)
    sb = (2.0 ** rs.randint(-2, 3, (K // 128, 3))).astype(np.float32)
    got = _run_fp8(qa, sa, qb, sb, out_dt=torch.float32)
    ref = oracle.gemm_fp8(qa, sa, qb, sb, out_dtype=oracle.F32)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("act", ["gelu_tanh", "silu"])
def test_fp8_gemm_bias_activation(cuda_device, act):
    qa, sa, qb, sb = _quantised_problem(200, 300, 256, seed=77)
    bias = torch.from_numpy(synth.normal(77, 5, (300,), 0.5)).to(torch.bfloat16)
    got = _run_fp8(qa, sa, qb, sb, bias=bias, act=act)
    bb = bias.view(torch.int16).numpy().view(np.uint16)
    ref, acc = oracle.gemm_fp8(qa, sa, qb, sb, bias=bb, bias_dtype=oracle.BF16,
                               act={"gelu_tanh": oracle.ACT_GELU_TANH, "silu": oracle.ACT_SILU}[act],
                               out_dtype=oracle.BF16, want_absacc=True)
    check_tolerance(got, ref, acc, torch.bfloat16, what=f"fp8 {act}")


def test_quantise_then_gemm_end_to_end_on_gpu(cuda_device):
    """Both quantisations and the GEMM on the GPU; codes and scales must equal the
    oracle's, so the GEMM reference is computed from identical operands."""
    A = synth.normal_with_outliers(80, 0, (256, 512))
    B = synth.normal_with_outliers(80, 1, (512, 384))
    qa, sa = sg.quantize_fp8_blockwise(torch.from_numpy(A).cuda(), 1)
    qb, sb = sg.quantize_fp8_blockwise(torch.from_numpy(B).cuda(), 128)
    out = sg.gemm_fp8_blockscaled(qa, sa, qb, sb, out_dtype=torch.bfloat16)
    assert sg.check() == sg.OK
    qa_r, sa_r = oracle.quant_1x128(A)
    qb_r, sb_r = oracle.quant_128x128(B)
    assert np.array_equal(qa.cpu().numpy(), qa_r) and np.array_equal(qb.cpu().numpy(), qb_r)
    ref, acc = oracle.gemm_fp8(qa_r, sa_r, qb_r, sb_r, out_dtype=oracle.BF16, want_absacc=True)
    check_tolerance(out.float().cpu().numpy(), ref, acc, torch.bfloat16, what="quant+gemm")


# ------------------------------------------------------------------ partial last scale group (K % 128 != 0)

@pytest.mark.parametrize("K", [144, 400, 4112])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_fp8_ragged_k_quantise_then_gemm(cuda_device, monkeypatch, K, pair):
    """K not a multiple of 128: the last 1x128 group of every A row and the last
    128 x 128 block row of B hold K mod 128 elements, their scales come from those
    elements only, and the codes past K are never read (TMA zero fill). Both
    quantisations run on the GPU and must equal the oracle's bit for bit; the GEMM is
    then checked against the oracle on the same operands, on the CTA-pair (pair=1) and
    the one-SM (pair=0) kernels."""
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    M, N = 300, 260
    A = synth.normal_with_outliers(81, K, (M, K))
    B = synth.normal_with_outliers(82, K, (K, N))
    qa, sa = sg.quantize_fp8_blockwise(torch.from_numpy(A).cuda(), 1)
    qb, sb = sg.quantize_fp8_blockwise(torch.from_numpy(B).cuda(), 128)
    assert sg.check() == sg.OK
    qa_r, sa_r = oracle.quant_1x128(A)
    qb_r, sb_r = oracle.quant_128x128(B)
    assert np.array_equal(qa.cpu().numpy(), qa_r) and np.array_equal(sa.cpu().numpy().view(np.uint32),
                                                                     sa_r.view(np.uint32))
    assert np.array_equal(qb.cpu().numpy(), qb_r) and np.array_equal(sb.cpu().numpy().view(np.uint32),
                                                                     sb_r.view(np.uint32))
    out = torch.empty((M, -(-N // 8) * 8), dtype=torch.bfloat16, device="cuda")[:, :N]   # 16-byte row pitch
    sg.gemm_fp8_blockscaled(qa, sa, qb, sb, out=out)
    assert sg.check() == sg.OK
    ref, acc = oracle.gemm_fp8(qa_r, sa_r, qb_r, sb_r, out_dtype=oracle.BF16, want_absacc=True)
    check_tolerance(out.float().cpu().numpy(), ref, acc, torch.bfloat16, what=f"ragged K={K} pair={pair}")


@pytest.mark.parametrize("K", [144, 400, 4112])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_fp8_ragged_k_integer_codes_exact(cuda_device, monkeypatch, K, pair):
    """Integer codes with unit scales and a partial last K-block: every partial sum is
    exact, so the output equals the oracle's bit for bit; a code read past K (instead of
    the zero fill) or a dropped partial block would change it."""
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    rs = np.random.RandomState(K)
    M, N = 260, 300
    qa = oracle.e4m3_encode(rs.randint(-8, 9, (M, K)).astype(np.float32))
    qb = oracle.e4m3_encode(rs.randint(-8, 9, (N, K)).astype(np.float32))
    kb = -(-K // 128)
    sa = np.ones((kb, M), np.float32)
    sb = np.ones((kb, -(-N // 128)), np.float32)
    # rows are K apart, so bytes past K in a row are the next row's (non-zero) codes:
    # only the tensor map's bounds keep them out of the last K-block
    got = _run_fp8(qa, sa, qb, sb, out_dt=torch.float32)
    ref = oracle.gemm_fp8(qa, sa, qb, sb, out_dtype=oracle.F32)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("out_dt", [torch.float16, torch.float32])
@pytest.mark.parametrize("bias_dt", [torch.float32, torch.float16])
@pytest.mark.parametrize("pair", ["1", "0"])
def test_fp8_gemm_output_and_bias_types(cuda_device, monkeypatch, out_dt, bias_dt, pair):
    """F16 and F32 outputs with F32 and F16 bias (and SiLU) on both FP8 kernels."""
    monkeypatch.setenv("SMGEMM_PAIR", pair)
    qa, sa, qb, sb = _quantised_problem(200, 300, 400, seed=83)
    bias = torch.from_numpy(synth.normal(83, 5, (300,), 0.5)).to(bias_dt)
    got = _run_fp8(qa, sa, qb, sb, out_dt=out_dt, bias=bias, act="silu")
    bb, bd = orc_view(bias)
    ref, acc = oracle.gemm_fp8(qa, sa, qb, sb, bias=bb, bias_dtype=bd, act=oracle.ACT_SILU,
                               out_dtype=TORCH_TO_ORC[out_dt], want_absacc=True)
    check_tolerance(got, ref, acc, out_dt, what=f"fp8 out={out_dt} bias={bias_dt}")


# ------------------------------------------------------------------ seeded random sweep

def _fp8_sweep(n=64, seed=4242):
    rs = np.random.RandomState(seed)
    cases = []
    for i in range(n):
        cases.append(dict(M=int(rs.choice([int(rs.randint(1, 65)), int(rs.randint(65, 600))])),
                          N=int(rs.randint(1, 600)), K=16 * int(rs.randint(1, 64)),
                          pair=["1", "0"][rs.randint(2)], sched=["auto", "dp", "sk"][rs.randint(3)],
                          act=["none", "gelu_tanh", "silu"][rs.randint(3)], bias=bool(rs.randint(2)),
                          seed=500 + i))
    return cases


@pytest.mark.parametrize("case", _fp8_sweep(), ids=lambda c: "M{M}N{N}K{K}".format(**c))
def test_fp8_seeded_random_sweep(cuda_device, monkeypatch, case):
    """Random shapes (K any multiple of 16, so partial last scale groups are common),
    kernels, schedules, bias and activation: both quantisations on the GPU equal the
    oracle's bit for bit, and the block-scaled GEMM on those codes meets the contract."""
    monkeypatch.setenv("SMGEMM_PAIR", case["pair"])
    monkeypatch.setenv("SMGEMM_SCHED", case["sched"])
    M, N, K, s = case["M"], case["N"], case["K"], case["seed"]
    A = synth.normal_with_outliers(s, 0, (M, K))
    B = synth.normal_with_outliers(s, 1, (K, N))
    Bd = torch.zeros((K, -(-N // 4) * 4), dtype=torch.float32, device="cuda")  # 16-byte row pitch
    Bd[:, :N] = torch.from_numpy(B).cuda()
    qa, sa = sg.quantize_fp8_blockwise(torch.from_numpy(A).cuda(), 1)
    qb, sb = sg.quantize_fp8_blockwise(Bd[:, :N], 128)
    assert sg.check() == sg.OK
    qa_r, sa_r = oracle.quant_1x128(A)
    qb_r, sb_r = oracle.quant_128x128(B)
    assert np.array_equal(qa.cpu().numpy(), qa_r)
    assert np.array_equal(sa.cpu().numpy().view(np.uint32), sa_r.view(np.uint32))
    assert np.array_equal(qb.cpu().numpy(), qb_r)
    assert np.array_equal(sb.cpu().numpy().view(np.uint32), sb_r.view(np.uint32))
    bias = torch.from_numpy(synth.normal(s, 2, (N,), 0.5)).to(torch.bfloat16) if case["bias"] else None
    out = torch.empty((M, -(-N // 8) * 8), dtype=torch.bfloat16, device="cuda")[:, :N]
    sg.gemm_fp8_blockscaled(qa, sa, qb, sb, bias=None if bias is None else bias.cuda(), act=case["act"], out=out)
    assert sg.check() == sg.OK
    kw = {} if bias is None else dict(zip(("bias", "bias_dtype"), orc_view(bias)))
    act = {"none": oracle.ACT_NONE, "gelu_tanh": oracle.ACT_GELU_TANH, "silu": oracle.ACT_SILU}[case["act"]]
    ref, acc = oracle.gemm_fp8(qa_r, sa_r, qb_r, sb_r, act=act, out_dtype=oracle.BF16, want_absacc=True, **kw)
    check_tolerance(out.float().cpu().numpy(), ref, acc, torch.bfloat16, what=sg.last_config())
