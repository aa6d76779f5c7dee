"""Offline schedule sweep for the shapes the library is benchmarked on (needs a B200).

    python -m sm_gemm_b200.tune [--write]

For each shape it times every candidate schedule (grouped-raster band height
SMGEMM_GROUP_M in {4, 8, 16}; ragged-last-wave split on or off, SMGEMM_SPLITK 0 / 1)
with CUDA events over 20 calls (three rounds, the best round kept), and prints the
fastest. With --write it rewrites csrc/tuned_configs.inc, the static table the planner
consults for exactly these shapes (rebuild the library afterwards), and tuned_configs.json
with the measured time of each chosen schedule, which the performance-floor test reads.
This is the "sweep offline, ship a per-shape table" practice of the DeepGEMM
kernel-library walkthrough (zwxr.cn), section 5.2.
"""
from __future__ import annotations

import json
import os
import sys

HERE = os.path.dirname(os.path.abspath(__file__))
ROOT = os.path.dirname(HERE)
sys.path.insert(0, ROOT)

# (name, kind, M, N, K, layout of A, layout of B): the square GEMM, the FFN layer's two
# GEMMs and backward GEMMs, and the FP8 GEMMs (kind 1)
SHAPES = [
    ("square_bf16_4096", 0, 4096, 4096, 4096, "row", "col"),
    ("ffn_gemm1", 0, 1024, 16384, 4096, "row", "row"),
    ("ffn_gemm2", 0, 1024, 4096, 16384, "row", "row"),
    ("ffn_backward_dX", 0, 1024, 4096, 16384, "row", "col"),
    ("ffn_backward_dW1", 0, 4096, 16384, 1024, "col", "row"),
    ("fp8_blockscaled", 1, 2048, 16384, 4096, "row", "col"),
    ("ffn_gemm2_fp8", 1, 1024, 4096, 16384, "row", "col"),
]
CANDIDATES = [(g, s) for g in (4, 8, 16) for s in (0, 1)]


def _operands(torch, kind, M, N, K, la, lb, dev):
    g = torch.Generator(device="cpu").manual_seed(M * 31 + N * 7 + K)
    if kind == 1:
        qa = torch.randint(0, 0x7E, (M, K), dtype=torch.uint8, generator=g).to(dev)
        qb = torch.randint(0, 0x7E, (N, K), dtype=torch.uint8, generator=g).to(dev)
        sa = torch.rand((K // 128, M), generator=g).to(dev) + 0.5
        sb = torch.rand((K // 128, -(-N // 128)), generator=g).to(dev) + 0.5
        return qa, sa, qb, sb
    A = torch.randn((M, K) if la == "row" else (K, M), generator=g).to(torch.bfloat16).to(dev)
    B = torch.randn((K, N) if lb == "row" else (N, K), generator=g).to(torch.bfloat16).to(dev)
    return (A if la == "row" else A.t()), (B if lb == "row" else B.t())


def time_shape(sg, torch, kind, M, N, K, la, lb, calls=20, rounds=3):
    dev = torch.device("cuda", torch.cuda.current_device())
    ops = _operands(torch, kind, M, N, K, la, lb, dev)
    out = torch.empty((M, N), dtype=torch.bfloat16, device=dev)
    ws = torch.empty(max(sg.workspace_size(M, N, K, kind), 16) * 2, dtype=torch.uint8, device=dev)
    if kind == 1:
        run = lambda: sg.gemm_fp8_blockscaled(*ops, out=out, workspace=ws)
    else:
        run = lambda: sg.gemm_bf16(*ops, out=out, workspace=ws)
    best = float("inf")
    for _ in range(rounds):
        for _ in range(3):
            run()
        torch.cuda.synchronize()
        s, e = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        s.record()
        for _ in range(calls):
            run()
        e.record()
        torch.cuda.synchronize()
        best = min(best, s.elapsed_time(e) / calls * 1e3)
    assert sg.check() == sg.OK
    return best


def main():
    import torch
    import sm_gemm_b200 as sg
    write = "--write" in sys.argv
    rows, record = [], {}
    for name, kind, M, N, K, la, lb in SHAPES:
        times = {}
        for group_m, splitk in CANDIDATES:
            os.environ["SMGEMM_GROUP_M"] = str(group_m)
            os.environ["SMGEMM_SPLITK"] = str(splitk)
            times[(group_m, splitk)] = time_shape(sg, torch, kind, M, N, K, la, lb)
        os.environ.pop("SMGEMM_GROUP_M")
        os.environ.pop("SMGEMM_SPLITK")
        (g, s), us = min(times.items(), key=lambda kv: kv[1])
        print(name, {f"g{a}s{b}": round(t, 2) for (a, b), t in times.items()}, "->", (g, s), round(us, 2), flush=True)
        rows.append(f"    {{{kind}, {M}, {N}, {K}, {0 if la == 'row' else 1}, {g}, {s}}},  // {name}: {us:.1f} us")
        record[name] = {"kind": kind, "M": M, "N": N, "K": K, "layout_a": la, "layout_b": lb, "group_m": g,
                        "splitk": s, "us": round(us, 2),
                        "candidates_us": {f"group_m={a},splitk={b}": round(t, 2) for (a, b), t in times.items()}}
    if write:
        with open(os.path.join(HERE, "csrc", "tuned_configs.inc"), "w") as f:
            f.write("// Per-shape schedule choices measured on B200 (written by sm_gemm_b200/tune.py; the\n"
                    "// heuristics of make_plan apply to every shape not listed).\n"
                    "// {kind (0 = 16-bit, 1 = FP8), M, N, K, layout_a (0 = row-major), group_m, splitk "
                    "(0 = tail split, 1 = none)}\n")
            f.write("\n".join(rows) + "\n")
        with open(os.path.join(HERE, "tuned_configs.json"), "w") as f:
            json.dump({"device": torch.cuda.get_device_name(), "shapes": record}, f, indent=1)


if __name__ == "__main__":
    main()
