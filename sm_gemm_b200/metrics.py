"""Work and traffic counts used to report throughput and roofline fractions.

FLOPs follow the pages' convention: a multiply-add is two operations, so a GEMM of
[M,K] x [K,N] is 2*M*N*K ("为什么我们要死磕GEMM", kwkr.cn, section 3.1; DeepGEMM
kernel-library walkthrough, zwxr.cn, section 3.4). The epilogue is not counted.
Algorithmic bytes read every operand once and write the output once; re-reads
served by L2 are not counted.
"""

ELEM_BYTES = {"f32": 4, "bf16": 2, "f16": 2, "e4m3": 1}


def gemm_flops(M: int, N: int, K: int) -> int:
    return 2 * M * N * K


def tflops(flops: float, seconds: float) -> float:
    return flops / seconds / 1e12


def gemm_bytes(M: int, N: int, K: int, a: str, b: str, c: str, bias: str | None = None) -> int:
    n = M * K * ELEM_BYTES[a] + K * N * ELEM_BYTES[b] + M * N * ELEM_BYTES[c]
    if bias is not None:
        n += N * ELEM_BYTES[bias]
    return n


def fp8_gemm_bytes(M: int, N: int, K: int, c: str, bias: str | None = None) -> int:
    kb = -(-K // 128)
    nb = -(-N // 128)
    n = M * K + N * K + 4 * (kb * M + kb * nb) + M * N * ELEM_BYTES[c]
    if bias is not None:
        n += N * ELEM_BYTES[bias]
    return n


def quant_bytes(rows: int, cols: int, group_rows: int) -> int:
    """fp32 input read once, one code byte per element and one fp32 scale per group written."""
    groups = rows * (-(-cols // 128)) if group_rows == 1 else (-(-rows // 128)) * (-(-cols // 128))
    return rows * cols * 4 + rows * cols + groups * 4
