"""Vocabulary-parallel LM head with its row log-softmax, one process per GPU.

The LM head is the thin-and-tall GEMM X[M, K] * W[K, V] of "为什么我们要死磕GEMM"
(kwkr.cn), sections 2.2 and 7.2: at decode sizes its time is the time to stream W
from HBM. Splitting W by columns (the vocabulary) over g GPUs gives each one V/g
columns to stream, so the g GPUs bring g times the bandwidth to one token batch.

Each rank holds only its slice W[:, c0:c1] (``shard_columns``). One step is:
  1. gemm_bf16_lse_partials on the slice: the slice's logits and, per 128-column tile
     and row, (max, sum of exp) - the skinny kernel's epilogue forms these pairs;
  2. an all-gather of those pairs, padded to the same count on every rank with the
     neutral pair (-inf, 0) - M * ceil(V/(128 g)) * 8 bytes per rank, the only exchange;
  3. logsoftmax_apply_partials: every rank merges all pairs in the same fixed order (so
     all ranks get the same log-sum-exp, bit for bit) and subtracts it from its slice;
  4. optionally an all-gather of the slices into the full [M, V] log-probabilities.
The arithmetic of every step runs in the library's kernels; this module only splits,
pads and moves data (torch.distributed; NCCL on GPUs).
"""
from __future__ import annotations

from types import SimpleNamespace

TILE = 128


def shard_columns(n: int, world: int, rank: int, align: int = TILE):
    """Columns [c0, c1) of rank `rank` when n columns are split over `world` ranks in
    contiguous slices whose boundaries are multiples of `align` (the kernels' tile
    width), as even as that allows; the last slices may be shorter or empty."""
    units = -(-n // align)
    base, extra = divmod(units, world)
    u0 = rank * base + min(rank, extra)
    u1 = u0 + base + (1 if rank < extra else 0)
    return min(n, u0 * align), min(n, u1 * align)


def max_tiles(n: int, world: int, align: int = TILE) -> int:
    """The largest number of 128-column tiles any rank's slice has."""
    return max(-(-(c1 - c0) // TILE) for c0, c1 in (shard_columns(n, world, r, align) for r in range(world)))


def _library_ops():
    import sm_gemm_b200 as sg
    return SimpleNamespace(lse_partials=sg.gemm_bf16_lse_partials, apply_partials=sg.logsoftmax_apply_partials)


def lm_head_log_softmax(X, W_slice, n_total: int, *, bias_slice=None, dist=None, gather=False, ops=None,
                        workspace=None, out=None):
    """Log-probabilities of this rank's vocabulary slice (or of the whole vocabulary with
    gather=True) for X[M, K] against the slice W_slice[K, c1 - c0] of a V = n_total column
    head split by ``shard_columns``. ``dist`` is torch.distributed (initialised) or None
    for one process. Returns (log-probabilities, lse[M])."""
    import torch
    ops = ops or _library_ops()
    world = dist.get_world_size() if dist is not None else 1
    rank = dist.get_rank() if dist is not None else 0
    c0, c1 = shard_columns(n_total, world, rank)
    M = X.shape[0]
    if W_slice.shape[1] != c1 - c0:
        raise ValueError(f"rank {rank}: W slice has {W_slice.shape[1]} columns, the split gives {c1 - c0}")
    C, part = ops.lse_partials(X, W_slice, bias=bias_slice, out=out, workspace=workspace)
    P = max_tiles(n_total, world)
    if part.shape[0] < P:  # pad with the neutral pair (-inf, 0)
        pad = torch.zeros((P - part.shape[0], M, 2), dtype=part.dtype, device=part.device)
        pad[:, :, 0] = float("-inf")
        part = torch.cat([part, pad], dim=0)
    if world > 1:
        every = torch.empty((world * P, M, 2), dtype=part.dtype, device=part.device)
        dist.all_gather_into_tensor(every, part.contiguous())
    else:
        every = part
    lse = ops.apply_partials(C, every)
    if not gather or world == 1:
        return C, lse
    width = max(b - a for a, b in (shard_columns(n_total, world, r) for r in range(world)))
    mine = torch.zeros((M, width), dtype=C.dtype, device=C.device)
    mine[:, :c1 - c0] = C
    slabs = torch.empty((world * M, width), dtype=C.dtype, device=C.device)  # rank r: rows r*M ..
    dist.all_gather_into_tensor(slabs, mine)
    full = torch.empty((M, n_total), dtype=C.dtype, device=C.device)
    for r in range(world):
        a, b = shard_columns(n_total, world, r)
        full[:, a:b] = slabs[r * M:(r + 1) * M, :b - a]
    return full, lse
