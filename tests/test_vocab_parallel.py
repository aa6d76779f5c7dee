"""Host logic of the vocabulary-parallel LM head (sm_gemm_b200.vocab_parallel) on CPU
ranks over gloo: the column split, the padding and all-gather of the per-tile
(max, sum of exp) pairs, the global log-sum-exp merge and the gather of the slices.

The library's two kernels (GEMM with partials; merge and subtract) are replaced here by
plain float64 stand-ins with the same inputs and outputs, so the test checks what this
module adds on top of them: every rank must end with the row log-softmax of the whole
vocabulary (the oracle's log_softmax_rows on the full logits), the same lse bit for bit
on every rank, and - with gather - the full [M, V] log-probabilities. World sizes 2 and
4; with V = 300 and 4 ranks the last slice is empty.
"""
import os
import socket
from types import SimpleNamespace

import numpy as np
import pytest
import torch

from sm_gemm_b200 import vocab_parallel as vp


def test_shard_columns_cover_once_tile_aligned():
    for n in (1, 127, 128, 300, 1000, 128256):
        for world in (1, 2, 3, 4, 8):
            spans = [vp.shard_columns(n, world, r) for r in range(world)]
            assert spans[0][0] == 0 and spans[-1][1] == n
            for (a0, a1), (b0, b1) in zip(spans, spans[1:]):
                assert a1 == b0
            for a, b in spans:
                assert a <= b and (a % 128 == 0 or a == n)
            tiles = [-(-(b - a) // 128) for a, b in spans]
            assert max(tiles) - min(tiles) <= 1                  # as even as whole tiles allow
            assert vp.max_tiles(n, world) == max(tiles)


def _standin_ops():
    """float64 restatements of the two library calls (definitions, not the kernels)."""
    def lse_partials(X, W, bias=None, out=None, workspace=None):
        z = X.double() @ W.double()
        if bias is not None:
            z = z + bias.double()
        M, N = z.shape
        T = -(-N // 128)
        part = torch.empty((T, M, 2), dtype=torch.float64)
        for t in range(T):
            blk = z[:, 128 * t:128 * t + 128]
            mx = blk.max(dim=1).values
            part[t, :, 0] = mx
            part[t, :, 1] = torch.exp(blk - mx[:, None]).sum(dim=1)
        return z, part

    def apply_partials(C, part):
        m = torch.full((part.shape[1],), float("-inf"), dtype=torch.float64)
        s = torch.zeros(part.shape[1], dtype=torch.float64)
        for p in range(part.shape[0]):        # the online merge, in part order
            pm, ps = part[p, :, 0], part[p, :, 1]
            live = ps > 0
            new = torch.where(live, torch.maximum(m, pm), m)
            s = torch.where(live, s * torch.exp(m - new).nan_to_num(0.0) + ps * torch.exp(pm - new), s)
            m = new
        lse = m + torch.log(s)
        C -= lse[:, None]
        return lse

    return SimpleNamespace(lse_partials=lse_partials, apply_partials=apply_partials)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank(rank, world, port, M, K, V, gather, q):
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        rs = np.random.RandomState(7)
        X = torch.from_numpy(rs.standard_normal((M, K)))
        W = torch.from_numpy(rs.standard_normal((K, V)) * 0.5)
        b = torch.from_numpy(rs.standard_normal(V))
        c0, c1 = vp.shard_columns(V, world, rank)
        out, lse = vp.lm_head_log_softmax(X, W[:, c0:c1].contiguous(), V, bias_slice=b[c0:c1].contiguous(),
                                          dist=dist, gather=gather, ops=_standin_ops())
        q.put((rank, c0, c1, out.numpy(), lse.numpy()))
    finally:
        dist.destroy_process_group()


@pytest.mark.parametrize("world,V,gather", [(2, 1000, True), (2, 1000, False), (4, 300, True)])
def test_vocab_parallel_log_softmax_matches_full_row(world, V, gather):
    import multiprocessing as mp
    import oracle
    M, K = 5, 64
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank, args=(r, world, port, M, K, V, gather, q)) for r in range(world)]
    for p in procs:
        p.start()
    res = sorted(q.get(timeout=90) for _ in range(world))
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    rs = np.random.RandomState(7)
    X = rs.standard_normal((M, K))
    W = rs.standard_normal((K, V)) * 0.5
    b = rs.standard_normal(V)
    want, want_lse = oracle.log_softmax_rows(X @ W + b)
    lses = [r[4] for r in res]
    for l in lses[1:]:
        assert np.array_equal(l, lses[0])                    # one lse, bit for bit, on every rank
    np.testing.assert_allclose(lses[0], want_lse, rtol=0, atol=1e-9)
    for rank, c0, c1, out, lse in res:
        if gather:
            np.testing.assert_allclose(out, want, rtol=0, atol=1e-9)
        else:
            assert out.shape == (M, c1 - c0)
            np.testing.assert_allclose(out, want[:, c0:c1], rtol=0, atol=1e-9)
    assert sum(c1 - c0 for _, c0, c1, _, _ in res) == V
