"""The seeded input generator: determinism, sub-block regeneration and the value
distributions the workloads ask for (N(0, std) by standard deviation, U[-1, 1],
1% outliers x50)."""
import numpy as np

import synth


def test_deterministic_and_seed_dependent():
    a = synth.normal(1, 0, (1000,))
    assert (a == synth.normal(1, 0, (1000,))).all()
    assert not (a == synth.normal(2, 0, (1000,))).all()
    assert not (a == synth.normal(1, 1, (1000,))).all()


def test_chunked_generation_equals_one_shot():
    n = (1 << 22) + 12345                      # crosses the parallel chunk boundary
    a = synth.normal(3, 5, (n,))
    key = synth.stream_key(3, 5)
    tail = synth._normal_chunk(key, n - 1001, 1001).astype(np.float32)
    assert (a[-1001:] == tail).all()
    odd = synth._normal_chunk(key, 7, 10).astype(np.float32)   # odd start: second of a pair
    assert (a[7:17] == odd).all()


def test_distributions():
    z = synth.normal(4, 0, (1 << 20,)).astype(np.float64)
    assert abs(z.mean()) < 5e-3 and abs(z.std() - 1) < 5e-3
    w = synth.normal(4, 1, (1 << 20,), 0.02).astype(np.float64)
    assert abs(w.std() - 0.02) < 1e-4
    u = synth.uniform(4, 2, (1 << 20,)).astype(np.float64)
    assert u.min() >= -1 and u.max() < 1 and abs(u.mean()) < 5e-3
    o = synth.normal_with_outliers(4, 3, (1 << 20,)).astype(np.float64)
    frac = (np.abs(o) > 6).mean()               # |N(0,1)| > 6 is ~2e-9; x50 outliers mostly exceed it
    assert 0.008 < frac < 0.0105


def test_workload_shapes():
    t = synth.tiny_fp16()
    assert t["A"].shape == (64, 64) and t["B"].shape == (64, 64)
    f = synth.ffn_pair(tokens=8, d_model=16, d_ff=32)
    assert f["X"].shape == (8, 16) and f["W1"].shape == (16, 32) and f["W2"].shape == (32, 16)
    assert f["b1"].shape == (32,)
    l1, l2 = synth.lm_head(m=2, d_model=8, vocab=40), synth.lm_head(m=3, d_model=8, vocab=40)
    assert (l1["W"] == l2["W"]).all()           # one weight shared by every M


def test_splitmix64_reference_sequence():
    """The counter-based stream equals the published sequential generator: output i of
    stream `key` is the finaliser of key + (i + 1) * gamma, so key = 1234567 must give
    the generator's check values for that initial state (tests/golden)."""
    import os
    path = os.path.join(os.path.dirname(__file__), "golden", "splitmix64_state_1234567.txt")
    want = [int(l) for l in open(path) if l.strip() and not l.startswith("#")]
    got = synth._bits(1234567, 0, len(want))
    assert [int(v) for v in got] == want
    assert [int(v) for v in synth._bits(1234567, 2, 3)] == want[2:]   # any counter range alone
