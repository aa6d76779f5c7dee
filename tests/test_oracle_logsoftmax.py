"""Pins of the oracle's row log-softmax (the LM-head epilogue of "为什么我们要死磕GEMM",
section 7.2) against closed forms, invariants and a library routine."""
import math

import numpy as np
import scipy.special

import oracle


def test_constant_row_is_minus_log_n():
    for n in (1, 7, 128256):
        out, lse = oracle.log_softmax_rows(np.full((2, n), 3.25))
        assert np.allclose(out, -math.log(n), rtol=0, atol=1e-12)
        assert np.allclose(lse, 3.25 + math.log(n), rtol=0, atol=1e-12)


def test_two_element_closed_form():
    out, lse = oracle.log_softmax_rows(np.array([[0.0, math.log(3.0)]]))
    assert abs(out[0, 0] + math.log(4.0)) < 1e-15
    assert abs(out[0, 1] - (math.log(3.0) - math.log(4.0))) < 1e-15
    assert abs(lse[0] - math.log(4.0)) < 1e-15


def test_large_logits_do_not_overflow():
    out, lse = oracle.log_softmax_rows(np.array([[1000.0, 1000.0, -1000.0]]))
    assert abs(out[0, 0] + math.log(2.0)) < 1e-12 and abs(out[0, 1] + math.log(2.0)) < 1e-12
    assert out[0, 2] < -1999.0 and np.isfinite(out).all()
    assert abs(lse[0] - (1000.0 + math.log(2.0))) < 1e-12


def test_probabilities_sum_to_one_and_shift_invariance():
    rng = np.random.default_rng(3)
    z = rng.normal(0, 4, (5, 1000))
    out, _ = oracle.log_softmax_rows(z)
    assert np.allclose(np.exp(out).sum(axis=1), 1.0, rtol=0, atol=1e-12)
    out2, _ = oracle.log_softmax_rows(z + rng.normal(0, 100, (5, 1)))
    assert np.allclose(out, out2, rtol=0, atol=1e-10)
    assert (out <= 0).all()


def test_matches_scipy():
    rng = np.random.default_rng(4)
    z = rng.normal(0, 10, (3, 5000))
    out, _ = oracle.log_softmax_rows(z)
    assert np.allclose(out, scipy.special.log_softmax(z, axis=1), rtol=0, atol=1e-10)
