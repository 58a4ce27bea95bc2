"""Pins for the oracle's per-row vocabulary statistics (CPU only).

Checked against scipy's logsumexp / entropy / rel_entr, closed forms
(constant rows, two-token KL), invariants (KL >= 0, KL(p||p) = 0,
0 <= H <= ln V, shift invariance) and the lowest-index tie rule.
"""
import math

import numpy as np
import pytest
from scipy import special, stats

from oracle import vocab


def _rows(n=20, V=257, seed=0):
    rng = np.random.default_rng(seed)
    l = rng.normal(0, 3, size=(n, V))
    l[np.arange(n), rng.integers(0, V, n)] += 8 * (rng.random(n) < 0.7)
    m = l + rng.normal(0, 1, size=(n, V))
    return l, m


def test_against_scipy():
    l, m = _rows()
    s = vocab.row_stats(l, m)
    np.testing.assert_allclose(s["lse_t"], special.logsumexp(l, axis=1), rtol=1e-13)
    np.testing.assert_allclose(s["lse_d"], special.logsumexp(m, axis=1), rtol=1e-13)
    p_t = special.softmax(l, axis=1)
    p_d = special.softmax(m, axis=1)
    np.testing.assert_allclose(s["entropy_t"], stats.entropy(p_t, axis=1), rtol=1e-10)
    np.testing.assert_allclose(s["kl_dt"], special.rel_entr(p_d, p_t).sum(1), rtol=1e-10)
    np.testing.assert_allclose(s["conf_t"], p_t.max(1), rtol=1e-13)


def test_constant_row_closed_form():
    V = 1000
    l = np.full((1, V), 2.5)
    s = vocab.row_stats(l, l)
    assert math.isclose(s["lse_t"][0], 2.5 + math.log(V), rel_tol=1e-14)
    assert math.isclose(s["entropy_t"][0], math.log(V), rel_tol=1e-13)
    assert math.isclose(s["conf_t"][0], 1 / V, rel_tol=1e-12)
    assert s["kl_dt"][0] == 0.0
    assert s["argmax_t"][0] == 0  # all tied -> lowest index


def test_dominant_logit_zero_entropy():
    l = np.zeros((1, 50))
    l[0, 17] = 1000.0
    s = vocab.row_stats(l, l)
    assert s["entropy_t"][0] < 1e-12
    assert math.isclose(s["conf_t"][0], 1.0)
    assert s["argmax_t"][0] == 17


def test_two_token_kl_closed_form():
    a, b = 0.8, 0.3
    m = np.log([[a, 1 - a]])
    l = np.log([[b, 1 - b]])
    s = vocab.row_stats(l, m)
    want = a * math.log(a / b) + (1 - a) * math.log((1 - a) / (1 - b))
    assert math.isclose(s["kl_dt"][0], want, rel_tol=1e-12)
    # direction: KL(drafter || verifier), not the reverse
    rev = b * math.log(b / a) + (1 - b) * math.log((1 - b) / (1 - a))
    assert not math.isclose(s["kl_dt"][0], rev, rel_tol=1e-3)


def test_invariants_random_rows():
    l, m = _rows(n=50, V=1000, seed=3)
    s = vocab.row_stats(l, m)
    assert np.all(s["kl_dt"] >= 0)
    assert np.all(s["entropy_t"] >= 0) and np.all(s["entropy_t"] <= math.log(1000) + 1e-12)
    s2 = vocab.row_stats(l, l)
    np.testing.assert_allclose(s2["kl_dt"], 0, atol=1e-12)
    # shift invariance
    s3 = vocab.row_stats(l + 7.0, m - 3.0)
    np.testing.assert_allclose(s3["entropy_t"], s["entropy_t"], rtol=1e-10)
    np.testing.assert_allclose(s3["kl_dt"], s["kl_dt"], rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(s3["lse_t"], s["lse_t"] + 7.0, rtol=1e-13)
    assert np.array_equal(s3["argmax_t"], s["argmax_t"])


def test_argmax_lowest_index_on_ties():
    l = np.array([[1.0, 3.0, 2.0, 3.0, 3.0]])
    s = vocab.row_stats(l, l[:, ::-1])
    assert s["argmax_t"][0] == 1
    assert s["argmax_d"][0] == 0


def test_verify_rows_temperature_zero_uses_argmax():
    l, m = _rows(n=8, V=100)
    out = vocab.verify_rows(l, m, 0.0, seed=0, step=0, b=0, positions=np.arange(8))
    assert np.array_equal(out["sample_t"], out["argmax_t"])
    np.testing.assert_allclose(out["p_sample_t"], out["conf_t"], rtol=1e-13)


def test_verify_rows_sampled_probability():
    l, m = _rows(n=8, V=100)
    out = vocab.verify_rows(l, m, 1.0, seed=5, step=1, b=0, positions=np.arange(8) + 3)
    p_t = special.softmax(l, axis=1)
    np.testing.assert_allclose(out["p_sample_t"], p_t[np.arange(8), out["sample_t"]], rtol=1e-12)


def test_single_entry_vocabulary():
    l = np.array([[1.5], [-2.0]])
    out = vocab.verify_rows(l, l + 1, 1.0, seed=0, step=0, b=0, positions=np.arange(2))
    assert list(out["sample_t"]) == [0, 0] and np.all(np.isinf(out["margin_t"]))
    np.testing.assert_allclose(out["entropy_t"], 0, atol=1e-15)
    np.testing.assert_allclose(out["conf_t"], 1.0)
