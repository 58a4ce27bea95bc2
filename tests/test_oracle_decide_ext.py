"""Pins for the oracle's adaptive seed set, stochastic KL remasking and dynamic
threshold commit (CPU only).

  adaptive seed set  [COVER] section 2 ("small, adaptive" seed set): only scores
                     reaching min_score compete -- brute force over subsets.
  KL_STOCHASTIC      [DD] section 2, KL remasking "or probabilistically high":
                     REMASK iff U * tau < KL -- certain above tau, never at KL = 0,
                     frequency KL / tau below it (binomial bound), U uniform (KS).
  COMMIT             [SPOT] section 3, dynamic threshold decoding: hand-built cases
                     for the threshold, the progress rule and its tie rule.
"""
import itertools

import numpy as np
import pytest
from scipy import stats

from oracle import decide, philox, seeds


# ----------------------------------------------------------------------------- adaptive seeds
@pytest.mark.parametrize("trial", range(40))
def test_adaptive_seed_set_matches_brute_force(trial):
    rng = np.random.default_rng(500 + trial)
    L = int(rng.integers(1, 9))
    k = int(rng.integers(0, L + 2))
    s = rng.integers(0, 5, L).astype(float)
    s[rng.random(L) < 0.25] = -np.inf
    min_score = float(rng.integers(0, 4))
    got, is_seed = seeds.select(s, k, min_score)
    cands = [i for i in range(L) if np.isfinite(s[i]) and s[i] >= min_score]
    kk = min(k, len(cands))
    best = None
    for sub in itertools.combinations(cands, kk):
        key = sorted((-s[i], i) for i in sub)
        if best is None or key < best:
            best = key
    want = [i for _, i in best] + [-1] * (k - kk)
    assert list(got) == want
    assert int(is_seed.sum()) == kk


def test_adaptive_seed_set_size_and_reduction():
    s = np.array([5.0, 1.0, 3.0, 4.0, 0.5, 2.0])
    assert list(seeds.select(s, 4, 2.5)[0]) == [0, 3, 2, -1]      # three reach 2.5
    assert list(seeds.select(s, 2, 2.5)[0]) == [0, 3]             # capped at k
    assert list(seeds.select(s, 3, 3.0)[0]) == [0, 3, 2]          # >= is a candidate
    assert list(seeds.select(s, 3, 9.0)[0]) == [-1, -1, -1]       # nobody qualifies
    for k in range(7):
        assert np.array_equal(seeds.select(s, k, -np.inf)[0], seeds.select(s, k)[0])


def test_adaptive_margin_counts_the_threshold():
    s = np.array([5.0, 1.0, 3.00005, 4.0])
    assert seeds.boundary_margin(s, 2, 3.0) == pytest.approx(5e-5)  # 3.00005 vs min_score
    assert seeds.boundary_margin(s, 2) == pytest.approx(1.0 - 0.00005, rel=1e-9)
    assert seeds.boundary_margin(s, 0, 3.0) == np.inf


# ----------------------------------------------------------------------------- stochastic KL
def _kl_stats(kl):
    n = len(kl)
    z = np.zeros(n)
    return dict(kl_dt=np.asarray(kl, float), conf_t=z + 0.5, argmax_t=np.zeros(n, int),
                argmax_d=np.zeros(n, int), sample_t=np.zeros(n, int), sample_d=np.zeros(n, int),
                p_sample_t=z + 0.5, margin_t=z + np.inf, margin_d=z + np.inf)


def _kl_run(kl, tau=0.5, seed=7, step=3, b=1):
    n = len(kl)
    tok = np.arange(n) % 11
    one = np.ones(n, np.uint8)
    d, nt, _, near = decide.decide("kl_stochastic", tok, one, one, _kl_stats(kl), 0, n, 0.0, tau,
                                   0.9, seed=seed, step=step, b=b)
    return d, nt, near


def test_kl_stochastic_certain_above_threshold_never_at_zero():
    d, nt, _ = _kl_run(np.full(500, 0.5000001))
    assert np.all(d == decide.REMASK) and np.all(nt == -1)
    d, nt, _ = _kl_run(np.zeros(500))
    assert np.all(d == decide.KEEP)


@pytest.mark.parametrize("ratio", [0.1, 0.3, 0.8])
def test_kl_stochastic_frequency_is_kl_over_tau(ratio):
    n, tau = 4000, 0.5
    d, _, _ = _kl_run(np.full(n, ratio * tau), tau=tau, seed=int(ratio * 100))
    k = int((d == decide.REMASK).sum())
    # two-sided binomial test at a tight level: a wrong reading (1 - ratio, ratio^2,
    # a fixed threshold) lands far outside
    assert stats.binomtest(k, n, ratio).pvalue > 1e-4, (k, n * ratio)


def test_decision_draws_are_uniform_and_independent_of_sampling_noise():
    u = np.array([philox.decision_uniform(11, 5, 2, p) for p in range(3000)])
    assert np.all((u > 0) & (u < 1))
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    # the draw's counter word 0 is 2^31: never a vocabulary counter (v >> 2)
    w = philox.noise_words(11, 5, 2, 17, np.arange(0, 2**12))
    assert philox.uniform_from_word(w[0]) != philox.decision_uniform(11, 5, 2, 17)


# ----------------------------------------------------------------------------- commit
def _commit_case(p, masked, tau_commit, min_commit, pred=None, T=0.0):
    n = len(p)
    tok = np.where(masked, -1, 9)
    pred = np.arange(100, 100 + n) if pred is None else pred
    st = dict(kl_dt=np.zeros(n), conf_t=np.asarray(p, float), argmax_t=pred, argmax_d=pred,
              sample_t=pred, sample_d=pred, p_sample_t=np.asarray(p, float),
              margin_t=np.full(n, np.inf), margin_d=np.full(n, np.inf))
    elig = (~np.asarray(masked)).astype(np.uint8)
    return decide.decide("trust", tok, elig, elig, st, 0, n, T, 0.5, 0.9,
                         tau_commit=tau_commit, min_commit=min_commit)


def test_commit_threshold():
    p = [0.95, 0.40, 0.90, 0.99, 0.20]
    masked = np.array([1, 1, 1, 0, 1], bool)
    d, nt, acc, _ = _commit_case(p, masked, 0.9, 0)
    assert list(d) == [decide.COMMIT, decide.NONE, decide.COMMIT, decide.KEEP, decide.NONE]
    assert list(nt) == [100, -1, 102, 9, -1]
    assert acc == 1  # commits do not enter accepted


def test_commit_progress_rule_and_its_tie():
    p = [0.30, 0.60, 0.10, 0.60, 0.99]
    masked = np.array([1, 1, 1, 1, 0], bool)   # the 0.99 row is not masked
    d, nt, _, near = _commit_case(p, masked, 0.9, 1)
    assert list(d) == [0, decide.COMMIT, 0, 0, decide.KEEP]  # most confident, lower position
    assert nt[1] == 101 and nt[3] == -1
    assert near[1] and near[3]                               # a tie: flagged near
    d, _, _, _ = _commit_case(p, masked, 0.9, 0)
    assert not np.any(d == decide.COMMIT)                    # no progress rule: nothing
    d, _, _, _ = _commit_case(p, masked, 0.0, 1)
    assert not np.any(d == decide.COMMIT)                    # commit disabled


def test_commit_uses_the_sample_at_positive_temperature():
    p = [0.95]
    st_pred = np.array([7])
    d, nt, _, _ = _commit_case(p, np.array([1], bool), 0.9, 0, pred=st_pred, T=1.0)
    assert d[0] == decide.COMMIT and nt[0] == 7
