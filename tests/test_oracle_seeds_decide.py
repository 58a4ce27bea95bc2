"""Pins for the oracle's seed selection and decision policies (CPU only).

Golden fixtures under tests/golden/ (hand arithmetic on the page's score
equation; hand-built revision outcomes, each file citing its page section),
plus brute-force top-k on tiny inputs.
"""
import itertools
import os

import numpy as np
import pytest

from oracle import decide, seeds

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rows(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return [ln.split() for ln in f if ln.strip() and not ln.startswith("#")]


def test_stability_score_golden():
    for u, din, dout, want in _rows("stability_score.txt"):
        got = seeds.stability_score([float(u)], [float(din)], [float(dout)], [1])[0]
        assert got == pytest.approx(float(want), rel=1e-15)


def test_ineligible_positions_score_minus_inf():
    s = seeds.stability_score([1, 2, 3], [0, 0, 0], [0, 0, 0], [1, 0, 1])
    assert s[1] == -np.inf and s[0] == 1 and s[2] == 3


@pytest.mark.parametrize("trial", range(30))
def test_topk_matches_brute_force(trial):
    rng = np.random.default_rng(trial)
    L = int(rng.integers(1, 9))
    k = int(rng.integers(0, L + 2))
    # small integer scores to force ties
    score = rng.integers(0, 3, L).astype(float)
    score[rng.random(L) < 0.3] = -np.inf
    got, is_seed = seeds.select(score, k)
    # brute force: among all subsets of size min(k, #finite), the chosen one is the
    # lexicographically best list of (-score, position) pairs
    finite = [i for i in range(L) if np.isfinite(score[i])]
    kk = min(k, len(finite))
    best = None
    for sub in itertools.combinations(finite, kk):
        key = sorted((-score[i], i) for i in sub)
        if best is None or key < best:
            best = key
    want = [i for _, i in best] + [-1] * (k - kk)
    assert list(got) == want
    assert sorted(np.nonzero(is_seed)[0].tolist()) == sorted(i for i in want if i >= 0)


def test_ties_go_to_lower_position():
    got, _ = seeds.select([1.0, 2.0, 2.0, 2.0, 0.5], 2)
    assert list(got) == [1, 2]


CODES = {"NONE": decide.NONE, "KEEP": decide.KEEP, "REPLACE": decide.REPLACE,
         "REMASK": decide.REMASK}


def test_revision_outcomes_golden():
    rows = _rows("revision_outcomes.txt")
    assert len(rows) >= 15
    for (policy, dom, cur, am_t, am_d, conf, p_pred, kl, tau_kl, tau_conf, want,
         want_tok) in rows:
        stats = dict(kl_dt=[float(kl)], conf_t=[float(conf)], argmax_t=[int(am_t)],
                     argmax_d=[int(am_d)], sample_t=[int(am_t)], sample_d=[int(am_d)],
                     p_sample_t=[float(p_pred)], margin_t=[np.inf], margin_d=[np.inf])
        flag = [int(dom)]
        d, nt, acc, near = decide.decide(policy, [int(cur)], flag, flag, stats, pos_offset=0,
                                         R=1, temperature=0.0, tau_kl=float(tau_kl),
                                         tau_conf=float(tau_conf))
        assert d[0] == CODES[want], (policy, want)
        assert nt[0] == int(want_tok), (policy, want_tok)
        assert acc == int(want in ("KEEP", "NONE"))


def test_positions_without_rows_are_not_decided():
    stats = dict(kl_dt=[9.0], conf_t=[0.1], argmax_t=[1], argmax_d=[2], sample_t=[1],
                 sample_d=[2], p_sample_t=[0.1], margin_t=[np.inf], margin_d=[np.inf])
    d, nt, acc, _ = decide.decide("kl", [4, 4, 4], [1, 1, 1], [1, 1, 1], stats, pos_offset=1,
                                  R=1, temperature=0.0, tau_kl=0.5, tau_conf=0.9)
    assert list(d) == [decide.NONE, decide.REMASK, decide.NONE]
    assert list(nt) == [4, -1, 4] and acc == 0


def test_near_threshold_flagged():
    stats = dict(kl_dt=[0.50001], conf_t=[0.5], argmax_t=[1], argmax_d=[1], sample_t=[1],
                 sample_d=[1], p_sample_t=[0.5], margin_t=[np.inf], margin_d=[np.inf])
    _, _, _, near = decide.decide("kl", [1], [1], [1], stats, 0, 1, 0.0, 0.5, 0.9)
    assert near[0]
