"""Pins for the oracle's near-tie margins (CPU only).

The GPU parity tests skip a row or a sequence only when the oracle says its
decision sits within 1e-4 of a tie; these margins decide which. Each is pinned
against an independent brute-force definition on tiny inputs and against the
property that makes it the right margin: perturbing the scores by less than
half the margin cannot change the decision, and a perturbation just over half
of it, in the adverse direction, does.

  _top2_gap(x)            gap between the largest and the runner-up entry of a
                          row: the Gumbel-max / argmax decision of the coupled
                          samples ([SPOT] section 1, Coupled-Noise Verification)
  boundary_margin(s, k)   gap between the k-th and (k+1)-th finite scores: the
                          top-k seed set of [COVER] section 2 (Stability-Aware
                          Seed Selection)
"""
import itertools

import numpy as np
import pytest

from oracle import philox, seeds, vocab


# ----------------------------------------------------------------------------- top-2 gap
def _gap_brute(row):
    """Smallest lead of an argmax entry over any other entry (pairwise loops)."""
    row = [float(v) for v in row]
    if len(row) < 2:
        return np.inf
    best = max(range(len(row)), key=lambda i: (row[i], -i))
    return min(row[best] - row[j] for j in range(len(row)) if j != best)


@pytest.mark.parametrize("trial", range(40))
def test_top2_gap_matches_pairwise_brute_force(trial):
    rng = np.random.default_rng(trial)
    V = int(rng.integers(2, 9))
    x = rng.integers(-3, 4, size=(5, V)).astype(float)  # small integers: frequent ties
    x[::2] += rng.normal(0, 0.3, size=(3, V))
    got = vocab._top2_gap(x)
    want = np.array([_gap_brute(r) for r in x])
    assert np.array_equal(got, want)


def test_top2_gap_special_cases():
    assert vocab._top2_gap(np.array([[3.0, 1.0]]))[0] == 2.0          # V = 2: |a - b|
    assert vocab._top2_gap(np.array([[1.0, 3.0]]))[0] == 2.0
    assert vocab._top2_gap(np.array([[2.0, 5.0, 5.0, 1.0]]))[0] == 0.0  # tie at the top
    assert vocab._top2_gap(np.array([[7.0, 5.0, 6.0, 6.5]]))[0] == 0.5  # runner-up is not the 2nd entry
    assert np.isinf(vocab._top2_gap(np.array([[4.0]]))[0])             # no runner-up


@pytest.mark.parametrize("trial", range(20))
def test_top2_gap_is_the_argmax_stability_margin(trial):
    rng = np.random.default_rng(100 + trial)
    x = rng.normal(0, 2, size=(1, 7))
    gap = vocab._top2_gap(x)[0]
    top = int(np.argmax(x[0]))
    # any perturbation below half the gap keeps the argmax
    for _ in range(50):
        eps = rng.uniform(-1, 1, size=7) * 0.499 * gap
        assert int(np.argmax(x[0] + eps)) == top
    # pushing the leader down and the runner-up up by just over half the gap flips it
    runner = int(np.argsort(-x[0], kind="stable")[1])
    y = x[0].copy()
    y[top] -= 0.501 * gap
    y[runner] += 0.501 * gap
    assert int(np.argmax(y)) == runner


def test_coupled_margins_are_gaps_of_the_noisy_scores():
    # the margin of a coupled sample is the gap of l/T + g (what the argmax sees),
    # not of the logits alone
    rng = np.random.default_rng(7)
    V, T = 11, 0.7
    l = rng.normal(0, 3, size=(4, V))
    m = l + rng.normal(0, 1, size=(4, V))
    g = philox.gumbel(99, 3, 1, np.arange(4)[:, None] + 20, np.arange(V)[None, :])
    out = vocab.coupled_samples(l, m, T, g)
    for r in range(4):
        assert out["margin_t"][r] == _gap_brute(l[r] / T + g[r])
        assert out["margin_d"][r] == _gap_brute(m[r] / T + g[r])
        assert out["sample_t"][r] == int(np.argmax(l[r] / T + g[r]))


def test_sampled_rows_report_margins_and_argmax_rows_do_not():
    rng = np.random.default_rng(3)
    l = rng.normal(0, 3, size=(6, 50))
    m = l + rng.normal(0, 1, size=(6, 50))
    hot = vocab.verify_rows(l, m, 1.0, seed=1, step=2, b=0, positions=np.arange(6))
    assert np.all(np.isfinite(hot["margin_t"])) and np.all(hot["margin_t"] >= 0)
    cold = vocab.verify_rows(l, m, 0.0, seed=1, step=2, b=0, positions=np.arange(6))
    # at T = 0 both sides take the argmax of the same logit bits: no tolerance involved
    assert np.all(np.isinf(cold["margin_t"])) and np.all(np.isinf(cold["margin_d"]))


# ----------------------------------------------------------------------------- top-k boundary
def _boundary_brute(score, k):
    """Smallest lead of a chosen score over an unchosen finite score, taking the
    chosen set by brute force over all subsets (inf when nothing is contested)."""
    score = [float(s) for s in score]
    finite = [i for i, s in enumerate(score) if np.isfinite(s)]
    if k == 0 or len(finite) <= k:
        return np.inf
    best = None
    for sub in itertools.combinations(finite, k):
        key = sorted((-score[i], i) for i in sub)
        if best is None or key < best:
            best, chosen = key, set(sub)
    return min(score[i] - score[j] for i in chosen for j in finite if j not in chosen)


@pytest.mark.parametrize("trial", range(60))
def test_boundary_margin_matches_brute_force(trial):
    rng = np.random.default_rng(200 + trial)
    L = int(rng.integers(1, 9))
    k = int(rng.integers(0, L + 2))
    s = rng.integers(0, 4, L).astype(float)  # small integers: frequent ties
    s += rng.normal(0, 0.05, L) * (rng.random(L) < 0.5)
    s[rng.random(L) < 0.25] = -np.inf
    assert seeds.boundary_margin(s, k) == _boundary_brute(s, k)


def test_boundary_margin_special_cases():
    inf = np.inf
    assert seeds.boundary_margin([3.0, 1.0, 2.0], 0) == inf           # k = 0: nothing chosen
    assert seeds.boundary_margin([3.0, 1.0, -inf], 2) == inf          # k >= #finite
    assert seeds.boundary_margin([3.0, 1.0, 2.0], 3) == inf
    assert seeds.boundary_margin([3.0, 1.0, 2.0], 1) == 1.0           # 3 vs 2
    assert seeds.boundary_margin([3.0, 1.0, 2.0], 2) == 1.0           # 2 vs 1
    assert seeds.boundary_margin([2.0, 5.0, 2.0, 0.0], 2) == 0.0      # tie across the boundary
    assert seeds.boundary_margin([5.0, 5.0, 2.0], 1) == 0.0
    assert seeds.boundary_margin([5.0, 5.0, 2.0], 2) == 3.0           # tie inside the set is fine
    assert seeds.boundary_margin([-inf, 4.0, -inf, 1.5], 1) == 2.5    # -inf never contests


@pytest.mark.parametrize("trial", range(20))
def test_boundary_margin_is_the_selection_stability_margin(trial):
    rng = np.random.default_rng(300 + trial)
    L, k = 9, int(rng.integers(1, 8))
    s = rng.normal(0, 1, L)
    s[rng.random(L) < 0.2] = -np.inf
    margin = seeds.boundary_margin(s, k)
    _, chosen = seeds.select(s, k)
    if not np.isfinite(margin):
        return
    for _ in range(50):
        eps = rng.uniform(-1, 1, L) * 0.499 * margin
        _, c2 = seeds.select(np.where(np.isfinite(s), s + eps, s), k)
        assert np.array_equal(c2, chosen)
    # the weakest chosen score down, the strongest unchosen finite one up: the set changes
    fin = np.isfinite(s)
    weakest = min((i for i in range(L) if chosen[i]), key=lambda i: s[i])
    strongest = max((i for i in range(L) if fin[i] and not chosen[i]), key=lambda i: s[i])
    y = s.copy()
    y[weakest] -= 0.501 * margin
    y[strongest] += 0.501 * margin
    _, c3 = seeds.select(y, k)
    assert not np.array_equal(c3, chosen)
