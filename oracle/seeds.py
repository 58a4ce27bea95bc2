"""Stability-aware seed selection (oracle, fp64).

Test infrastructure only (see the package docstring).

[COVER] Methodology section 2, "Stability-Aware Seed Selection": the seed set
is a small set of previously unmasked tokens chosen by the score
    Score = u * (1 + d_in) / (1 + d_out)
with u the entropy of the current token assignment, d_in the influence on the
remaining masked positions and d_out the drift sensitivity (attention to newly
written positions).

Our reading where the page is silent: eligible positions are the unmasked
generated positions (never prompt positions); the k highest scores win, ties
going to the lower position; fewer than k candidates leave the tail -1. The
page calls the set "small and adaptive" without a rule; our reading of the
adaptive size: only positions whose score reaches min_score compete, so the
set holds min(k, #{score >= min_score}) seeds (min_score = -inf: a fixed k).
"""
from __future__ import annotations

import numpy as np


def stability_score(u, d_in, d_out, eligible):
    """score_i = u_i (1 + d_in_i) / (1 + d_out_i) on eligible positions, -inf elsewhere."""
    u, d_in, d_out = (np.asarray(x, dtype=np.float64) for x in (u, d_in, d_out))
    s = u * (1.0 + d_in) / (1.0 + d_out)
    return np.where(np.asarray(eligible).astype(bool), s, -np.inf)


def select(score, k, min_score=-np.inf):
    """Top-k positions by (score descending, position ascending) among those whose
    score reaches min_score. Returns seeds [k] (rank order, -1 padded) and is_seed [L]
    uint8."""
    score = np.asarray(score, dtype=np.float64)
    score = np.where(score >= min_score, score, -np.inf)
    L = score.shape[0]
    order = np.lexsort((np.arange(L), -score))  # primary key: -score; ties: position
    chosen = [int(i) for i in order[:k] if np.isfinite(score[i])]
    seeds = np.full(k, -1, dtype=np.int64)
    seeds[:len(chosen)] = chosen
    is_seed = np.zeros(L, dtype=np.uint8)
    is_seed[chosen] = 1
    return seeds, is_seed


def boundary_margin(score, k, min_score=-np.inf):
    """Gap between the k-th and (k+1)-th finite scores (inf if there is no contest);
    with a min_score, also the distance of any finite score to it."""
    if k == 0:
        return np.inf
    score = np.asarray(score, dtype=np.float64)
    fin = score[np.isfinite(score)]
    to_min = np.abs(fin - min_score).min() if np.isfinite(min_score) and len(fin) else np.inf
    s = np.sort(np.where(fin >= min_score, fin, -np.inf))[::-1]
    s = s[np.isfinite(s)]
    if len(s) <= k:
        return to_min
    return min(s[k - 1] - s[k], to_min)
    if len(s) <= k or k == 0:
        return np.inf
    return s[k - 1] - s[k]
