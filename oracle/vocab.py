"""Per-row vocabulary statistics of the verification pass (oracle, fp64).

Test infrastructure only (see the package docstring).

For each verified row (one sequence position) with verifier logits l[V] and
drafter logits m[V]:

  LSE_t = log sum_v e^{l_v},  LSE_d = log sum_v e^{m_v}
  argmax_t, argmax_d        -- lowest index among the maxima
  conf_t  = max_v p_t(v)    -- the verifier's confidence ([DD] section 2,
                               Confidence-based Remasking: the verifier's max probability)
  H_t     = -sum_v p_t log p_t -- entropy of the verifier's distribution; the
                               uncertainty u of [COVER] section 2
  KL_dt   = KL(p_d || p_t) = sum_v p_d (log p_d - log p_t)
                            -- [DD] section 2, KL Divergence-based Remasking
                               (the page says "between drafter and verifier";
                               our reading: drafter relative to verifier)
and, at temperature T > 0, the coupled Gumbel-argmax samples of [SPOT]
section 1 (Coupled-Noise Verification):
  sample_x = argmax_v (x_v / T + g_v) for x in {l, m}, with the same g_v,
  p_t(sample_t) = e^{l_s - LSE_t}.
Statistics use the raw (T = 1) distributions; T only scales the sampling.
At T = 0 the samples are the argmaxes.

Each sum is computed in two passes (maximum first), in fp64.
"""
from __future__ import annotations

import numpy as np

from . import philox


def _lse(x):
    mx = x.max(axis=-1, keepdims=True)
    return mx[..., 0] + np.log(np.exp(x - mx).sum(axis=-1))


def _argmax_lowest(x):
    # np.argmax returns the first (lowest) index among equal maxima.
    return np.argmax(x, axis=-1).astype(np.int64)


def _top2_gap(x):
    """Gap between the largest and the second largest entry of each row
    (infinite when a row has a single entry: there is no runner-up)."""
    if x.shape[-1] < 2:
        return np.full(x.shape[:-1], np.inf)
    part = -np.partition(-x, 1, axis=-1)[..., :2]
    return part[..., 0] - part[..., 1]


def row_stats(l, m):
    """l, m: [n, V] verifier / drafter logits (any float dtype, widened to fp64)."""
    l = np.asarray(l, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    lse_t, lse_d = _lse(l), _lse(m)
    logp_t = l - lse_t[:, None]
    logp_d = m - lse_d[:, None]
    p_t, p_d = np.exp(logp_t), np.exp(logp_d)
    argmax_t, argmax_d = _argmax_lowest(l), _argmax_lowest(m)
    conf_t = np.exp(l.max(axis=1) - lse_t)
    entropy_t = -(p_t * logp_t).sum(axis=1)
    kl_dt = (p_d * (logp_d - logp_t)).sum(axis=1)
    return dict(lse_t=lse_t, lse_d=lse_d, argmax_t=argmax_t, argmax_d=argmax_d,
                conf_t=conf_t, entropy_t=entropy_t, kl_dt=kl_dt)


def gumbel_rows(seed, step, b, positions, V):
    """Noise g[n, V] for rows at `positions` of batch entry b."""
    positions = np.asarray(positions)
    return philox.gumbel(seed, step, b, positions[:, None], np.arange(V)[None, :])


def coupled_samples(l, m, temperature, g):
    """sample_t, sample_d = argmax(l/T + g), argmax(m/T + g); their decision margins
    (top-1 minus top-2 score gap) for near-tie accounting."""
    l = np.asarray(l, dtype=np.float64)
    m = np.asarray(m, dtype=np.float64)
    st = l / temperature + g
    sd = m / temperature + g
    return dict(sample_t=_argmax_lowest(st), sample_d=_argmax_lowest(sd),
                margin_t=_top2_gap(st), margin_d=_top2_gap(sd))


def verify_rows(l, m, temperature, seed, step, b, positions):
    """All per-row outputs of the verification pass for rows of batch entry b.

    l, m: [n, V]; positions: the sequence position of each row."""
    out = row_stats(l, m)
    l64 = np.asarray(l, dtype=np.float64)
    n, V = l64.shape
    if temperature > 0:
        g = gumbel_rows(seed, step, b, positions, V)
        s = coupled_samples(l, m, temperature, g)
        out.update(s)
    else:
        out.update(sample_t=out["argmax_t"].copy(), sample_d=out["argmax_d"].copy(),
                   margin_t=np.full(n, np.inf), margin_d=np.full(n, np.inf))
    out["p_sample_t"] = np.exp(l64[np.arange(n), out["sample_t"]] - out["lse_t"])
    return out
