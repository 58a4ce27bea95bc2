"""Helpers for the GPU-vs-oracle parity tests.

Tolerances (the spec bar, written out here):
  attention output: max abs error <= 2e-2 (bf16 inputs), <= 1e-4 (fp32 inputs)
  LSE, entropy, KL: <= 1e-3 relative (plus an absolute floor of 1e-5 nats so
      that rows whose value is ~0 are meaningful)
  conf, p(sample): <= 1e-3 relative (our reading; the bar names no tolerance)
  d_in, d_out:      <= 1e-3 absolute + 1e-3 relative (our reading)
  argmax, samples, seed sets, decisions: bit-exact, except positions whose
      oracle statistic lies within 1e-4 of a threshold or a tie; those are
      counted and reported.
"""
from __future__ import annotations

import numpy as np
import torch

from oracle import attention as OA
from oracle import decide as OD
from oracle import seeds as OS
from oracle import vocab as OV

TIE_EPS = 1e-4
STAT_RTOL, STAT_ATOL = 1e-3, 1e-5
MASS_RTOL, MASS_ATOL = 1e-3, 1e-3


def np64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def npi(t):
    return t.detach().cpu().numpy().astype(np.int64)


def assert_close(name, got, want, rtol, atol):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    err = np.abs(got - want)
    bound = atol + rtol * np.abs(want)
    bad = ~(err <= bound)
    if bad.any():
        i = np.unravel_index(np.argmax(np.where(bad, err - bound, -np.inf)), err.shape)
        raise AssertionError(f"{name}: {int(bad.sum())} of {err.size} outside tolerance; "
                             f"worst at {i}: got {got[i]!r} want {want[i]!r}")
    return float(err.max()) if err.size else 0.0


# ----------------------------------------------------------------------------- verify
def oracle_verify(lt, lm, rows, R, pos_offset, temperature, seed, step):
    """Oracle statistics for the flattened rows `rows` (= b * R + r) of [B, R, V] logits."""
    lt2 = lt.reshape(-1, lt.shape[-1])
    lm2 = lm.reshape(-1, lm.shape[-1])
    idx = torch.as_tensor(rows, device=lt.device)
    l = np64(lt2.index_select(0, idx))
    m = np64(lm2.index_select(0, idx))
    out = {}
    for b in sorted(set(int(x) // R for x in rows)):
        sel = np.array([k for k, x in enumerate(rows) if int(x) // R == b])
        pos = np.array([pos_offset + int(rows[k]) % R for k in sel])
        o = OV.verify_rows(l[sel], m[sel], temperature, seed, step, b, pos)
        for key, val in o.items():
            out.setdefault(key, np.zeros(len(rows), dtype=val.dtype))[sel] = val
    return out


def compare_verify(stats, want, rows, temperature):
    """Compare dd_verify_logits outputs (RowStats of [B, R]) at flattened rows with the oracle.
    Returns the number of near-tie rows excluded from the sample comparison."""
    idx = torch.as_tensor(rows, device=stats.lse_t.device)

    def g(t):
        return t.reshape(-1).index_select(0, idx)

    assert_close("lse_t", np64(g(stats.lse_t)), want["lse_t"], STAT_RTOL, STAT_ATOL)
    assert_close("lse_d", np64(g(stats.lse_d)), want["lse_d"], STAT_RTOL, STAT_ATOL)
    assert_close("entropy_t", np64(g(stats.entropy_t)), want["entropy_t"], STAT_RTOL, STAT_ATOL)
    assert_close("kl_dt", np64(g(stats.kl_dt)), want["kl_dt"], STAT_RTOL, STAT_ATOL)
    assert_close("conf_t", np64(g(stats.conf_t)), want["conf_t"], STAT_RTOL, 1e-7)
    assert np.array_equal(npi(g(stats.argmax_t)), want["argmax_t"]), "argmax_t"
    assert np.array_equal(npi(g(stats.argmax_d)), want["argmax_d"]), "argmax_d"
    near = (want["margin_t"] < TIE_EPS) | (want["margin_d"] < TIE_EPS)
    st, sd = npi(g(stats.sample_t)), npi(g(stats.sample_d))
    ok = ~near
    assert np.array_equal(st[ok], want["sample_t"][ok]), "sample_t"
    assert np.array_equal(sd[ok], want["sample_d"][ok]), "sample_d"
    # p(sample) where the sample agrees
    agree = st == want["sample_t"]
    assert_close("p_sample_t", np64(g(stats.p_sample_t))[agree], want["p_sample_t"][agree],
                 STAT_RTOL, 1e-7)
    return int(near.sum())


# ----------------------------------------------------------------------------- attention
def oracle_attention_seq(x, b, heads=None, rows=None):
    """Oracle out/lse (for `rows`, `heads`) and d_in, d_out (all heads) of sequence b."""
    q, kc, vc = np64(x["q"][b]), np64(x["k_cur"][b]), np64(x["v_cur"][b])
    kp, vp = np64(x["k_prev"][b]), np64(x["v_prev"][b])
    seeds = npi(x["is_seed"][b]) if x.get("is_seed") is not None else np.zeros(q.shape[0])
    masked = npi(x["is_masked"][b]).astype(bool)
    new = npi(x["is_new"][b]).astype(bool)
    Hq = q.shape[1]
    out, lse, A = OA.dualview_attention(q, kc, vc, kp, vp, seeds)
    d_in = OA.d_in(A[:, masked, :], Hq)
    d_out = OA.d_out(A, new, Hq)
    if rows is not None:
        out, lse = out[rows], lse[:, rows]
    if heads is not None:
        out, lse = out[:, heads], lse[heads]
    return out, lse, d_in, d_out


# ----------------------------------------------------------------------------- seeds/decisions
def oracle_select(u_pos, d_in, d_out, eligible, k):
    score = OS.stability_score(u_pos, d_in, d_out, eligible)
    seeds, is_seed = OS.select(score, k)
    return seeds, is_seed, score, OS.boundary_margin(score, k)


def oracle_decide(policy, tokens, is_seed, eligible, stats_rows, pos_offset, R, temperature,
                  tau_kl, tau_conf):
    return OD.decide(policy, tokens, is_seed, eligible, stats_rows, pos_offset, R, temperature,
                     tau_kl, tau_conf, TIE_EPS)
