"""Dual-view attention and the attention-mass statistics d_in, d_out (oracle, fp64).

Test infrastructure only (see the package docstring).

[COVER] Methodology section 1, "Dual-View Feed Forward via KV cache override":
  * verification view: the seed positions' input tokens are replaced by [MASK],
    so the K/V computed at step t for a seed column (k_cur, v_cur) come from the
    masked input;
  * drafting view: every *non-seed* query reads the seed columns from the step
    t-1 cache (k_prev, v_prev), keeping the unmasked context intact;
  * diagonal correction: for a *seed* query, its own column is the one computed
    from the masked input (k_cur, v_cur), and the softmax is taken over the
    corrected scores, so the seed cannot see its cached self.

Our reading where the page is silent: only a seed's own column is swapped back
(other seed columns stay cached for it too); attention is fully bidirectional
with no mask (the DualDiffusion problem statement: every step recomputes full
bidirectional attention); softmax scale 1/sqrt(d); grouped-query heads share
kv head h // (Hq / Hkv).

[COVER] Methodology section 2, "Stability-Aware Seed Selection":
  d_in  -- how much the still-masked positions rely on a token as context:
           d_in_j  = (1/Hq) sum_h sum_{i in masked} A^h_ij
  d_out -- how strongly a token attends to newly written positions:
           d_out_i = (1/Hq) sum_h sum_{j in new} A^h_ij
Our reading: A is the row-normalised dual-view attention of the same pass
(one layer), averaged over heads and summed (not averaged) over rows/columns.
"""
from __future__ import annotations

import numpy as np


def dualview_scores(q_h, k_cur_g, k_prev_g, is_seed, rows, scale):
    """Scores s_ij = scale * q_i . k~_ij for query rows `rows`, all columns j.

    k~_ij = k_prev[j] if (j is a seed and j != i) else k_cur[j].
    Returns (s [len(rows), L], use_prev [len(rows), L] bool)."""
    L = k_cur_g.shape[0]
    rows = np.asarray(rows)
    cols = np.arange(L)
    use_prev = is_seed[None, :].astype(bool) & (rows[:, None] != cols[None, :])
    s_cur = scale * (q_h[rows] @ k_cur_g.T)
    s_prev = scale * (q_h[rows] @ k_prev_g.T)
    return np.where(use_prev, s_prev, s_cur), use_prev


def dualview_attention(q, k_cur, v_cur, k_prev, v_prev, is_seed, scale=None, rows=None,
                       heads=None):
    """One sequence of dual-view attention.

    q [L, Hq, d]; k_cur, v_cur, k_prev, v_prev [L, Hkv, d]; is_seed [L] (bool/0-1).
    rows: query rows to compute (default all); heads: query heads (default all).
    Returns out [len(rows), len(heads), d], lse [len(heads), len(rows)],
    A [len(heads), len(rows), L] (the row-normalised dual-view attention)."""
    q, k_cur, v_cur, k_prev, v_prev = (np.asarray(x, dtype=np.float64)
                                       for x in (q, k_cur, v_cur, k_prev, v_prev))
    L, Hq, d = q.shape
    Hkv = k_cur.shape[1]
    G = Hq // Hkv
    if scale is None:
        scale = 1.0 / np.sqrt(d)
    is_seed = np.asarray(is_seed).astype(bool)
    rows = np.arange(L) if rows is None else np.asarray(rows)
    heads = np.arange(Hq) if heads is None else np.asarray(heads)
    out = np.zeros((len(rows), len(heads), d))
    lse = np.zeros((len(heads), len(rows)))
    A = np.zeros((len(heads), len(rows), L))
    for hi, h in enumerate(heads):
        g = h // G
        s, use_prev = dualview_scores(q[:, h], k_cur[:, g], k_prev[:, g], is_seed, rows, scale)
        m = s.max(axis=1, keepdims=True)
        e = np.exp(s - m)
        z = e.sum(axis=1, keepdims=True)
        a = e / z
        A[hi] = a
        lse[hi] = m[:, 0] + np.log(z[:, 0])
        # O_i = sum_j A_ij v~_ij, with v~ taken from the same source as k~.
        out[:, hi] = (a * use_prev) @ v_prev[:, g] + (a * ~use_prev) @ v_cur[:, g]
    return out, lse, A


def d_in(A_masked_rows, Hq):
    """d_in_j = (1/Hq) sum_h sum_{i in masked} A^h_ij.
    A_masked_rows: [Hq, |masked|, L], the attention rows of the masked queries."""
    return A_masked_rows.sum(axis=(0, 1)) / Hq


def d_out(A_rows, is_new, Hq):
    """d_out_i = (1/Hq) sum_h sum_{j in new} A^h_ij for the rows in A_rows [Hq, R, L]."""
    new = np.asarray(is_new).astype(bool)
    return A_rows[:, :, new].sum(axis=(0, 2)) / Hq


def sequence(q, k_cur, v_cur, k_prev, v_prev, is_seed, is_masked, is_new, scale=None):
    """Everything the attention step returns for one sequence: out, lse, d_in, d_out."""
    Hq = np.asarray(q).shape[1]
    out, lse, A = dualview_attention(q, k_cur, v_cur, k_prev, v_prev, is_seed, scale)
    masked = np.asarray(is_masked).astype(bool)
    return out, lse, d_in(A[:, masked, :], Hq), d_out(A, is_new, Hq)


def layer_stack(layers, is_seed, is_masked, is_new, q_begin=0, scale=None):
    """A verification pass over several attention layers with a prefix cache.

    [COVER] Results: COVER composes with Fast-dLLM-style prefix caching. Our
    reading: the K/V rows of the prefix (positions < q_begin, the prompt) come
    from a cache that was filled once -- they are the given k/v rows, not
    recomputed -- and the queries of the prefix are not computed at all: only
    rows >= q_begin produce out and lse. Every layer applies the dual view of
    [COVER] section 1 with the same seed set. The seed score's statistics of
    section 2 are averaged over layers: d_in and d_out are the means of the
    per-layer values (each averaged over heads as in `sequence`); d_out of a
    prefix row is 0 (its query row is never computed). Seeds and masked
    positions lie at or after q_begin.

    layers: list of dicts with q [L,Hq,d], k_cur, v_cur, k_prev, v_prev [L,Hkv,d].
    Returns outs (per layer [L - q_begin, Hq, d]), lses (per layer
    [Hq, L - q_begin]), d_in [L], d_out [L]."""
    outs, lses, dins, douts = [], [], [], []
    masked = np.asarray(is_masked).astype(bool)
    L = np.asarray(is_masked).shape[0]
    rows = np.arange(q_begin, L)
    for x in layers:
        Hq = np.asarray(x["q"]).shape[1]
        out, lse, A = dualview_attention(x["q"], x["k_cur"], x["v_cur"], x["k_prev"],
                                         x["v_prev"], is_seed, scale=scale, rows=rows)
        # A is [Hq, L - q_begin, L]: masked rows are all >= q_begin
        dins.append(d_in(A[:, masked[rows], :], Hq))
        dout = np.zeros(L)
        dout[rows] = d_out(A, is_new, Hq)
        douts.append(dout)
        outs.append(out)
        lses.append(lse)
    return outs, lses, np.mean(dins, axis=0), np.mean(douts, axis=0)
