"""Planted mistakes in the oracle must be caught by its pins (CPU only).

Each case patches one oracle function with a plausible bug (a transposed
mask, a dropped diagonal correction, a reversed KL, a wrong Philox word, a
flipped tie rule) and checks that the corresponding pin test fails.
"""
import numpy as np
import pytest

import oracle.attention as att
import oracle.philox as ph
import oracle.seeds as sd
import oracle.vocab as vb
from tests import test_oracle_attention as TA
from tests import test_oracle_philox as TP
from tests import test_oracle_seeds_decide as TS
from tests import test_oracle_vocab as TV


def _fails(fn, *args):
    try:
        fn(*args)
    except AssertionError:
        return True
    return False


def test_transposed_cache_mask_is_caught(monkeypatch):
    orig = att.dualview_scores

    def bad(q_h, k_cur_g, k_prev_g, is_seed, rows, scale):
        s, use_prev = orig(q_h, k_cur_g, k_prev_g, is_seed, rows, scale)
        L = k_cur_g.shape[0]
        rows = np.asarray(rows)
        # bug: select by the query's seed flag instead of the column's
        up = np.asarray(is_seed).astype(bool)[rows][:, None] & (rows[:, None] != np.arange(L))
        s_cur = scale * (q_h[rows] @ k_cur_g.T)
        s_prev = scale * (q_h[rows] @ k_prev_g.T)
        return np.where(up, s_prev, s_cur), up

    monkeypatch.setattr(att, "dualview_scores", bad)
    assert _fails(TA.test_seed_rows_match_brute_force_assembly, 2, 2)


def test_dropped_diagonal_correction_is_caught(monkeypatch):
    def bad(q_h, k_cur_g, k_prev_g, is_seed, rows, scale):
        rows = np.asarray(rows)
        up = np.broadcast_to(np.asarray(is_seed).astype(bool)[None, :],
                             (len(rows), k_cur_g.shape[0]))
        s_cur = scale * (q_h[rows] @ k_cur_g.T)
        s_prev = scale * (q_h[rows] @ k_prev_g.T)
        return np.where(up, s_prev, s_cur), up

    monkeypatch.setattr(att, "dualview_scores", bad)
    assert _fails(TA.test_seed_rows_match_brute_force_assembly, 2, 2)
    assert _fails(TA.test_seed_diagonal_uses_masked_input_not_cache)


def test_d_in_over_wrong_axis_is_caught(monkeypatch):
    # bug: averages over the masked rows instead of summing them
    monkeypatch.setattr(att, "d_in", lambda A, Hq: A.sum(axis=(0, 1)) / Hq / max(A.shape[1], 1))
    assert _fails(TA.test_mass_statistics_match_brute_force)
    assert _fails(TA.test_mass_statistics_conservation_and_bounds)


def test_reversed_kl_is_caught(monkeypatch):
    orig = vb.row_stats

    def bad(l, m):
        out = orig(l, m)
        rev = orig(m, l)
        out["kl_dt"] = rev["kl_dt"]
        return out

    monkeypatch.setattr(vb, "row_stats", bad)
    assert _fails(TV.test_two_token_kl_closed_form)


def test_entropy_sign_is_caught(monkeypatch):
    orig = vb.row_stats

    def bad(l, m):
        out = orig(l, m)
        out["entropy_t"] = -out["entropy_t"]
        return out

    monkeypatch.setattr(vb, "row_stats", bad)
    assert _fails(TV.test_against_scipy)


def test_wrong_philox_word_order_is_caught(monkeypatch):
    orig = ph.philox_generic

    def bad(x, key, width, multipliers, weyl, rounds=10):
        y = orig(x, key, width, multipliers, weyl, rounds)
        return y[1], y[0], y[2], y[3]

    monkeypatch.setattr(ph, "philox_generic", bad)
    assert _fails(TP.test_round_structure_matches_numpy_philox4x64, (5, 7, 9, 11), (123, 456))
    assert _fails(TP.test_philox4x32_matches_curand_host_generator, 1)


def test_wrong_philox_multiplier_is_caught(monkeypatch):
    monkeypatch.setattr(ph, "PHILOX4x32_M", (0xD2511F53, 0xCD9E8D55))
    assert _fails(TP.test_philox4x32_matches_curand_host_generator, 1)


def test_gumbel_sign_is_caught(monkeypatch):
    monkeypatch.setattr(ph, "gumbel", lambda *a: np.log(-np.log(ph.uniform_from_word(
        ph.noise_words(*a)))))
    assert _fails(TP.test_gumbel_max_frequencies_match_softmax)


def test_topk_tie_rule_is_caught(monkeypatch):
    def bad(score, k):
        score = np.asarray(score, dtype=np.float64)
        L = score.shape[0]
        order = np.lexsort((-np.arange(L), -score))  # bug: ties to the higher position
        chosen = [int(i) for i in order[:k] if np.isfinite(score[i])]
        seeds = np.full(k, -1, dtype=np.int64)
        seeds[:len(chosen)] = chosen
        is_seed = np.zeros(L, dtype=np.uint8)
        is_seed[chosen] = 1
        return seeds, is_seed

    monkeypatch.setattr(sd, "select", bad)
    assert _fails(TS.test_ties_go_to_lower_position)


def test_score_formula_swap_is_caught(monkeypatch):
    monkeypatch.setattr(sd, "stability_score", lambda u, di, do, el: np.where(
        np.asarray(el).astype(bool), np.asarray(u, float) * (1 + np.asarray(do, float))
        / (1 + np.asarray(di, float)), -np.inf))
    assert _fails(TS.test_stability_score_golden)


# --------------------------------------------------------------------- near-tie margins
from tests import test_oracle_margins as TM  # noqa: E402


def test_top2_gap_to_third_entry_is_caught(monkeypatch):
    def bad(x):  # bug: gap to the third largest entry instead of the runner-up
        if x.shape[-1] < 3:
            return np.full(x.shape[:-1], np.inf)
        part = -np.sort(-x, axis=-1)
        return part[..., 0] - part[..., 2]

    monkeypatch.setattr(vb, "_top2_gap", bad)
    assert _fails(TM.test_top2_gap_special_cases)
    assert _fails(TM.test_top2_gap_matches_pairwise_brute_force, 1)


def test_top2_gap_of_logits_instead_of_scores_is_caught(monkeypatch):
    orig = vb.coupled_samples

    def bad(l, m, temperature, g):  # bug: margins of the raw logits, not of l/T + g
        out = orig(l, m, temperature, g)
        out["margin_t"] = vb._top2_gap(np.asarray(l, dtype=np.float64))
        out["margin_d"] = vb._top2_gap(np.asarray(m, dtype=np.float64))
        return out

    monkeypatch.setattr(vb, "coupled_samples", bad)
    assert _fails(TM.test_coupled_margins_are_gaps_of_the_noisy_scores)


def test_top2_gap_absolute_value_hides_ties_is_caught(monkeypatch):
    # bug: a zero gap (tied leaders) reported as the gap to the next distinct value
    def bad(x):
        out = []
        for r in np.asarray(x).reshape(-1, np.asarray(x).shape[-1]):
            u = np.unique(r)[::-1]
            out.append(u[0] - u[1] if len(u) > 1 else np.inf)
        return np.array(out).reshape(np.asarray(x).shape[:-1])

    monkeypatch.setattr(vb, "_top2_gap", bad)
    assert _fails(TM.test_top2_gap_special_cases)


def test_boundary_margin_off_by_one_is_caught(monkeypatch):
    def bad(score, k):  # bug: compares the (k+1)-th and (k+2)-th scores
        s = np.sort(np.asarray(score, dtype=np.float64)[np.isfinite(score)])[::-1]
        if len(s) <= k + 1 or k == 0:
            return np.inf
        return s[k] - s[k + 1]

    monkeypatch.setattr(sd, "boundary_margin", bad)
    assert _fails(TM.test_boundary_margin_special_cases)
    assert _fails(TM.test_boundary_margin_is_the_selection_stability_margin, 0)


def test_boundary_margin_always_zero_is_caught(monkeypatch):
    # a margin that skipped every sequence would make the GPU seed tests vacuous
    monkeypatch.setattr(sd, "boundary_margin", lambda score, k: 0.0)
    assert _fails(TM.test_boundary_margin_special_cases)
    assert _fails(TM.test_boundary_margin_matches_brute_force, 3)


# --------------------------------------------------------------------- multi-layer stack
from tests import test_oracle_layers as TL  # noqa: E402


def test_layer_sum_instead_of_mean_is_caught(monkeypatch):
    orig = att.layer_stack

    def bad(layers, is_seed, is_masked, is_new, q_begin=0, scale=None):
        outs, lses, din, dout = orig(layers, is_seed, is_masked, is_new, q_begin, scale)
        return outs, lses, din * len(layers), dout * len(layers)  # bug: summed over layers

    monkeypatch.setattr(att, "layer_stack", bad)
    assert _fails(TL.test_identical_layers_average_to_one_layer)
    assert _fails(TL.test_mass_conservation_and_bounds, 2)


def test_prefix_rows_computed_anyway_is_caught(monkeypatch):
    orig = att.layer_stack

    def bad(layers, is_seed, is_masked, is_new, q_begin=0, scale=None):
        # bug: the prefix's query rows are computed and counted in d_out
        outs, lses, din, _ = orig(layers, is_seed, is_masked, is_new, 0, scale)
        _, _, _, dout = orig(layers, is_seed, is_masked, is_new, 0, scale)
        return [o[q_begin:] for o in outs], [x[:, q_begin:] for x in lses], din, dout

    monkeypatch.setattr(att, "layer_stack", bad)
    assert _fails(TL.test_prefix_rows_change_nothing_after_them)


# --------------------------------------------------------------------- adaptive seeds, KL draws, commit
from oracle import decide as dc  # noqa: E402
from tests import test_oracle_decide_ext as TX  # noqa: E402


def test_inverted_kl_probability_is_caught(monkeypatch):
    orig = dc.decide

    def bad(policy, *a, **kw):  # bug: remask iff U * tau >= KL (probability 1 - KL / tau)
        d, nt, acc, near = orig(policy, *a, **kw)
        if policy == "kl_stochastic":
            flip = (d == dc.KEEP) | (d == dc.REMASK)
            d = np.where(flip, np.where(d == dc.KEEP, dc.REMASK, dc.KEEP), d).astype(d.dtype)
        return d, nt, acc, near

    monkeypatch.setattr(dc, "decide", bad)
    assert _fails(TX.test_kl_stochastic_frequency_is_kl_over_tau, 0.1)
    assert _fails(TX.test_kl_stochastic_certain_above_threshold_never_at_zero)


def test_min_score_strict_is_caught(monkeypatch):
    orig = sd.select
    monkeypatch.setattr(sd, "select", lambda score, k, min_score=-np.inf: orig(
        score, k, np.nextafter(min_score, np.inf)))  # bug: > instead of >=
    assert _fails(TX.test_adaptive_seed_set_size_and_reduction)


def test_commit_tie_to_higher_position_is_caught(monkeypatch):
    orig = dc.decide

    def bad(*a, **kw):
        d, nt, acc, near = orig(*a, **kw)
        tok = np.asarray(a[1])
        if kw.get("min_commit") and (d == dc.COMMIT).sum() == 1:
            i = int(np.nonzero(d == dc.COMMIT)[0][0])
            p = np.asarray(a[4]["p_sample_t"])
            same = [j for j in range(len(p)) if j > i and tok[j] == -1 and p[j] == p[i]]
            if same:  # bug: the tie goes to the higher position
                d[i], d[same[0]] = 0, dc.COMMIT
        return d, nt, acc, near

    monkeypatch.setattr(dc, "decide", bad)
    assert _fails(TX.test_commit_progress_rule_and_its_tie)
