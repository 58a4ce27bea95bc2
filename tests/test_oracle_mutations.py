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
