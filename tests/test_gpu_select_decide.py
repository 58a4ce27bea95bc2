"""dd_select_seeds and dd_decide against the oracle (GPU)."""
import numpy as np
import pytest
import torch

from speculative_verification_cover_b200 import dd
from oracle import decide as OD
from oracle import seeds as OS
from tests import parity as PA

pytestmark = pytest.mark.gpu


def _select(entropy, d_in, d_out, eligible, k, pos_offset):
    B, L = d_in.shape
    seeds = torch.full((B, k), -5, dtype=torch.int32, device="cuda")
    is_seed = torch.full((B, L), 9, dtype=torch.uint8, device="cuda")
    score = torch.empty(B, L, device="cuda")
    dd.dd_select_seeds(entropy, pos_offset, d_in, d_out, eligible, seeds, is_seed, score)
    torch.cuda.synchronize()
    return seeds, is_seed, score


@pytest.mark.parametrize("B,L,R,off,k,quant", [
    (1, 64, 48, 16, 6, 0),
    (4, 512, 384, 128, 16, 0),
    (3, 2048, 1536, 512, 64, 0),
    (2, 300, 300, 0, 40, 4),      # heavy ties: quantised inputs
    (2, 100, 60, 40, 100, 0),     # k larger than the eligible set
    (1, 1, 1, 0, 1, 0),
    (2, 50, 50, 0, 0, 0),         # k = 0
    (1, 5000, 5000, 0, 1024, 3),
])
def test_select_matches_oracle(B, L, R, off, k, quant):
    rng = np.random.default_rng(L + k)
    entropy = rng.random((B, R)) * 5
    d_in = rng.random((B, L)) * 3
    d_out = rng.random((B, L))
    if quant:
        entropy, d_in, d_out = (np.round(a * quant) / quant for a in (entropy, d_in, d_out))
    elig = (rng.random((B, L)) < 0.6).astype(np.uint8)
    t = lambda a, dt=torch.float32: torch.tensor(a, dtype=dt, device="cuda")
    seeds, is_seed, score = _select(t(entropy), t(d_in), t(d_out), t(elig, torch.uint8), k, off)
    near = 0
    for b in range(B):
        u = np.zeros(L)
        u[off:off + R] = entropy[b]
        el = elig[b].astype(bool).copy()
        el[:off] = False
        el[off + R:] = False
        u32, din32, dout32 = (np.float32(a) for a in (u, d_in[b], d_out[b]))
        # the oracle's fp64 score on the very fp32 inputs the kernel received
        want_seeds, want_is, want_score, margin = PA.oracle_select(
            u32.astype(np.float64), din32.astype(np.float64), dout32.astype(np.float64), el, k)
        got_score = PA.np64(score[b])
        PA.assert_close("score", np.where(el, got_score, 0), np.where(el, want_score, 0),
                        1e-6, 1e-6)
        assert np.all(np.isneginf(got_score[~el])), b
        # The set is an integer decided by floating point: both sides decide it in the
        # kernel's precision. The kernel's fp32 score is u * (1 + d_in) / (1 + d_out)
        # with IEEE rounding at each operation; numpy's float32 arithmetic in the same
        # order gives the same bits, and the oracle's rule (score descending, position
        # ascending) picks the set from them. No sequence is excluded.
        s32 = (u32 * (np.float32(1) + din32)) / (np.float32(1) + dout32)
        assert np.array_equal(got_score[el], s32[el].astype(np.float64)), b
        k_seeds, k_is = OS.select(np.where(el, s32.astype(np.float64), -np.inf), k)
        assert np.array_equal(PA.npi(seeds[b]), k_seeds), b
        assert np.array_equal(PA.npi(is_seed[b]), k_is.astype(np.int64)), b
        # Against the fp64 decision: identical unless the k-th place is a near-tie.
        if margin < PA.TIE_EPS:
            near += 1
        else:
            assert np.array_equal(PA.npi(is_seed[b]), want_is), b
            assert np.array_equal(PA.npi(seeds[b]), want_seeds), b
    # near-ties at the k-th place are counted; random continuous scores have none
    assert near == 0 or quant, near
    assert near <= B


POLICIES = ["trust", "kl", "conf", "cover", "coupled"]


@pytest.mark.parametrize("policy", POLICIES)
@pytest.mark.parametrize("T", [0.0, 0.8])
def test_decide_matches_oracle(policy, T):
    rng = np.random.default_rng(POLICIES.index(policy) * 10 + int(T * 10))
    B, L, R, off, V = 3, 300, 240, 60, 20
    tokens = rng.integers(0, V, (B, L)).astype(np.int32)
    masked = rng.random((B, L)) < 0.3
    tokens[masked] = -1
    elig = (~masked).astype(np.uint8)
    elig[:, :off] = 0
    is_seed = ((rng.random((B, L)) < 0.2) & (elig == 1)).astype(np.uint8)
    stats_np = dict(
        lse_t=rng.random((B, R)), lse_d=rng.random((B, R)), conf_t=rng.random((B, R)),
        p_sample_t=rng.random((B, R)), entropy_t=rng.random((B, R)), kl_dt=rng.random((B, R)),
        argmax_t=rng.integers(0, V, (B, R)), argmax_d=rng.integers(0, V, (B, R)),
        sample_t=rng.integers(0, V, (B, R)), sample_d=rng.integers(0, V, (B, R)))
    # make agreement common
    agree = rng.random((B, R)) < 0.4
    for a, b_ in (("argmax_d", "argmax_t"), ("sample_d", "sample_t")):
        stats_np[a] = np.where(agree, stats_np[b_], stats_np[a])
    gen_tok = tokens[:, off:off + R]
    pred = stats_np["sample_t"] if T > 0 else stats_np["argmax_t"]
    tokens[:, off:off + R] = np.where((rng.random((B, R)) < 0.4) & (gen_tok >= 0), pred, gen_tok)
    stats = dd.RowStats(**{k: torch.tensor(v, dtype=torch.float32 if v.dtype.kind == "f"
                                           else torch.int32, device="cuda")
                           for k, v in stats_np.items()})
    dec = torch.empty(B, L, dtype=torch.uint8, device="cuda")
    newt = torch.empty(B, L, dtype=torch.int32, device="cuda")
    acc = torch.empty(B, dtype=torch.uint8, device="cuda")
    tk = torch.tensor(tokens, device="cuda")
    dd.dd_decide(policy, tk, torch.tensor(is_seed, device="cuda"),
                 torch.tensor(elig, device="cuda"), stats, off, dec, newt, acc,
                 tau_kl=0.5, tau_conf=0.6, temperature=T)
    torch.cuda.synchronize()
    for b in range(B):
        rows = {k: np.float32(v[b]).astype(np.float64) if v.dtype.kind == "f" else v[b]
                for k, v in stats_np.items()}
        rows["margin_t"] = np.full(R, np.inf)
        rows["margin_d"] = np.full(R, np.inf)
        # The kernel compares fp32 statistics with fp32 thresholds; the oracle takes
        # the same decisions on the same values (thresholds rounded to fp32 too), so
        # every position must agree, near-ties included.
        wd, wt, wa, near = PA.oracle_decide(policy, tokens[b], is_seed[b], elig[b], rows, off, R,
                                            T, float(np.float32(0.5)), float(np.float32(0.6)))
        assert np.array_equal(PA.npi(dec[b]), wd.astype(np.int64)), (policy, b)
        assert np.array_equal(PA.npi(newt[b]), wt.astype(np.int64)), (policy, b)
        assert int(acc[b]) == wa, (policy, b)
        assert int(near.sum()) <= 2  # positions within 1e-4 of a threshold: counted


@pytest.mark.parametrize("min_score", [-1.0, 2.0, 6.5, 100.0])
def test_adaptive_seed_set_matches_oracle(min_score):
    rng = np.random.default_rng(int(min_score * 10) + 77)
    B, L, R, off, k = 3, 700, 560, 140, 48
    entropy = rng.random((B, R)) * 5
    d_in = rng.random((B, L)) * 3
    d_out = rng.random((B, L))
    elig = (rng.random((B, L)) < 0.6).astype(np.uint8)
    t = lambda a, dt=torch.float32: torch.tensor(a, dtype=dt, device="cuda")
    seeds = torch.full((B, k), -5, dtype=torch.int32, device="cuda")
    is_seed = torch.full((B, L), 9, dtype=torch.uint8, device="cuda")
    score = torch.empty(B, L, device="cuda")
    count = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    dd.dd_select_seeds_ex(t(entropy), off, t(d_in), t(d_out), t(elig, torch.uint8), seeds,
                          is_seed, score, count, min_score=min_score)
    torch.cuda.synchronize()
    for b in range(B):
        u32 = np.zeros(L, np.float32)
        u32[off:off + R] = np.float32(entropy[b])
        el = elig[b].astype(bool).copy()
        el[:off] = False
        el[off + R:] = False
        s32 = (u32 * (np.float32(1) + np.float32(d_in[b]))) / (np.float32(1) + np.float32(d_out[b]))
        sc = np.where(el, s32.astype(np.float64), -np.inf)
        want, want_is = OS.select(sc, k, float(np.float32(min_score)))
        assert np.array_equal(PA.npi(seeds[b]), want), b
        assert np.array_equal(PA.npi(is_seed[b]), want_is.astype(np.int64)), b
        assert int(count[b]) == int((want >= 0).sum())


def _random_stats(rng, B, R, V):
    st = dict(
        lse_t=rng.random((B, R)), lse_d=rng.random((B, R)), conf_t=rng.random((B, R)),
        p_sample_t=rng.random((B, R)), entropy_t=rng.random((B, R)), kl_dt=rng.random((B, R)),
        argmax_t=rng.integers(0, V, (B, R)), argmax_d=rng.integers(0, V, (B, R)),
        sample_t=rng.integers(0, V, (B, R)), sample_d=rng.integers(0, V, (B, R)))
    return st


def _stats_dev(st):
    return dd.RowStats(**{k: torch.tensor(v, dtype=torch.float32 if v.dtype.kind == "f"
                                          else torch.int32, device="cuda")
                          for k, v in st.items()})


@pytest.mark.parametrize("policy,T,tau_commit,min_commit", [
    ("kl_stochastic", 0.0, 0.0, 0), ("kl_stochastic", 0.8, 0.0, 0),
    ("kl_stochastic", 0.0, 0.7, 1), ("cover", 0.0, 0.8, 0), ("coupled", 0.8, 0.8, 1),
    ("trust", 0.0, 2.0, 1),      # nothing passes: the progress rule commits one per sequence
    ("trust", 0.8, 2.0, 0),      # nothing passes and no progress rule: no commit
])
def test_decide_stochastic_and_commit_match_oracle(policy, T, tau_commit, min_commit):
    rng = np.random.default_rng(hash((policy, T, tau_commit, min_commit)) % 2**32)
    B, L, R, off, V = 4, 300, 240, 60, 20
    tokens = rng.integers(0, V, (B, L)).astype(np.int32)
    masked = rng.random((B, L)) < 0.3
    tokens[masked] = -1
    elig = (~masked).astype(np.uint8)
    elig[:, :off] = 0
    is_seed = ((rng.random((B, L)) < 0.2) & (elig == 1)).astype(np.uint8)
    st = _random_stats(rng, B, R, V)
    st["p_sample_t"][0, :5] = 0.625  # exact ties for the progress rule (binary fraction)
    seed, step = 0x1234ABCD5678, 9
    dec = torch.empty(B, L, dtype=torch.uint8, device="cuda")
    newt = torch.empty(B, L, dtype=torch.int32, device="cuda")
    acc = torch.empty(B, dtype=torch.uint8, device="cuda")
    tau_kl = 0.5
    dd.dd_decide(policy, torch.tensor(tokens, device="cuda"), torch.tensor(is_seed, device="cuda"),
                 torch.tensor(elig, device="cuda"), _stats_dev(st), off, dec, newt, acc,
                 tau_kl=tau_kl, tau_conf=0.6, temperature=T, tau_commit=tau_commit,
                 min_commit=min_commit, seed=seed, step=step)
    torch.cuda.synchronize()
    f32 = lambda v: float(np.float32(v))
    commits = 0
    for b in range(B):
        rows = {k: np.float32(v[b]).astype(np.float64) if v.dtype.kind == "f" else v[b]
                for k, v in st.items()}
        rows["margin_t"] = np.full(R, np.inf)
        rows["margin_d"] = np.full(R, np.inf)
        wd, wt, wa, near = OD.decide(policy, tokens[b], is_seed[b], elig[b], rows, off, R, T,
                                     f32(tau_kl), f32(0.6), PA.TIE_EPS, f32(tau_commit),
                                     min_commit, seed, step, b)
        assert np.array_equal(PA.npi(dec[b]), wd.astype(np.int64)), (policy, b)
        assert np.array_equal(PA.npi(newt[b]), wt.astype(np.int64)), (policy, b)
        assert int(acc[b]) == wa, (policy, b)
        commits += int((wd == OD.COMMIT).sum())
    if tau_commit == 2.0:
        assert commits == (B if min_commit else 0)
