"""dd_select_seeds and dd_decide against the oracle (GPU)."""
import numpy as np
import pytest
import torch

from speculative_verification_cover_b200 import dd
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
    ties = 0
    for b in range(B):
        u = np.zeros(L)
        u[off:off + R] = entropy[b]
        el = elig[b].astype(bool).copy()
        el[:off] = False
        el[off + R:] = False
        # the GPU computes the score in fp32: feed the oracle the same fp32 inputs
        u32 = np.float32(u).astype(np.float64)
        want_seeds, want_is, want_score, margin = PA.oracle_select(
            u32, np.float32(d_in[b]).astype(np.float64), np.float32(d_out[b]).astype(np.float64),
            el, k)
        PA.assert_close("score", np.where(el, PA.np64(score[b]), 0), np.where(el, want_score, 0),
                        1e-6, 1e-6)
        if margin < PA.TIE_EPS:
            ties += 1
            continue
        # the chosen set is unique away from a tie at the k-th place
        assert np.array_equal(PA.npi(is_seed[b]), want_is), b
        got = PA.npi(seeds[b])
        assert sorted(got[got >= 0]) == sorted(want_seeds[want_seeds >= 0]), b
        assert np.array_equal(got < 0, want_seeds < 0), b
        # rank order: descending score, ties (within fp32 rounding) to the lower position
        chosen = got[got >= 0]
        for r in range(len(chosen) - 1):
            sa, sb = want_score[chosen[r]], want_score[chosen[r + 1]]
            assert sa > sb - PA.TIE_EPS, (b, r)
            if abs(sa - sb) >= PA.TIE_EPS:
                assert sa > sb
            elif sa == sb:
                assert chosen[r] < chosen[r + 1]
    assert ties <= B


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
        wd, wt, wa, near = PA.oracle_decide(policy, tokens[b], is_seed[b], elig[b], rows, off, R,
                                            T, 0.5, 0.6)
        ok = ~near
        assert np.array_equal(PA.npi(dec[b])[ok], wd[ok].astype(np.int64)), (policy, b)
        assert np.array_equal(PA.npi(newt[b])[ok], wt[ok].astype(np.int64)), (policy, b)
        if not near.any():
            assert int(acc[b]) == wa
