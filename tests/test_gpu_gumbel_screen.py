"""The noise screen of the sampling vocabulary pass, checked on the device over
every noise value (GPU).

dd_verify_logits skips the exact Gumbel noise g = -ln(-ln U) of entries that
cannot be sampled ([SPOT] section 1, Coupled-Noise Verification): from the best
exact score a warp holds it derives the noise level G an entry would need, and a
group of entries is evaluated only if one of its generator words could have
g > G. This is exact only if the screen never drops a word whose fp32 noise
exceeds G. The noise depends on a word only through its top 23 bits, so all
2^23 levels are enumerated here, with the library's own fp32 noise values.
"""
import numpy as np
import pytest
import torch

from speculative_verification_cover_b200 import dd

pytestmark = pytest.mark.gpu

N_LEVELS = 1 << 23


def test_screen_never_drops_a_word_that_could_win():
    # required noise levels: dense over the range the noise takes, plus extremes
    g_req = np.concatenate([
        np.linspace(-4.0, 17.0, 60001),
        np.linspace(15.0, 16.7, 20001),          # the sparse tail near U -> 1
        [-np.inf, -1e30, -50.0, 0.0, 16.6355, 16.64, 16.65, 20.0, 1e30],
    ]).astype(np.float32)
    g, j, limit, gmax = dd.dd_selftest_gumbel_screen(torch.tensor(g_req, device="cuda"))
    torch.cuda.synchronize()
    g, j, limit = g.cpu().numpy(), j.cpu().numpy(), limit.cpu().numpy()
    k = np.arange(N_LEVELS)
    # the screen's j is exact: 2^23 - 1 - k
    assert np.array_equal(j.astype(np.int64), N_LEVELS - 1 - k)
    # noise values: finite, increasing in k up to fp32 noise, within the closed-form range
    assert np.all(np.isfinite(g))
    u = (2.0 * k + 1.0) * 2.0 ** -24
    exact = -np.log(-np.log(u))
    assert np.max(np.abs(g - exact)) < 1e-4
    # the skip-everything constant bounds every noise value
    assert g.max() <= gmax and gmax < 16.7
    # soundness: at level G the screen keeps words with j + 1/2 < limit, i.e. levels
    # k > 2^23 - 1 - jcut where jcut = ceil(limit - 1/2); every dropped level
    # (k <= 2^23 - 1 - jcut) must have g <= G.
    prefix_max = np.maximum.accumulate(g.astype(np.float64))
    lim = limit.astype(np.float64)
    jcut = np.ceil(np.minimum(lim, 2.0 * N_LEVELS) - 0.5)
    kdrop = (N_LEVELS - 1 - jcut).astype(np.int64)  # last dropped level (-1: none)
    has = kdrop >= 0
    worst = np.full(len(g_req), -np.inf)
    worst[has] = prefix_max[np.minimum(kdrop[has], N_LEVELS - 1)]
    bad = worst > g_req.astype(np.float64)
    assert not bad.any(), (g_req[bad][:5], worst[bad][:5], lim[bad][:5])
    # and the screen is useful: at the levels a typical row reaches it drops nearly all
    typical = (g_req >= 9.0) & (g_req <= 14.0)
    kept = np.clip(N_LEVELS - 1 - kdrop[typical], 0, N_LEVELS) / N_LEVELS
    assert kept.max() < 2e-3
