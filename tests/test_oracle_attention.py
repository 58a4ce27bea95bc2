"""Pins for the oracle's dual-view attention and d_in / d_out (CPU only).

Independent checks: torch's scaled_dot_product_attention (fp64, CPU) where the
dual view reduces to plain attention; a brute-force per-query loop that
assembles each query's K/V explicitly; closed forms for uniform attention;
conservation of attention mass; permutation equivariance.
"""
import math

import numpy as np
import pytest
import torch

from oracle import attention


def _inputs(L=12, Hq=2, Hkv=2, d=8, seed=0, drift=0.3):
    rng = np.random.default_rng(seed)
    q = rng.normal(size=(L, Hq, d))
    k = rng.normal(size=(L, Hkv, d))
    v = rng.normal(size=(L, Hkv, d))
    kp = k + drift * rng.normal(size=k.shape)
    vp = v + drift * rng.normal(size=v.shape)
    return q, k, v, kp, vp


def _sdpa(q, k, v, G):
    # torch SDPA over [H, L, d], fp64, no mask, default scale 1/sqrt(d)
    qt = torch.from_numpy(q).permute(1, 0, 2)
    kt = torch.from_numpy(k).permute(1, 0, 2).repeat_interleave(G, 0)
    vt = torch.from_numpy(v).permute(1, 0, 2).repeat_interleave(G, 0)
    o = torch.nn.functional.scaled_dot_product_attention(qt[None], kt[None], vt[None])[0]
    return o.permute(1, 0, 2).numpy()


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2), (6, 1)])
def test_no_seeds_is_plain_attention(Hq, Hkv):
    q, k, v, kp, vp = _inputs(L=17, Hq=Hq, Hkv=Hkv, d=16)
    out, lse, A = attention.dualview_attention(q, k, v, kp, vp, np.zeros(17))
    np.testing.assert_allclose(out, _sdpa(q, k, v, Hq // Hkv), rtol=0, atol=1e-12)
    # lse against the textbook definition
    for h in range(Hq):
        s = (q[:, h] @ k[:, h // (Hq // Hkv)].T) / math.sqrt(16)
        np.testing.assert_allclose(lse[h], np.log(np.exp(s).sum(1)), rtol=1e-13)


def test_cache_equal_to_current_is_plain_attention():
    q, k, v, _, _ = _inputs(L=13)
    seeds = np.zeros(13)
    seeds[[2, 5, 11]] = 1
    out, lse, _ = attention.dualview_attention(q, k, v, k, v, seeds)
    np.testing.assert_allclose(out, _sdpa(q, k, v, 1), atol=1e-12)


def _brute_force(q, k, v, kp, vp, is_seed):
    """Per query: assemble its K/V explicitly, then a textbook softmax loop."""
    L, Hq, d = q.shape
    G = Hq // k.shape[1]
    out = np.zeros_like(q)
    lse = np.zeros((Hq, L))
    A = np.zeros((Hq, L, L))
    for h in range(Hq):
        g = h // G
        for i in range(L):
            Ki = np.array([kp[j, g] if (is_seed[j] and j != i) else k[j, g] for j in range(L)])
            Vi = np.array([vp[j, g] if (is_seed[j] and j != i) else v[j, g] for j in range(L)])
            s = [float(np.dot(q[i, h], Ki[j])) / math.sqrt(d) for j in range(L)]
            z = sum(math.exp(x) for x in s)
            a = [math.exp(x) / z for x in s]
            A[h, i] = a
            lse[h, i] = math.log(z)
            out[i, h] = sum(a[j] * Vi[j] for j in range(L))
    return out, lse, A


@pytest.mark.parametrize("Hq,Hkv", [(2, 2), (4, 2)])
def test_seed_rows_match_brute_force_assembly(Hq, Hkv):
    L = 11
    q, k, v, kp, vp = _inputs(L=L, Hq=Hq, Hkv=Hkv, d=8, seed=3, drift=0.8)
    seeds = np.zeros(L, dtype=np.uint8)
    seeds[[0, 4, 5, 10]] = 1
    out, lse, A = attention.dualview_attention(q, k, v, kp, vp, seeds)
    bo, bl, bA = _brute_force(q, k, v, kp, vp, seeds)
    np.testing.assert_allclose(out, bo, atol=1e-12)
    np.testing.assert_allclose(lse, bl, atol=1e-12)
    np.testing.assert_allclose(A, bA, atol=1e-12)


def test_seed_diagonal_uses_masked_input_not_cache():
    # A seed query's own column must come from k_cur: make the cached self
    # score huge; the seed row must not concentrate on itself.
    L = 6
    q, k, v, kp, vp = _inputs(L=L, Hq=1, Hkv=1, d=4, seed=5)
    kp[2, 0] = 50 * q[2, 0]
    seeds = np.zeros(L)
    seeds[2] = 1
    _, _, A = attention.dualview_attention(q, k, v, kp, vp, seeds)
    assert A[0, 2, 2] < 0.9
    # a non-seed query does read the cached column
    kp[2, 0] = 50 * q[3, 0]
    _, _, A = attention.dualview_attention(q, k, v, kp, vp, seeds)
    assert A[0, 3, 2] > 0.99


def test_rows_sum_to_one_and_row_subset_consistent():
    q, k, v, kp, vp = _inputs(L=15, Hq=3, Hkv=1, d=8)
    seeds = (np.arange(15) % 4 == 1).astype(np.uint8)
    out, lse, A = attention.dualview_attention(q, k, v, kp, vp, seeds)
    np.testing.assert_allclose(A.sum(-1), 1.0, atol=1e-13)
    rows = np.array([1, 2, 9, 13])
    o2, l2, A2 = attention.dualview_attention(q, k, v, kp, vp, seeds, rows=rows, heads=[2, 0])
    np.testing.assert_allclose(o2, out[rows][:, [2, 0]], atol=1e-13)
    np.testing.assert_allclose(A2, A[[2, 0]][:, rows], atol=1e-13)


def test_permutation_equivariance():
    L = 10
    q, k, v, kp, vp = _inputs(L=L, Hq=2, Hkv=1, d=8, seed=7)
    seeds = np.zeros(L)
    seeds[[1, 6]] = 1
    perm = np.random.default_rng(1).permutation(L)
    out, lse, A = attention.dualview_attention(q, k, v, kp, vp, seeds)
    out_p, lse_p, A_p = attention.dualview_attention(q[perm], k[perm], v[perm], kp[perm],
                                                     vp[perm], seeds[perm])
    np.testing.assert_allclose(out_p, out[perm], atol=1e-12)
    np.testing.assert_allclose(lse_p, lse[:, perm], atol=1e-12)
    np.testing.assert_allclose(A_p, A[:, perm][:, :, perm], atol=1e-12)


def test_mass_statistics_conservation_and_bounds():
    L, Hq = 20, 4
    q, k, v, kp, vp = _inputs(L=L, Hq=Hq, Hkv=2, d=8, seed=9)
    rng = np.random.default_rng(2)
    seeds = (rng.random(L) < 0.2).astype(np.uint8)
    masked = (rng.random(L) < 0.4) & (seeds == 0)
    new = (rng.random(L) < 0.3) & ~masked
    out, lse, din, dout = attention.sequence(q, k, v, kp, vp, seeds, masked, new)
    # every masked query distributes mass 1 per head -> sum_j d_in_j = |M|
    np.testing.assert_allclose(din.sum(), masked.sum(), rtol=1e-13)
    assert np.all(dout >= 0) and np.all(dout <= 1 + 1e-13)
    _, _, _, d_all = attention.sequence(q, k, v, kp, vp, seeds, masked, np.ones(L))
    np.testing.assert_allclose(d_all, 1.0, atol=1e-13)
    _, _, d_none_in, d_none = attention.sequence(q, k, v, kp, vp, seeds, np.zeros(L), np.zeros(L))
    assert np.all(d_none == 0) and np.all(d_none_in == 0)


def test_mass_statistics_closed_form_uniform_attention():
    # q = 0 -> every score is 0 -> A_ij = 1/L for all i, j, whatever the seeds.
    L, Hq = 16, 2
    _, k, v, kp, vp = _inputs(L=L, Hq=Hq, Hkv=2, d=8)
    q = np.zeros((L, Hq, 8))
    seeds = np.zeros(L)
    seeds[[3, 8]] = 1
    masked = np.zeros(L, bool)
    masked[[0, 5, 6, 7, 12]] = True
    new = np.zeros(L, bool)
    new[[1, 2, 9]] = True
    _, _, din, dout = attention.sequence(q, k, v, kp, vp, seeds, masked, new)
    np.testing.assert_allclose(din, masked.sum() / L, atol=1e-14)
    np.testing.assert_allclose(dout, new.sum() / L, atol=1e-14)


def test_mass_statistics_match_brute_force():
    L, Hq = 9, 2
    q, k, v, kp, vp = _inputs(L=L, Hq=Hq, Hkv=1, d=4, seed=11, drift=1.0)
    seeds = np.zeros(L, np.uint8)
    seeds[[2, 7]] = 1
    masked = np.zeros(L, bool)
    masked[[0, 4]] = True
    new = np.zeros(L, bool)
    new[[1, 7, 8]] = True
    _, _, din, dout = attention.sequence(q, k, v, kp, vp, seeds, masked, new)
    _, _, bA = _brute_force(q, k, v, kp, vp, seeds)
    bin_ = [sum(bA[h, i, j] for h in range(Hq) for i in range(L) if masked[i]) / Hq
            for j in range(L)]
    bout = [sum(bA[h, i, j] for h in range(Hq) for j in range(L) if new[j]) / Hq
            for i in range(L)]
    np.testing.assert_allclose(din, bin_, atol=1e-13)
    np.testing.assert_allclose(dout, bout, atol=1e-13)
