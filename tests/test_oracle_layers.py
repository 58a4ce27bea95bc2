"""Pins for the oracle's multi-layer pass with a prefix cache (CPU only).

[COVER] Results: COVER composes with Fast-dLLM-style prefix caching; the seed
score's d_in / d_out of section 2 come from the whole verifier pass. The oracle
(attention.layer_stack) computes only the query rows after the cached prefix
and averages the per-layer statistics. Pinned by: a one-layer stack without a
prefix is the single-layer call; identical layers average to that layer;
prefix rows change nothing for the rows after them; mass conservation
(sum_j d_in_j = |masked| per layer, hence on average); the uniform-attention
closed form.
"""
import numpy as np
import pytest

from oracle import attention as OA


def _layer(rng, L, Hq, Hkv, d, drift=0.1, qscale=1.0):
    q = rng.normal(0, 1, (L, Hq, d)) * qscale
    k = rng.normal(0, 1, (L, Hkv, d))
    v = rng.normal(0, 1, (L, Hkv, d))
    return dict(q=q, k_cur=k, v_cur=v, k_prev=k + rng.normal(0, drift, k.shape),
                v_prev=v + rng.normal(0, drift, v.shape))


def _masks(rng, L, P, n_masked=6, n_new=5, n_seed=4):
    gen = rng.permutation(np.arange(P, L))
    masked = np.zeros(L, np.uint8)
    masked[gen[:n_masked]] = 1
    rest = gen[n_masked:]
    new = np.zeros(L, np.uint8)
    new[rest[:n_new]] = 1
    seed = np.zeros(L, np.uint8)
    seed[rng.permutation(rest)[:n_seed]] = 1
    return seed, masked, new


def test_one_layer_without_prefix_is_the_single_call():
    rng = np.random.default_rng(0)
    L, Hq, Hkv, d = 20, 4, 2, 8
    x = _layer(rng, L, Hq, Hkv, d)
    seed, masked, new = _masks(rng, L, 0)
    outs, lses, din, dout = OA.layer_stack([x], seed, masked, new, q_begin=0)
    o1, l1, din1, dout1 = OA.sequence(x["q"], x["k_cur"], x["v_cur"], x["k_prev"], x["v_prev"],
                                      seed, masked, new)
    np.testing.assert_array_equal(outs[0], o1)
    np.testing.assert_array_equal(lses[0], l1)
    np.testing.assert_allclose(din, din1, rtol=1e-15, atol=0)
    np.testing.assert_allclose(dout, dout1, rtol=1e-15, atol=0)


def test_identical_layers_average_to_one_layer():
    rng = np.random.default_rng(1)
    L, P = 24, 8
    x = _layer(rng, L, 4, 4, 8)
    seed, masked, new = _masks(rng, L, P)
    _, _, din3, dout3 = OA.layer_stack([x, x, x], seed, masked, new, q_begin=P)
    _, _, din1, dout1 = OA.layer_stack([x], seed, masked, new, q_begin=P)
    np.testing.assert_allclose(din3, din1, rtol=1e-14, atol=1e-16)
    np.testing.assert_allclose(dout3, dout1, rtol=1e-14, atol=1e-16)


def test_prefix_rows_change_nothing_after_them():
    rng = np.random.default_rng(2)
    L, P, Hq = 30, 11, 3
    x = _layer(rng, L, Hq, 1, 16)
    seed, masked, new = _masks(rng, L, P)
    outs, lses, din, dout = OA.layer_stack([x], seed, masked, new, q_begin=P)
    full_o, full_l, full_din, full_dout = OA.sequence(
        x["q"], x["k_cur"], x["v_cur"], x["k_prev"], x["v_prev"], seed, masked, new)
    np.testing.assert_allclose(outs[0], full_o[P:], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(lses[0], full_l[:, P:], rtol=1e-13, atol=1e-15)
    np.testing.assert_allclose(din, full_din, rtol=1e-13, atol=1e-15)  # masked rows >= P
    np.testing.assert_allclose(dout[P:], full_dout[P:], rtol=1e-13, atol=1e-15)
    assert np.all(dout[:P] == 0.0)


@pytest.mark.parametrize("n_layers", [1, 2, 5])
def test_mass_conservation_and_bounds(n_layers):
    rng = np.random.default_rng(3 + n_layers)
    L, P = 28, 7
    layers = [_layer(rng, L, 4, 2, 8, qscale=0.5 + i) for i in range(n_layers)]
    seed, masked, new = _masks(rng, L, P, n_masked=9)
    _, _, din, dout = OA.layer_stack(layers, seed, masked, new, q_begin=P)
    assert din.sum() == pytest.approx(int(masked.sum()), rel=1e-12)
    assert np.all(dout >= 0) and np.all(dout <= 1 + 1e-12)


def test_uniform_attention_closed_form():
    # zero queries: every row attends uniformly, A_ij = 1/L in every layer and head
    rng = np.random.default_rng(4)
    L, P = 16, 5
    layers = [_layer(rng, L, 2, 2, 4, qscale=0.0) for _ in range(3)]
    seed, masked, new = _masks(rng, L, P)
    _, _, din, dout = OA.layer_stack(layers, seed, masked, new, q_begin=P)
    np.testing.assert_allclose(din, np.full(L, masked.sum() / L), rtol=1e-14)
    want = np.zeros(L)
    want[P:] = new.sum() / L
    np.testing.assert_allclose(dout, want, rtol=1e-14, atol=0)
