"""Pins for the oracle's Philox4x32-10 and Gumbel noise (CPU only).

The round structure is pinned against numpy's Philox4x64-10 bit generator
(same construction, 64-bit words); the 32-bit instance the oracle uses is
pinned against cuRAND's host-side Philox4x32-10 generator, called through
its C API. The Gumbel mapping is pinned by the Gumbel-max property: the
argmax of x/T + g is distributed as softmax(x/T).
"""
import ctypes
import ctypes.util
import glob
import os

import numpy as np
import pytest
from scipy import stats

from oracle import philox, vocab


def _generic64(counter, key):
    return philox.philox_generic(tuple(int(c) for c in counter), key, 64,
                                 philox.PHILOX4x64_M, philox.PHILOX4x64_W)


@pytest.mark.parametrize("counter,key", [
    ((0, 0, 0, 0), (0, 0)),
    ((5, 7, 9, 11), (123, 456)),
    ((2**64 - 2, 3, 2**63, 1), (2**64 - 1, 0x0123456789ABCDEF)),
])
def test_round_structure_matches_numpy_philox4x64(counter, key):
    # numpy's Philox increments its 256-bit counter before each block.
    bg = np.random.Philox(counter=np.array(counter, dtype=np.uint64),
                          key=np.array(key, dtype=np.uint64))
    got = [int(x) for x in bg.random_raw(4)]
    c = list(counter)
    c[0] = (c[0] + 1) % 2**64
    if c[0] == 0:
        c[1] = (c[1] + 1) % 2**64
    want = list(_generic64(c, key))
    assert got == want


def _curand_host():
    cands = glob.glob("/usr/local/cuda/lib64/libcurand.so*")
    name = ctypes.util.find_library("curand")
    for path in ([name] if name else []) + cands:
        try:
            return ctypes.CDLL(path)
        except OSError:
            continue
    return None


@pytest.mark.parametrize("seed", [0, 1, 0xDEADBEEF, 0x0123456789ABCDEF])
def test_philox4x32_matches_curand_host_generator(seed):
    lib = _curand_host()
    if lib is None:
        pytest.skip("libcurand not found")
    gen = ctypes.c_void_p()
    CURAND_RNG_PSEUDO_PHILOX4_32_10 = 161
    if lib.curandCreateGeneratorHost(ctypes.byref(gen), CURAND_RNG_PSEUDO_PHILOX4_32_10) != 0:
        pytest.skip("cuRAND host generator unavailable")
    try:
        assert lib.curandSetPseudoRandomGeneratorSeed(gen, ctypes.c_ulonglong(seed)) == 0
        n = 4 * 64
        out = np.zeros(n, dtype=np.uint32)
        assert lib.curandGenerate(gen, out.ctypes.data_as(ctypes.c_void_p), ctypes.c_size_t(n)) == 0
    finally:
        lib.curandDestroyGenerator(gen)
    # The host generator's default ordering emits block c from counter (0, 0, c, 0)
    # with key (seed lo, seed hi).
    c = np.arange(64, dtype=np.uint64)
    z = np.zeros_like(c)
    words = philox.philox4x32_10((z, z, c, z), (seed & 0xFFFFFFFF, seed >> 32))
    mine = np.stack(words, axis=1).reshape(-1)
    assert np.array_equal(mine, out)


def test_uniform_is_open_interval_and_fp32_exact():
    w = np.array([0, 1, 511, 512, 2**31, 2**32 - 1], dtype=np.uint64)
    u = philox.uniform_from_word(w)
    assert np.all(u > 0) and np.all(u < 1)
    assert np.array_equal(u.astype(np.float32).astype(np.float64), u)
    assert u[0] == 2.0**-24 and u[-1] == 1 - 2.0**-24


def test_noise_word_layout():
    # word for v is output word v&3 of counter (v>>2, pos, b, step)
    seed, step, b, pos = 0x1234_5678_9ABC, 7, 3, 100
    v = np.arange(16)
    words = philox.noise_words(seed, step, b, pos, v)
    for vv in range(16):
        blk = philox.philox4x32_10(([vv >> 2], [pos], [b], [step]), (seed & 0xFFFFFFFF, seed >> 32))
        assert words[vv] == blk[vv & 3][0]


def test_gumbel_max_frequencies_match_softmax():
    # Gumbel-max: argmax_v(x_v/T + g_v) ~ softmax(x/T). Many independent rows
    # (distinct positions) of a 5-entry vocabulary.
    x = np.array([1.0, 0.0, -0.5, 2.0, 0.3])
    T = 0.8
    n = 40000
    g = vocab.gumbel_rows(seed=42, step=0, b=0, positions=np.arange(n), V=5)
    s = vocab.coupled_samples(np.tile(x, (n, 1)), np.tile(x, (n, 1)), T, g)
    counts = np.bincount(s["sample_t"], minlength=5)
    p = np.exp(x / T) / np.exp(x / T).sum()
    chi2 = stats.chisquare(counts, n * p)
    assert chi2.pvalue > 1e-3
    # identical drafter and verifier logits -> identical coupled samples
    assert np.array_equal(s["sample_t"], s["sample_d"])


def test_gumbel_small_temperature_is_argmax():
    rng = np.random.default_rng(0)
    l = rng.normal(0, 3, size=(50, 300))
    g = vocab.gumbel_rows(seed=1, step=2, b=0, positions=np.arange(50), V=300)
    s = vocab.coupled_samples(l, l, 1e-6, g)
    assert np.array_equal(s["sample_t"], np.argmax(l, axis=1))


def test_gumbel_noise_marginal_is_standard_gumbel():
    g = vocab.gumbel_rows(seed=9, step=1, b=2, positions=np.arange(200), V=500).ravel()
    ks = stats.kstest(g, stats.gumbel_r.cdf)
    assert ks.pvalue > 1e-3
