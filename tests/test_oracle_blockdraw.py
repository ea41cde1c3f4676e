"""Pins of the two-level Gumbel-max draw (the reading of how the SMC-SD bonus
token is sampled from the target distribution)."""

import time

import numpy as np
from scipy import special, stats

from oracle.blockdraw import BLOCK, block_gumbel_argmax, block_log_masses
from oracle.philox import STREAM_BONUS, STREAM_BONUS_BLOCK, gumbel_from_uniform, stream_words, uniform_from_bits


def entry_noise(seed, rnd, row, n):
    return gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_BONUS, row, n)))


def test_one_block_is_plain_gumbel_max():
    rng = np.random.default_rng(0)
    for V in (1, 7, 100, 128):
        for row in range(20):
            a = rng.standard_normal(V) * 2
            v, _ = block_gumbel_argmax(a, 5, 3, STREAM_BONUS_BLOCK, STREAM_BONUS, row)
            assert v == int(np.argmax(a + entry_noise(5, 3, row, V)))


def test_block_log_masses_are_block_logsumexps():
    rng = np.random.default_rng(1)
    a = rng.standard_normal(1000) * 3
    a[256:384] = -np.inf                       # one block fully masked
    lam = block_log_masses(a)
    assert lam.shape == (8,) and lam[2] == -np.inf
    for j in (0, 1, 3, 7):
        assert abs(lam[j] - special.logsumexp(a[j * BLOCK:(j + 1) * BLOCK])) < 1e-12


def test_draw_confined_to_the_only_live_block_uses_global_entry_noise():
    rng = np.random.default_rng(2)
    a = np.full(900, -np.inf)
    a[640:768] = rng.standard_normal(128)      # block 5 only
    for row in range(30):
        v, m = block_gumbel_argmax(a, 9, 1, STREAM_BONUS_BLOCK, STREAM_BONUS, row)
        g = entry_noise(9, 1, row, 768)
        assert v == 640 + int(np.argmax(a[640:768] + g[640:768]))
        assert 640 <= v < 768


def test_draw_frequencies_match_softmax_v1000():
    """20000 draws over 8 blocks (the last one short) against softmax, in 40 bins."""
    V, M = 1000, 20000
    v = np.arange(V)
    a = 1.5 * np.sin(v / 37.0) + 0.8 * np.cos(v / 5.0)
    p = np.exp(a - special.logsumexp(a))
    t0 = time.time()
    draws = np.array([block_gumbel_argmax(a, 21, 4, STREAM_BONUS_BLOCK, STREAM_BONUS, r)[0]
                      for r in range(M)])
    assert time.time() - t0 < 120
    bins = v // 25
    counts = np.bincount(bins[draws], minlength=40)
    expect = np.bincount(bins, weights=p, minlength=40) * M
    chi2, pval = stats.chisquare(counts, expect)
    assert pval > 1e-3, (chi2, pval)
    # and the block masses alone
    cb = np.bincount(draws // BLOCK, minlength=8)
    eb = np.bincount(v // BLOCK, weights=p, minlength=8) * M
    assert stats.chisquare(cb, eb)[1] > 1e-3
