"""Pins for the oracle's draft-step sampler (two-level Gumbel-max over zD / tau)."""

import numpy as np
from scipy import special, stats

import oracle


def test_draw_frequencies_match_softmax_v16():
    """x ~ softmax(z / tau): chi-square of 2e5 draws (rows with distinct noise)."""
    V, M = 16, 200_000
    rng = np.random.default_rng(5)
    z = rng.standard_normal(V) * 1.5
    for tau in (1.0, 0.6):
        t = np.float64(np.float32(tau))
        p = np.exp(z / t - special.logsumexp(z / t))
        # M rows of the same logits: the draw of row r uses its own noise (row id r)
        g = oracle.gumbel_from_uniform(oracle.uniform_from_bits(
            oracle.stream_words(9, 2, oracle.STREAM_DRAFT, np.arange(M), V)))
        x = np.argmax(z[None, :] / t + g, axis=1)
        counts = np.bincount(x, minlength=V)
        _, pval = stats.chisquare(counts, p * M)
        assert pval > 1e-3, (tau, pval)
        out = oracle.sd_draft_sample(np.broadcast_to(z, (64, V)), tau, 9, 2)
        assert np.array_equal(out["tokens"], x[:64])


def test_logq_is_the_log_softmax_of_the_draw():
    rng = np.random.default_rng(6)
    z = rng.standard_normal((8, 300)) * 3
    out = oracle.sd_draft_sample(z, 0.7, 1, 1, row0=40)
    t = np.float64(np.float32(0.7))
    ref = z / t - special.logsumexp(z / t, axis=1, keepdims=True)
    assert np.allclose(out["logq"], ref[np.arange(8), out["tokens"]], atol=1e-12)
    # row r draws with row id row0 + r: the same rows started one later agree
    assert np.array_equal(out["tokens"][1:], oracle.sd_draft_sample(z[1:], 0.7, 1, 1, row0=41)["tokens"])


def test_masked_entries_never_drawn_and_bad_rows():
    z = np.full((3, 10), -np.inf)
    z[0, [2, 7]] = [0.0, 0.5]
    z[1, 4] = np.nan
    out = oracle.sd_draft_sample(z, 1.0, 3, 0)
    assert out["tokens"][0] in (2, 7)
    assert out["tokens"][1] == -1 and out["tokens"][2] == -1
    assert out["err"] == oracle.DEV_NONFINITE
    # over many rows only the two finite entries ever come up, in ratio e^0 : e^0.5
    zz = np.broadcast_to(z[0], (20000, 10))
    x = oracle.sd_draft_sample(zz, 1.0, 3, 0)["tokens"]
    assert set(np.unique(x)) == {2, 7}
    frac7 = np.mean(x == 7)
    p7 = np.exp(0.5) / (1 + np.exp(0.5))
    assert abs(frac7 - p7) < 4 * np.sqrt(p7 * (1 - p7) / 20000)


def test_draw_frequencies_match_softmax_v1000_blocks():
    """V = 1000 (8 blocks of the two-level draw): 12000 rows against softmax, 20 bins."""
    V, M = 1000, 12000
    v = np.arange(V)
    z = 2.0 * np.sin(v / 53.0) + np.cos(v / 7.0)
    t = np.float64(np.float32(0.8))
    p = np.exp(z / t - special.logsumexp(z / t))
    x = oracle.sd_draft_sample(np.broadcast_to(z, (M, V)), 0.8, 4, 6)["tokens"]
    bins = v // 50
    counts = np.bincount(bins[x], minlength=20)
    expect = np.bincount(bins, weights=p, minlength=20) * M
    _, pval = stats.chisquare(counts, expect)
    assert pval > 1e-3, pval
