"""Pins for the oracle's SMC-SD scoring: lse, gathered log-probs, log-weights, TV, bonus."""

import numpy as np
import pytest
from scipy import special, stats

import oracle
from oracle import score as osc


def _rows(rng, shape, scale=2.0):
    return (rng.standard_normal(shape) * scale).astype(np.float32)


def test_lse_closed_forms():
    # constant logits c over V entries: lse = c / tau + log V
    z = np.full((1, 7), 3.0)
    _, lse = osc.row_log_softmax(z, 2.0)
    assert abs(lse[0] - (1.5 + np.log(7))) < 1e-14
    # logits (0, log 3): lse = log 4
    _, lse = osc.row_log_softmax(np.array([[0.0, np.log(3.0)]]), 1.0)
    assert abs(lse[0] - np.log(4.0)) < 1e-14
    # masked entries (-inf) drop out
    _, lse = osc.row_log_softmax(np.array([[0.0, -np.inf, 0.0]]), 1.0)
    assert abs(lse[0] - np.log(2.0)) < 1e-14


def test_lse_matches_library_logsumexp():
    rng = np.random.default_rng(0)
    z = _rows(rng, (16, 1000), 5.0)
    for tau in (1.0, 0.7, 1.6):
        _, lse = osc.row_log_softmax(z, tau)
        ref = special.logsumexp(z.astype(np.float64) / np.float64(np.float32(tau)), axis=-1)
        assert np.allclose(lse, ref, rtol=0, atol=1e-12)


def test_logweight_hand_example():
    # K = 2, V = 3; probabilities written down directly, logits = their logs
    pT = np.array([[0.5, 0.25, 0.25], [0.2, 0.3, 0.5], [0.1, 0.1, 0.8]])
    qD = np.array([[0.25, 0.5, 0.25], [0.6, 0.2, 0.2], [0.3, 0.3, 0.4]])
    x = np.array([1, 2])
    zT = np.log(pT)[None, None]
    zD = np.log(qD)[None, None]
    out = oracle.smcsd_score(zT, zD, x[None, None], 1.0, seed=1, rnd=0)
    expect = np.log(0.25 / 0.5) + np.log(0.5 / 0.2)
    assert abs(out["logw"][0, 0] - expect) < 1e-13
    assert np.allclose(out["lp"][0, 0, :, 0], np.log([0.25, 0.5]), atol=1e-13)
    assert np.allclose(out["lp"][0, 0, :, 1], np.log([0.5, 0.2]), atol=1e-13)
    tv_expect = 0.5 * np.abs(pT - qD).sum(axis=1)
    assert np.allclose(out["tv"][0, 0], tv_expect, atol=1e-13)
    # a carried log-weight is added
    prev = np.array([[0.75]])
    out2 = oracle.smcsd_score(zT, zD, x[None, None], 1.0, seed=1, rnd=0, logw_prev=prev)
    assert abs(out2["logw"][0, 0] - (expect + 0.75)) < 1e-13
    assert list(out["tokens"][0, 0, :2]) == [1, 2]
    assert out["tokens"][0, 0, 2] == out["bonus"][0, 0]


def test_temperature_divides_both():
    # two-entry rows: p_1 = 1 / (1 + exp((z0 - z1) / tau))
    zT = np.array([[[[0.0, 1.0], [0.0, 0.0]]]])
    zD = np.array([[[[0.0, 3.0], [0.0, 0.0]]]])
    tau = 2.0
    out = oracle.smcsd_score(zT, zD, np.array([[[1]]]), tau, 0, 0)
    lp = np.log(1 / (1 + np.exp(-1.0 / tau)))
    lq = np.log(1 / (1 + np.exp(-3.0 / tau)))
    assert abs(out["logw"][0, 0] - (lp - lq)) < 1e-14


def test_identical_target_and_draft():
    rng = np.random.default_rng(1)
    z = _rows(rng, (2, 4, 5, 300))
    x = rng.integers(0, 300, size=(2, 4, 4))
    out = oracle.smcsd_score(z, z.copy(), x, 0.8, seed=5, rnd=2)
    assert np.all(out["logw"] == 0.0)
    assert np.all(out["tv"] == 0.0)
    rs = oracle.smcsd_resample(out["logw"], seed=5, rnd=2)
    assert np.allclose(rs["W"], 0.25, atol=0, rtol=1e-15)
    assert np.all(rs["ess"] == 4.0)
    assert np.array_equal(rs["ancestors"], np.tile(np.arange(4), (2, 1)))


def test_tv_range_and_disjoint_support():
    rng = np.random.default_rng(2)
    a = _rows(rng, (50, 64), 3.0).astype(np.float64)
    b = _rows(rng, (50, 64), 3.0).astype(np.float64)
    _, la = osc.row_log_softmax(a, 1.0)
    _, lb = osc.row_log_softmax(b, 1.0)
    tv = osc.total_variation(a, la, b, lb)
    assert np.all(tv >= 0) and np.all(tv <= 1)
    # one-hot on different entries: TV = 1
    A = np.array([[0.0, -np.inf]])
    Bm = np.array([[-np.inf, 0.0]])
    _, la = osc.row_log_softmax(A, 1.0)
    _, lb = osc.row_log_softmax(Bm, 1.0)
    assert osc.total_variation(A, la, Bm, lb)[0] == 1.0


def test_exact_expectation_and_tv_identity_v4():
    # E_{x ~ q}[ p(x) / q(x) ] = 1, and sum_x min(p, q) = 1 - TV
    rng = np.random.default_rng(3)
    for _ in range(20):
        zT = rng.standard_normal((1, 1, 2, 4)) * 2
        zD = rng.standard_normal((1, 1, 2, 4)) * 2
        tot = 0.0
        for x in range(4):
            out = oracle.smcsd_score(zT, zD, np.array([[[x]]]), 0.9, 0, 0)
            q = np.exp(out["lp"][0, 0, 0, 1])
            tot += q * np.exp(out["logw"][0, 0])
        assert abs(tot - 1.0) < 1e-12
        a, la = osc.row_log_softmax(zT[0, 0], 0.9)
        b, lb = osc.row_log_softmax(zD[0, 0], 0.9)
        p = np.exp(a - la[:, None])
        q = np.exp(b - lb[:, None])
        assert np.allclose(np.minimum(p, q).sum(axis=1), 1 - out["tv"][0, 0], atol=1e-14)


def test_bad_tokens_and_nonfinite_rows():
    rng = np.random.default_rng(4)
    zT = _rows(rng, (1, 2, 3, 20))
    zD = _rows(rng, (1, 2, 3, 20))
    x = np.array([[[1, 20], [3, 4]]])
    out = oracle.smcsd_score(zT, zD, x, 1.0, 0, 0)
    assert out["err"] & oracle.DEV_TOKEN_OOB
    assert np.isnan(out["logw"][0, 0]) and np.isfinite(out["logw"][0, 1])
    zT2 = zT.copy()
    zT2[0, 1, 2, 5] = np.nan
    out = oracle.smcsd_score(zT2, zD, np.array([[[1, 2], [3, 4]]]), 1.0, 0, 0)
    assert out["err"] & oracle.DEV_NONFINITE
    assert out["bonus"][0, 1] == -1 and out["bonus"][0, 0] >= 0
    assert np.isnan(out["tv"][0, 1, 2])


def test_bonus_is_gumbel_max_of_target_row():
    rng = np.random.default_rng(5)
    zT = _rows(rng, (1, 3, 2, 50))
    out = oracle.smcsd_score(zT, zT, np.zeros((1, 3, 1), dtype=int), 0.5, seed=77, rnd=9)
    for n in range(3):
        g = osc.bonus_noise(77, 9, n, 50)
        assert out["bonus"][0, n] == int(np.argmax(zT[0, n, 1].astype(np.float64) / 0.5 + g))


@pytest.mark.parametrize("tau", [1.0, 0.6])
def test_gumbel_max_chi_square_v16(tau):
    """Bonus-token law equals softmax(z / tau): chi-square at V = 16."""
    V, M = 16, 200_000
    z = np.linspace(-2.0, 2.0, V)
    a = z / np.float64(np.float32(tau))
    p = np.exp(a - special.logsumexp(a))
    from oracle.philox import STREAM_BONUS, gumbel_from_uniform, stream_words, uniform_from_bits
    g = gumbel_from_uniform(uniform_from_bits(stream_words(11, 0, STREAM_BONUS, np.arange(M), V)))
    idx = np.argmax(a[None, :] + g, axis=1)
    counts = np.bincount(idx, minlength=V)
    chi2, pval = stats.chisquare(counts, p * M)
    assert pval > 1e-3, (chi2, pval)
