"""Pins for the oracle's weight normalisation, ESS and systematic resampling."""

import numpy as np

import oracle
from oracle import resample as ors


def test_weights_sum_to_one_and_ess_bounds():
    rng = np.random.default_rng(0)
    logw = rng.standard_normal((40, 32)) * 3
    out = oracle.smcsd_resample(logw, seed=1, rnd=0)
    assert np.allclose(out["W"].sum(axis=1), 1.0, atol=1e-14)
    assert np.all(out["ess"] >= 1.0 - 1e-12) and np.all(out["ess"] <= 32 + 1e-12)


def test_ess_closed_forms():
    out = oracle.smcsd_resample(np.zeros((1, 16)), 0, 0)
    assert out["ess"][0] == 16.0
    one_hot = np.full((1, 8), -np.inf)
    one_hot[0, 5] = 2.0
    out = oracle.smcsd_resample(one_hot, 0, 0)
    assert out["ess"][0] == 1.0
    assert np.all(out["ancestors"][0] == 5)
    # two equal weights among N: ESS = 2
    lw = np.full((1, 6), -np.inf)
    lw[0, [1, 4]] = 0.3
    assert abs(oracle.smcsd_resample(lw, 0, 0)["ess"][0] - 2.0) < 1e-15


def test_systematic_offspring_invariant_and_monotone():
    rng = np.random.default_rng(1)
    for trial in range(200):
        N = int(rng.integers(1, 40))
        logw = rng.standard_normal((1, N)) * rng.uniform(0.1, 5)
        out = oracle.smcsd_resample(logw, seed=trial, rnd=3)
        a = out["ancestors"][0]
        assert np.all(np.diff(a) >= 0)
        counts = np.bincount(a, minlength=N)
        nw = N * out["W"][0]
        assert np.all(counts >= np.floor(nw) - 1e-9) and np.all(counts <= np.ceil(nw) + 1e-9)
        assert counts.sum() == N


def test_brute_force_interval_count_n4():
    """At N = 4, count U_i = (i + u0)/4 falling in each [C_{j-1}, C_j) by enumeration,
    and check that the average offspring count over a u0 grid is N * W_j (unbiasedness)."""
    W = np.array([0.1, 0.45, 0.05, 0.4])
    C = np.cumsum(W)
    grid = (np.arange(4000) + 0.5) / 4000
    mean_counts = np.zeros(4)
    for u0 in grid:
        a, _ = ors.systematic_ancestors(W, u0)
        expect = []
        for i in range(4):
            U = (i + u0) / 4
            lo = 0.0
            for j in range(4):
                if lo <= U < C[j]:
                    expect.append(j)
                    break
                lo = C[j]
            else:
                expect.append(3)
        assert list(a) == expect
        mean_counts += np.bincount(a, minlength=4)
    mean_counts /= grid.size
    assert np.allclose(mean_counts, 4 * W, atol=2e-3)


def test_equal_weights_give_identity():
    for u0 in (1e-7, 0.3, 0.999999):
        a, _ = ors.systematic_ancestors(np.full(32, 1 / 32), u0)
        assert np.array_equal(a, np.arange(32))


def test_offset_stream_and_nonfinite():
    u0 = ors.resample_offset(seed=5, rnd=1, b=3)
    assert 0 < u0 < 1
    out = oracle.smcsd_resample(np.array([[0.0, np.nan], [0.0, 1.0]]), 0, 0)
    assert out["err"] & oracle.DEV_NONFINITE
    assert np.all(np.isnan(out["W"][0])) and np.array_equal(out["ancestors"][0], [0, 1])
    assert np.isfinite(out["W"][1]).all()


def test_adaptive_limits():
    """ess_frac = 0: never resampled (identity, weights carried); ess_frac > 1:
    always, and then exactly smcsd_resample with log-weights reset to 0."""
    rng = np.random.default_rng(7)
    lw = rng.standard_normal((5, 16)) * 2
    never = oracle.smcsd_resample_adaptive(lw, 0.0, 3, 1)
    assert (never["resampled"] == 0).all()
    assert np.array_equal(never["ancestors"], np.tile(np.arange(16), (5, 1)))
    assert np.array_equal(never["logw_next"], lw)
    always = oracle.smcsd_resample_adaptive(lw, 2.0, 3, 1)
    ref = oracle.smcsd_resample(lw, 3, 1)
    assert (always["resampled"] == 1).all()
    assert np.array_equal(always["ancestors"], ref["ancestors"])
    assert (always["logw_next"] == 0).all()
    assert np.allclose(always["ess"], ref["ess"], rtol=0, atol=0)


def test_adaptive_threshold_is_exact_at_known_ess():
    """k equal weights and N - k zero weights (-inf) give ESS = k exactly: the
    sequence is resampled iff k < ess_frac * N (strict)."""
    N = 8
    lw = np.full((N, N), -np.inf)
    for k in range(1, N + 1):
        lw[k - 1, :k] = 0.3
    out = oracle.smcsd_resample_adaptive(lw, 0.5, 1, 0)  # threshold ESS < 4
    assert np.allclose(out["ess"], np.arange(1, N + 1), atol=1e-12)
    assert list(out["resampled"]) == [1, 1, 1, 0, 0, 0, 0, 0]
    # resampled sequences never pick a zero-weight particle
    for k in range(1, 4):
        assert out["ancestors"][k - 1].max() < k


def test_reward_weighted_target_closed_form():
    """With identical target and draft rows the draft terms cancel (logw = 0), so
    a log-potential phi makes W = softmax(phi) exactly; phi = -inf drops a particle."""
    rng = np.random.default_rng(8)
    B, N, K, V = 2, 6, 2, 50
    zT = rng.standard_normal((B, N, K + 1, V))
    x = rng.integers(0, V, (B, N, K))
    phi = rng.standard_normal((B, N))
    phi[1, 2] = -np.inf
    o = oracle.smcsd_score(zT, zT.copy(), x, 1.0, 0, 0, log_potential=phi)
    assert np.array_equal(o["logw"], phi)
    r = oracle.smcsd_resample(o["logw"], 0, 0)
    W = np.exp(phi - phi.max(axis=1, keepdims=True))
    W /= W.sum(axis=1, keepdims=True)
    assert np.allclose(r["W"], W, atol=1e-15)
    assert 2 not in r["ancestors"][1]
    # the potential enters like a carried weight
    o2 = oracle.smcsd_score(zT, zT.copy(), x, 1.0, 0, 0, logw_prev=np.where(np.isinf(phi), -np.inf, phi))
    assert np.array_equal(o2["logw"], o["logw"])
