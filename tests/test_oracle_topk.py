"""Pins for the oracle's Gumbel-top-k (dense and sparse)."""

import itertools

import numpy as np
from scipy import stats

import oracle
from oracle.philox import STREAM_TOPK_DENSE, gumbel_from_uniform, stream_words, uniform_from_bits


def _softmax(z):
    e = np.exp(z - z.max())
    return e / e.sum()


def test_plackett_luce_pairs_v6_k2():
    """Ordered pairs (i, j) come up with probability p_i p_j / (1 - p_i)."""
    V, M = 6, 200_000
    z = np.array([1.0, 0.2, -0.5, 0.7, -1.2, 0.0])
    tau = 0.8
    s = z / np.float64(np.float32(tau))
    p = _softmax(s)
    g = gumbel_from_uniform(uniform_from_bits(stream_words(21, 4, STREAM_TOPK_DENSE, np.arange(M), V)))
    sc = s[None, :] + g
    order = np.argsort(-sc, axis=1, kind="stable")[:, :2]
    pairs = order[:, 0] * V + order[:, 1]
    counts = np.bincount(pairs, minlength=V * V)
    expect = np.zeros(V * V)
    for i, j in itertools.permutations(range(V), 2):
        expect[i * V + j] = p[i] * p[j] / (1 - p[i]) * M
    mask = expect > 0
    assert counts[~mask].sum() == 0
    _, pval = stats.chisquare(counts[mask], expect[mask])
    assert pval > 1e-3
    # the oracle function agrees with this ordering on a few rows
    out = oracle.gumbel_topk(np.broadcast_to(z, (8, V)), 2, tau, seed=21, rnd=4)
    assert np.array_equal(out["idx"], order[:8])


def test_dense_outputs_consistent():
    rng = np.random.default_rng(0)
    z = rng.standard_normal((5, 100)).astype(np.float32) * 3
    out = oracle.gumbel_topk(z, 8, 0.6, seed=1, rnd=0)
    for r in range(5):
        assert len(set(out["idx"][r])) == 8
        assert np.all(np.diff(out["score"][r]) <= 0)
        s = z[r].astype(np.float64) / np.float64(np.float32(0.6))
        lse = np.log(np.exp(s - s.max()).sum()) + s.max()
        assert np.allclose(out["logp"][r], s[out["idx"][r]] - lse, atol=1e-12)
    # k = V returns a permutation
    out = oracle.gumbel_topk(z[:, :10], 10, 1.0, 0, 0)
    assert all(sorted(r) == list(range(10)) for r in out["idx"].tolist())


def test_masked_entries_never_selected():
    z = np.full((1, 12), -np.inf)
    z[0, [2, 7]] = [0.5, 0.1]
    out = oracle.gumbel_topk(z, 4, 1.0, 3, 0)
    assert sorted(out["idx"][0, :2].tolist()) == [2, 7]
    assert out["idx"][0, 2:].tolist() == [-1, -1]


def test_sparse_rows():
    rng = np.random.default_rng(1)
    rows, L = 200, 10
    idx = np.stack([rng.choice(100000, L, replace=False) for _ in range(rows)])
    prob = rng.dirichlet(np.full(L, 0.3), size=rows)
    prob[:, -2:] = 0.0                          # two unstored / zero entries per row
    out = oracle.gumbel_topk_sparse(idx, prob, 8, 1.0, seed=2, rnd=0)
    for r in range(rows):
        got = out["idx"][r]
        assert set(got.tolist()) == set(idx[r, :8].tolist())   # the 8 positive entries
    out = oracle.gumbel_topk_sparse(idx, prob, 3, 0.5, seed=2, rnd=0)
    assert np.all(np.isin(out["idx"], idx[:, :8]) | (out["idx"] == -1))


def test_sparse_first_pick_law():
    """k = 1 over stored probabilities at tau = 1 samples prob itself."""
    L, M = 5, 100_000
    prob = np.array([0.5, 0.2, 0.15, 0.1, 0.05])
    idx = np.arange(L) + 1000
    out = oracle.gumbel_topk_sparse(np.broadcast_to(idx, (M, L)), np.broadcast_to(prob, (M, L)), 1, 1.0, 5, 0)
    counts = np.bincount(out["idx"][:, 0] - 1000, minlength=L)
    _, pval = stats.chisquare(counts, prob * M)
    assert pval > 1e-3


def test_plackett_luce_pairs_across_blocks_v600_k2():
    """Five blocks of the top-down draw: ordered first-two picks over six heavy
    tokens in different blocks and the pooled rest follow Plackett-Luce."""
    V, M = 600, 30000
    z = np.full(V, -1.0)
    heavy = [5, 140, 260, 262, 390, 599]          # blocks 0, 1, 2, 2, 3, 4
    z[heavy] = [2.5, 2.0, 1.8, 1.5, 2.2, 1.0]
    tau = 1.0
    s = z / np.float64(np.float32(tau))
    p = _softmax(s)
    out = oracle.gumbel_topk(np.broadcast_to(z, (M, V)), 2, tau, seed=8, rnd=3)
    cat = np.full(V, len(heavy))
    cat[heavy] = np.arange(len(heavy))
    C = len(heavy) + 1
    pairs = cat[out["idx"][:, 0]] * C + cat[out["idx"][:, 1]]
    counts = np.bincount(pairs, minlength=C * C).astype(float)
    expect = np.zeros(C * C)
    for u in range(V):
        for w in range(V):
            if u != w:
                expect[cat[u] * C + cat[w]] += p[u] * p[w] / (1 - p[u])
    expect *= M
    mask = expect > 5
    assert counts[~mask].sum() <= 5 * (~mask).sum() + 20
    _, pval = stats.chisquare(counts[mask], expect[mask] * counts[mask].sum() / expect[mask].sum())
    assert pval > 1e-3, pval


def test_conditioned_scores_keep_order_and_hit_the_block_maximum():
    from oracle.topk import _conditioned_scores
    rng = np.random.default_rng(4)
    h = rng.gumbel(size=128) + rng.standard_normal(128)
    h[[3, 50]] = -np.inf
    S = _conditioned_scores(h, 7.25)
    z = int(np.argmax(h))
    assert S[z] == 7.25 and np.all(S[np.arange(128) != z] < 7.25)
    live = np.isfinite(h)
    assert np.array_equal(np.argsort(-h[live], kind="stable"), np.argsort(-S[live], kind="stable"))
    assert np.all(S[[3, 50]] == -np.inf)
    # -log(e^{-M} - e^{-Z} + e^{-h}) written directly, where it is well conditioned
    Zm = h.max()
    direct = -np.log(np.exp(-7.25) - np.exp(-Zm) + np.exp(-h[live]))
    assert np.allclose(S[live], direct, rtol=1e-10, atol=1e-10)
