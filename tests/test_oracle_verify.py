"""Pins for the oracle's standard SD verify (accept rule, residual, sampler)."""

import itertools

import numpy as np
from scipy import special, stats

import oracle
from oracle import score as osc
from oracle import verify as ov


def _softmax(z):
    e = np.exp(z - z.max())
    return e / e.sum()


def test_exhaustive_enumeration_v4_k2():
    """Integrating the accept rule and the residual analytically over u, the emitted
    token at every reached position follows the target law exactly."""
    rng = np.random.default_rng(0)
    V, K = 4, 2
    for _ in range(50):
        p = [_softmax(rng.standard_normal(V) * 2) for _ in range(K + 1)]
        q = [_softmax(rng.standard_normal(V) * 2) for _ in range(K)]
        law = [np.zeros(V) for _ in range(K + 1)]     # P(position k emits v, k reached)
        reach = np.zeros(K + 1)
        for xs in itertools.product(range(V), repeat=K):
            w = np.prod([q[k][xs[k]] for k in range(K)])
            alive = w
            for k in range(K):
                reach[k] += alive
                acc = ov.accept_probability(p[k], q[k], xs[k])
                law[k][xs[k]] += alive * acc
                res = ov.residual_distribution(p[k], q[k])
                if res is not None:
                    law[k] += alive * (1 - acc) * res
                alive *= acc
            reach[K] += alive
            law[K] += alive * p[K]
        for k in range(K + 1):
            assert np.allclose(law[k] / reach[k], p[k], atol=1e-12, rtol=0)


def test_acceptance_rate_equals_one_minus_tv():
    rng = np.random.default_rng(1)
    for _ in range(20):
        p = _softmax(rng.standard_normal(6))
        q = _softmax(rng.standard_normal(6))
        rate = sum(q[x] * ov.accept_probability(p, q, x) for x in range(6))
        assert abs(rate - (1 - 0.5 * np.abs(p - q).sum())) < 1e-14


def test_identical_rows_accept_everything():
    rng = np.random.default_rng(2)
    B, K, V = 4, 3, 40
    zT = rng.standard_normal((B, K + 1, V)) * 2
    zD = zT[:, :K].copy()
    x = rng.integers(0, V, size=(B, K))
    out = oracle.sd_verify_reject(zT, zD, x, 1.0, seed=3, rnd=0)
    assert np.all(out["accepted_len"] == K)
    assert np.array_equal(out["out_tokens"][:, :K], x)
    assert np.all(out["out_tokens"][:, K] >= 0)
    assert np.all(out["tv"] == 0)


def test_disjoint_support_rejects_first_and_draws_from_target():
    V, K = 5, 2
    zT = np.full((1, K + 1, V), -np.inf)
    zT[0, :, :2] = 0.0                    # p uniform on {0, 1}
    zD = np.full((1, K, V), -np.inf)
    zD[0, :, 3] = 0.0                     # q one-hot on 3
    out = oracle.sd_verify_reject(zT, zD, np.array([[3, 3]]), 1.0, 0, 0)
    assert out["accepted_len"][0] == 0
    assert out["out_tokens"][0, 0] in (0, 1)
    assert list(out["out_tokens"][0, 1:]) == [-1, -1]
    assert np.allclose(out["tv"][0], 1.0)


def test_monte_carlo_first_token_law():
    """Over many sequences with x ~ q, the first emitted token follows p (chi-square),
    and the acceptance frequency at position 0 is 1 - TV (binomial bound)."""
    V, K, B = 6, 1, 20000
    rng = np.random.default_rng(4)
    zt = rng.standard_normal(V) * 1.5
    zd = zt + rng.standard_normal(V)
    p, q = _softmax(zt), _softmax(zd)
    zT = np.broadcast_to(np.stack([zt, zt]), (B, K + 1, V))
    zD = np.broadcast_to(zd[None], (B, K, V))
    x = rng.choice(V, size=(B, K), p=q)
    out = oracle.sd_verify_reject(zT, zD, x, 1.0, seed=9, rnd=1)
    counts = np.bincount(out["out_tokens"][:, 0], minlength=V)
    _, pval = stats.chisquare(counts, p * B)
    assert pval > 1e-3
    rate = (out["accepted_len"] >= 1).mean()
    tv = 0.5 * np.abs(p - q).sum()
    assert abs(rate - (1 - tv)) < 5 * np.sqrt(tv * (1 - tv) / B)
    assert np.allclose(out["tv"][:, 0], tv, atol=1e-12)


def test_bad_token_is_rejected():
    rng = np.random.default_rng(5)
    zT = rng.standard_normal((1, 3, 8))
    zD = rng.standard_normal((1, 2, 8))
    out = oracle.sd_verify_reject(zT, zD, np.array([[9, 1]]), 1.0, 0, 0)
    assert out["err"] & oracle.DEV_TOKEN_OOB
    assert out["accepted_len"][0] == 0 and 0 <= out["out_tokens"][0, 0] < 8
    # residual token uses stream 3 with row id b*(K+1)+k
    a, lse = osc.row_log_softmax(zT[0], 1.0)
    d, lsd = osc.row_log_softmax(zD[0], 1.0)
    r = np.maximum(np.exp(a[0] - lse[0]) - np.exp(d[0] - lsd[0]), 0)
    from oracle.philox import STREAM_RESIDUAL, gumbel_from_uniform, stream_words, uniform_from_bits
    g = gumbel_from_uniform(uniform_from_bits(stream_words(0, 0, STREAM_RESIDUAL, 0, 8)))
    with np.errstate(divide="ignore"):
        expect = int(np.argmax(np.where(r > 0, np.log(r), -np.inf) + g))
    assert out["out_tokens"][0, 0] == expect


def test_first_token_law_across_blocks_v700():
    """Drafts x ~ q, target p over V = 700 (six blocks of the two-level residual
    draw): the first emitted token (the accepted draft, or the residual draw
    after a rejection) follows p; chi-square over 14 bins of 6000 sequences."""
    V, B = 700, 6000
    v = np.arange(V)
    zt = 1.5 * np.sin(v / 41.0) + 0.5 * np.cos(v / 3.0)
    zd = 1.5 * np.cos(v / 29.0)
    p = np.exp(zt - special.logsumexp(zt))
    q = np.exp(zd - special.logsumexp(zd))
    rng = np.random.default_rng(17)
    x = rng.choice(V, size=(B, 1), p=q)
    zT = np.broadcast_to(np.stack([zt, zt]), (B, 2, V))
    zD = np.broadcast_to(zd[None, None, :], (B, 1, V))
    out = oracle.sd_verify_reject(zT, zD, x, 1.0, seed=3, rnd=1)
    first = out["out_tokens"][:, 0]
    assert (first >= 0).all()
    bins = v // 50
    counts = np.bincount(bins[first], minlength=14)
    expect = np.bincount(bins, weights=p, minlength=14) * B
    _, pval = stats.chisquare(counts, expect)
    assert pval > 1e-3, pval
