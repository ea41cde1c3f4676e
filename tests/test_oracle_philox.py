"""Pins for the oracle's Philox4x32-10 and the uniform / Gumbel maps built on it."""

import os

import numpy as np

from oracle import philox

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "philox4x32_10_kat.txt")


def _kat():
    rows = []
    with open(GOLDEN) as f:
        for line in f:
            line = line.strip()
            if not line or line.startswith("#"):
                continue
            vals = [int(t, 16) for t in line.split()]
            rows.append((vals[:4], vals[4:6], vals[6:10]))
    return rows


def test_known_answer_vectors():
    kat = _kat()
    assert len(kat) == 3
    for ctr, key, expect in kat:
        out = philox.philox4x32_10(*ctr, *key)
        assert [int(o) for o in out] == expect


def test_known_answer_vectors_vectorised():
    kat = _kat()
    ctr = np.array([k[0] for k in kat], dtype=np.uint64).T
    key = np.array([k[1] for k in kat], dtype=np.uint64).T
    out = philox.philox4x32_10(ctr[0], ctr[1], ctr[2], ctr[3], key[0], key[1])
    for j, (_, _, expect) in enumerate(kat):
        assert [int(o[j]) for o in out] == expect


def test_stream_word_layout():
    # position v reads word v % 4 of the call with c0 = v // 4
    w = philox.stream_words(seed=0x1234_5678_9ABC_DEF0, rnd=(7 << 32) + 3, tag=5, c1=11, n=10)
    for v in range(10):
        out = philox.philox4x32_10(v // 4, 11, 3, 5 + 16 * 7, 0x9ABCDEF0, 0x12345678)
        assert int(w[v]) == int(out[v % 4])
    rows = philox.stream_words(seed=9, rnd=1, tag=1, c1=np.array([4, 5]), n=6)
    assert rows.shape == (2, 6)
    assert np.array_equal(rows[1], philox.stream_words(9, 1, 1, 5, 6))


def test_uniform_endpoints_and_exactness():
    u = philox.uniform_from_bits(np.array([0, 0xFFFFFFFF, 1 << 31], dtype=np.uint64))
    assert u[0] == 2.0 ** -24
    assert u[1] == 1.0 - 2.0 ** -24
    assert u[2] == 0.5 + 2.0 ** -24
    # exact in fp32 as well
    assert np.all(u.astype(np.float32).astype(np.float64) == u)
    assert np.all((1.0 - u).astype(np.float32).astype(np.float64) == 1.0 - u)


def test_uniform_moments():
    x = philox.stream_words(seed=42, rnd=0, tag=7, c1=np.arange(64), n=4096).reshape(-1)
    u = philox.uniform_from_bits(x)
    n = u.size
    assert abs(u.mean() - 0.5) < 5 * np.sqrt(1 / 12 / n)
    assert abs(u.var() - 1 / 12) < 5 * np.sqrt(1 / 180 / n)
    # bit balance of the raw words
    bits = ((x[:, None] >> np.arange(32, dtype=np.uint64)) & np.uint64(1)).mean(axis=0)
    assert np.all(np.abs(bits - 0.5) < 5 * np.sqrt(0.25 / n))


def test_gumbel_closed_forms():
    # F(g) = exp(-exp(-g)): g(u) inverts it
    u = np.linspace(1e-6, 1 - 1e-6, 1001)
    g = philox.gumbel_from_uniform(u)
    assert np.allclose(np.exp(-np.exp(-g)), u, rtol=1e-12, atol=0)
    # bounds of the 23-bit uniform
    assert abs(philox.GUMBEL_MIN - (-np.log(24 * np.log(2.0)))) < 1e-12
    assert 16.6 < philox.GUMBEL_MAX < 16.7
    # mean = Euler-Mascheroni, variance = pi^2 / 6
    x = philox.stream_words(seed=3, rnd=0, tag=7, c1=np.arange(32), n=8192).reshape(-1)
    gs = philox.gumbel_from_uniform(philox.uniform_from_bits(x))
    n = gs.size
    assert abs(gs.mean() - 0.5772156649) < 5 * np.sqrt(np.pi ** 2 / 6 / n)
    assert abs(gs.var() - np.pi ** 2 / 6) < 0.02
