"""Pins of the logit n-gram store oracle (STAND page, Methodology item 1:
top-k (index, probability) rows, weighted-average merge with unstored = 0,
truncation back to the top entries)."""

import numpy as np

import oracle
from oracle import NgramStore, ngram_merge, observe_topk


def f32(x):
    return np.float32(x)


def test_merge_worked_example():
    # stored {5: 0.5, 7: 0.3} seen once; observed {7: 0.6, 9: 0.2}:
    # 5 -> (0.5 + 0) / 2 = 0.25, 7 -> (0.3 + 0.6) / 2 = 0.45, 9 -> (0 + 0.2) / 2 = 0.1
    idx, prob = ngram_merge([5, 7, -1], f32([0.5, 0.3, 0]), 1, [7, 9, -1], f32([0.6, 0.2, 0]), 3)
    assert idx.tolist() == [7, 5, 9]
    assert np.allclose(prob, [0.45, 0.25, 0.1], rtol=1e-7, atol=0)
    # seen three times before: weights 3 : 1
    idx, prob = ngram_merge([5, 7], f32([0.5, 0.3]), 3, [7, 9], f32([0.6, 0.2]), 3)
    assert idx.tolist() == [5, 7, 9]
    assert np.allclose(prob, [0.375, 0.375, 0.05], rtol=1e-7, atol=0)
    # 5 and 7 tie exactly at 0.375: the lower index first


def test_truncation_keeps_the_largest_with_low_index_ties():
    idx, prob = ngram_merge([1, 2, 3], f32([0.4, 0.3, 0.2]), 1, [4, 5, 6], f32([0.6, 0.2, 0.2]), 3)
    # values: 1 .2, 2 .15, 3 .1, 4 .3, 5 .1, 6 .1 -> keep 4, 1, 2
    assert idx.tolist() == [4, 1, 2]
    idx, prob = ngram_merge([], [], 0, [9, 3, 8, 2], f32([0.25, 0.25, 0.25, 0.25]), 2)
    assert idx.tolist() == [2, 3] and np.all(prob == f32(0.25))


def test_running_mean_of_observations():
    """With no truncation the weights make the stored value the mean of every
    observation; equal weights (1 : 1) or a missing count would fail here."""
    rng = np.random.default_rng(1)
    st = NgramStore(2, 10)
    obs = rng.dirichlet(np.ones(6), size=25).astype(np.float32)
    ids = np.array([11, 3, 7, 40, 5, 2])
    for o in obs:
        assert st.update([[4, 8]], [ids], [o]) == 0
    idx, prob, cnt = st.lookup([[4, 8], [8, 4]])
    assert cnt.tolist() == [25, 0] and idx[1].tolist() == [-1] * 10
    mean = obs.astype(np.float64).mean(axis=0)
    got = {int(i): float(p) for i, p in zip(idx[0], prob[0]) if i >= 0}
    assert sorted(got) == sorted(ids.tolist())
    for i, m in zip(ids, mean):
        assert abs(got[int(i)] - m) < 1e-5
    # a repeated identical observation is a fixed point
    st2 = NgramStore(1, 4)
    for _ in range(7):
        st2.update([[3]], [[1, 2, -1, -1]], [f32([0.75, 0.25, 0, 0])])
    i2, p2, c2 = st2.lookup([[3]])
    assert c2[0] == 7 and i2[0, :2].tolist() == [1, 2] and np.all(p2[0, :2] == f32([0.75, 0.25]))


def test_order_within_a_batch_and_faults():
    st = NgramStore(3, 2)
    err = st.update([[1, 2, 3], [1, 2, 3], [1 << 20, 0, 0], [5, 5, 5], [6, 6, 6]],
                    [[1, -1], [2, -1], [1, -1], [1, 1], [1, 2]],
                    f32([[1.0, 0], [1.0, 0], [1.0, 0], [0.5, 0.5], [np.nan, 0.1]]))
    assert err == oracle.DEV_TOKEN_OOB | oracle.DEV_NONFINITE
    idx, prob, cnt = st.lookup([[1, 2, 3], [5, 5, 5], [6, 6, 6]])
    assert cnt.tolist() == [2, 0, 0]
    assert idx[0].tolist() == [1, 2] and np.all(prob[0] == f32(0.5))


def test_observe_topk_matches_a_sort_of_the_softmax():
    rng = np.random.default_rng(2)
    z = rng.standard_normal((5, 300)).astype(np.float32)
    z[1, [10, 20, 30]] = 9.0              # a three-way tie at the top
    z[2, :] = -np.inf
    z[2, 7] = 0.0                          # one finite entry: rest of the row is past V
    z[3, 4] = np.nan
    idx, prob, err = observe_topk(z, 0.7, 10)
    assert err == oracle.DEV_NONFINITE
    for r in (0, 1, 4):
        p = np.exp(z[r].astype(np.float64) / np.float64(np.float32(0.7)))
        p /= p.sum()
        order = sorted(range(300), key=lambda v: (-p[v], v))[:10]
        assert idx[r].tolist() == order
        assert np.allclose(prob[r], p[order], rtol=1e-6, atol=0)
    assert idx[1, :3].tolist() == [10, 20, 30]
    assert idx[2].tolist() == [7] + [-1] * 9 and prob[2, 0] == 1.0 and np.all(prob[2, 1:] == 0)
    assert idx[3].tolist() == [-1] * 10 and np.isnan(prob[3]).all()
    # rows past the first: row selection
    idx2, prob2, _ = observe_topk(z, 0.7, 10, rows=[4, 0])
    assert np.array_equal(idx2[0], idx[4]) and np.array_equal(prob2[1], prob[0])
