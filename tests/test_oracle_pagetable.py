"""Pins for the oracle's KV page-table remap."""

import numpy as np

import oracle


def test_hand_example():
    pt = np.array([[[0, 1, -1], [2, 3, 4], [5, 6, 7]]])
    anc = np.array([[1, 1, 2]])
    tok = np.array([[[10, 11], [20, 21], [30, 31]]])
    out = oracle.kv_pagetable_remap(pt, anc, num_pages=8, tok_in=tok)
    assert out["pt_out"].tolist() == [[[2, 3, 4], [2, 3, 4], [5, 6, 7]]]
    assert out["tok_out"].tolist() == [[[20, 21], [20, 21], [30, 31]]]
    assert out["refcnt"].tolist() == [0, 0, 2, 2, 2, 1, 1, 1]
    assert out["err"] == 0


def test_refcount_identity_and_errors():
    rng = np.random.default_rng(0)
    B, N, P = 3, 5, 7
    pt = rng.integers(-1, 50, size=(B, N, P))
    anc = np.sort(rng.integers(0, N, size=(B, N)), axis=1)
    out = oracle.kv_pagetable_remap(pt, anc, num_pages=50)
    assert out["refcnt"].sum() == int((out["pt_out"] >= 0).sum())
    for b in range(B):
        for i in range(N):
            assert np.array_equal(out["pt_out"][b, i], pt[b, anc[b, i]])
    pt[0, 0, 0] = 99
    anc2 = anc.copy()
    anc2[1, 2] = N
    out = oracle.kv_pagetable_remap(pt, anc2, num_pages=50)
    assert out["err"] & oracle.DEV_ANCESTOR_OOB
    assert np.all(out["pt_out"][1, 2] == -1)
