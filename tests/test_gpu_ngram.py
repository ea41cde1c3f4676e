"""GPU parity of the logit n-gram store (STAND page, Methodology item 1) against
the oracle, through the C ABI: observed top-k rows, count-weighted merges with
truncation, lookups, faults, and the observe -> update -> lookup -> sparse
Gumbel-top-k drafting chain."""

import numpy as np
import pytest
import torch

import oracle
import resample_online_log_b200 as lib
from synth import gen
from tests.parity import discrete, requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def run_observe(z, k, tau, dtype="bf16", rows=None, ld=None):
    z = np.asarray(z, dtype=np.float32)
    R, V = z.shape
    if dtype == "bf16":
        bits = gen.f32_to_bf16_bits(z)
        zd = torch.from_numpy(bits.view(np.int16)).cuda().view(torch.bfloat16)
        z = gen.bf16_bits_to_f32(bits)
    else:
        zd = to_dev(z)
    if ld is not None and ld != V:
        wide = torch.zeros((R, ld), dtype=zd.dtype, device="cuda")
        wide[:, :V] = zd
        zd = wide[:, :V]
    U = R if rows is None else len(rows)
    rid = None if rows is None else to_dev(np.asarray(rows, np.int32))
    idx = torch.empty((U, k), dtype=torch.int32, device="cuda")
    prob = torch.empty((U, k), dtype=torch.float32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.ngram_observe_topk(zd, k, tau, idx, prob, row_ids=rid, dev_err=err)
    torch.cuda.synchronize()
    return z, idx.cpu().numpy(), prob.cpu().numpy(), int(err.item())


def check_observe(z, k, tau, g_idx, g_prob, g_err, rows=None):
    o_idx, o_prob, o_err = oracle.observe_topk(z, tau, k, rows=rows)
    assert g_err == o_err
    assert np.array_equal(g_idx, o_idx)
    fin = ~np.isnan(o_prob)
    assert np.array_equal(np.isnan(g_prob), ~fin)
    assert np.allclose(g_prob[fin], o_prob[fin], rtol=1e-5, atol=1e-30)


@pytest.mark.parametrize("R,V,k,dtype,scale", [(3, 1, 10, "bf16", 1.0), (5, 7, 10, "f32", 2.0),
                                               (16, 300, 10, "bf16", 2.0), (7, 32000, 10, "bf16", 3.0),
                                               (4, 152064, 10, "bf16", 2.5), (9, 5003, 16, "f32", 1.0),
                                               (300, 4096, 1, "bf16", 2.0)])
def test_observe_parity(R, V, k, dtype, scale):
    rng = np.random.default_rng(R * 11 + V)
    z = (rng.standard_normal((R, V)) * scale).astype(np.float32)
    z, g_idx, g_prob, g_err = run_observe(z, k, 0.8, dtype)
    check_observe(z, k, 0.8, g_idx, g_prob, g_err)


def test_observe_ties_masks_faults_and_row_ids():
    rng = np.random.default_rng(4)
    V = 6000
    z = rng.standard_normal((8, V)).astype(np.float32)
    z[0, [100, 7, 5000]] = 6.0                # ties at the top: lower index first
    z[1, :] = 1.0                              # every entry tied: more than the gather buffer
    z[2, :] = -np.inf
    z[2, [3, 9]] = [0.5, 0.25]                 # two finite entries: the rest unstored
    z[3, 0] = np.nan                           # a NaN before any finite entry of its thread
    z[3, 1:8] = -np.inf
    z[4, 2000] = np.inf
    z[5, :] = -np.inf
    z[6, ::2] = 3.0                            # 3000 ties above the rest
    z[6, 1::2] = 0.0
    z, g_idx, g_prob, g_err = run_observe(z, 10, 1.0, "f32", ld=6016)
    check_observe(z, 10, 1.0, g_idx, g_prob, g_err)
    assert g_idx[0, :3].tolist() == [7, 100, 5000]
    assert g_idx[1].tolist() == list(range(10)) and g_idx[6].tolist() == list(range(0, 20, 2))
    assert g_idx[2].tolist() == [3, 9] + [-1] * 8
    assert np.isnan(g_prob[3]).all() and np.isnan(g_prob[4]).all() and np.isnan(g_prob[5]).all()
    # row selection, and a row id out of range
    rows = [7, 0, 0, 6]
    _, g_idx2, g_prob2, g_err2 = run_observe(z, 10, 1.0, "f32", rows=rows)
    check_observe(z, 10, 1.0, g_idx2, g_prob2, g_err2, rows=rows)
    _, g_idx3, g_prob3, g_err3 = run_observe(z[:2], 10, 1.0, "f32", rows=[1, 2])
    assert g_err3 == lib.DEV_TOKEN_OOB and g_idx3[1].tolist() == [-1] * 10
    assert np.isnan(g_prob3[1]).all() and np.array_equal(g_idx3[0], g_idx[1])


def observations(rng, U, k, V, zero_frac=0.0):
    """Observation rows shaped like observe_topk output: distinct ids, descending
    probabilities summing to at most 1, a few rows shorter than k."""
    idx = np.full((U, k), -1, np.int32)
    prob = np.zeros((U, k), np.float32)
    for u in range(U):
        m = k if rng.random() > 0.2 else int(rng.integers(0, k + 1))
        ids = rng.choice(V, size=m, replace=False)
        p = np.sort(rng.dirichlet(np.ones(m + 1) * 0.7)[:m])[::-1].astype(np.float32)
        if zero_frac and m:
            p[rng.random(m) < zero_frac] = 0.0
        idx[u, :m] = ids
        prob[u, :m] = p
    return idx, prob


def lookup_all(tab, keys, k):
    ctx = to_dev(np.asarray(keys, np.int32))
    Q = ctx.shape[0]
    idx = torch.empty((Q, k), dtype=torch.int32, device="cuda")
    prob = torch.empty((Q, k), dtype=torch.float32, device="cuda")
    cnt = torch.empty((Q,), dtype=torch.int32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tab.lookup(ctx, idx, prob, count_out=cnt, dev_err=err)
    torch.cuda.synchronize()
    return idx.cpu().numpy(), prob.cpu().numpy(), cnt.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("n,k,cap,U,nkeys,batches,V", [(1, 10, 64, 40, 20, 6, 50), (2, 10, 4096, 500, 300, 5, 2000),
                                                      (3, 16, 1 << 15, 4000, 3000, 3, 152064),
                                                      (2, 4, 1024, 16384, 700, 2, 30), (3, 1, 128, 77, 50, 4, 9)])
def test_update_lookup_parity(n, k, cap, U, nkeys, batches, V):
    rng = np.random.default_rng(n * 100 + k + U)
    pool = rng.integers(0, 1 << 20, size=(nkeys, n)).astype(np.int32)
    tab = lib.NgramTable(cap, k, max_update=U)
    st = oracle.NgramStore(n, k)
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    for b in range(batches):
        # skewed key frequencies: many repeats within one batch and across batches
        which = np.minimum(rng.zipf(1.3, size=U) - 1, nkeys - 1)
        ctx = pool[which]
        idx, prob = observations(rng, U, k, V, zero_frac=0.05 if b == 1 else 0.0)
        tab.update(to_dev(ctx), to_dev(idx), to_dev(prob), dev_err=err)
        assert st.update(ctx, idx, prob) == 0
        queries = np.concatenate([pool, rng.integers(0, 1 << 20, size=(20, n)).astype(np.int32)])
        g_idx, g_prob, g_cnt, g_err = lookup_all(tab, queries, k)
        o_idx, o_prob, o_cnt = st.lookup(queries)
        assert g_err == 0 and int(err.item()) == 0
        assert np.array_equal(g_cnt, o_cnt), b
        assert np.array_equal(g_idx, o_idx), b
        # one rounding per fp64 operation on both sides: equal bits
        assert np.array_equal(g_prob.view(np.uint32), o_prob.view(np.uint32)), b


def test_update_faults():
    k, n = 4, 2
    tab = lib.NgramTable(64, k, max_update=8)
    ctx = np.array([[1, 2], [1 << 20, 0], [3, 4], [5, 6], [1, 2], [-1, 0]], np.int32)
    idx = np.array([[1, 2, -1, -1], [1, -1, -1, -1], [7, 7, -1, -1], [1, 2, 3, -1],
                    [2, 9, -1, -1], [1, -1, -1, -1]], np.int32)
    prob = np.array([[0.5, 0.25, 0, 0], [1, 0, 0, 0], [0.5, 0.5, 0, 0], [0.5, np.nan, 0.1, 0],
                     [0.5, 0.5, 0, 0], [1, 0, 0, 0]], np.float32)
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tab.update(to_dev(ctx), to_dev(idx), to_dev(prob), dev_err=err)
    torch.cuda.synchronize()
    st = oracle.NgramStore(n, k)
    o_err = st.update(ctx, idx, prob)
    assert int(err.item()) == o_err == lib.DEV_TOKEN_OOB | lib.DEV_NONFINITE
    q = np.array([[1, 2], [3, 4], [5, 6], [0, 0]], np.int32)
    g_idx, g_prob, g_cnt, g_err = lookup_all(tab, q, k)
    o_idx, o_prob, o_cnt = st.lookup(q)
    assert np.array_equal(g_cnt, o_cnt) and np.array_equal(g_idx, o_idx)
    assert np.array_equal(g_prob, o_prob)
    # (3, 4) and (5, 6) had only faulty rows: their slots are claimed but hold no
    # observation, which a lookup reports as count 0 and an empty row
    assert g_cnt.tolist() == [2, 0, 0, 0]
    _, _, _, g_err = lookup_all(tab, np.array([[1, 1 << 20]], np.int32), k)
    assert g_err == lib.DEV_TOKEN_OOB


def test_table_full():
    k, n, cap = 2, 1, 32
    tab = lib.NgramTable(cap, k, max_update=64)
    ctx = np.arange(40, dtype=np.int32)[:, None]
    idx = np.tile(np.array([[3, 4]], np.int32), (40, 1))
    prob = np.tile(np.array([[0.5, 0.25]], np.float32), (40, 1))
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    tab.update(to_dev(ctx), to_dev(idx), to_dev(prob), dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == lib.DEV_TABLE_FULL
    g_idx, g_prob, g_cnt, _ = lookup_all(tab, ctx, k)
    assert int((g_cnt == 1).sum()) == cap and set(np.unique(g_cnt).tolist()) == {0, 1}
    stored = g_cnt == 1
    assert np.all(g_idx[stored] == [3, 4]) and np.all(g_prob[stored] == np.float32([0.5, 0.25]))
    assert np.all(g_idx[~stored] == -1)


def test_observe_update_lookup_draft_chain():
    """Target rows -> observed top-10 -> store -> lookup -> Gumbel-top-k drafts."""
    rng = np.random.default_rng(8)
    R, V, k, n = 64, 32000, 10, 2
    z = (rng.standard_normal((R, V)) * 3).astype(np.float32)
    z, g_idx, g_prob, g_err = run_observe(z, k, 0.7, "bf16")
    assert g_err == 0
    ctx = rng.integers(0, 50, size=(R, n)).astype(np.int32)
    ctx[R // 2:] = ctx[:R // 2]                       # every n-gram seen twice
    tab = lib.NgramTable(1024, k, max_update=R)
    tab.update(to_dev(ctx), to_dev(g_idx), to_dev(g_prob))
    st = oracle.NgramStore(n, k)
    st.update(ctx, g_idx, g_prob)
    l_idx, l_prob, l_cnt, _ = lookup_all(tab, ctx[:R // 2], k)
    o_idx, o_prob, o_cnt = st.lookup(ctx[:R // 2])
    assert np.array_equal(l_idx, o_idx) and np.array_equal(l_prob, o_prob) and np.all(l_cnt >= 2)
    drafts = torch.empty((R // 2, 3), dtype=torch.int32, device="cuda")
    lib.gumbel_topk_sparse(to_dev(l_idx), to_dev(l_prob), 3, 1.0, 5, 1, drafts)
    torch.cuda.synchronize()
    o = oracle.gumbel_topk_sparse(l_idx, l_prob, 3, 1.0, 5, 1)
    discrete(drafts.cpu().numpy(), o["idx"], o["margin"][:, None], "drafts")
