"""GPU test of ngram_store_update_noalloc: the n-gram store update with the
library's own fixed workspace.  It must leave the table exactly as the
caller-workspace entry point does, reject batches beyond its capacity, and
allocate no device memory.  Self-contained: passes alone in a fresh process and
after every other test."""

import ctypes

import numpy as np
import pytest
import torch

import resample_online_log_b200 as lib
from tests.parity import requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def batch(rng, U, n, k, nkeys, V):
    pool = rng.integers(0, 1 << 20, size=(nkeys, n)).astype(np.int32)
    ctx = pool[np.minimum(rng.zipf(1.4, size=U) - 1, nkeys - 1)]
    idx = np.full((U, k), -1, np.int32)
    prob = np.zeros((U, k), np.float32)
    for u in range(U):
        m = int(rng.integers(1, k + 1))
        idx[u, :m] = rng.choice(V, size=m, replace=False)
        prob[u, :m] = rng.dirichlet(np.ones(m + 1))[:m]
    return to_dev(ctx), to_dev(idx), to_dev(prob)


@pytest.mark.parametrize("U,n,k,cap", [(1, 1, 10, 64), (3000, 2, 10, 8192), (16384, 3, 4, 1 << 15)])
def test_noalloc_matches_workspace_entry(U, n, k, cap):
    rng = np.random.default_rng(U + n)
    ref = lib.NgramTable(cap, k, max_update=U)
    tab = torch.empty_like(ref.table)
    lib.ngram_table_clear(tab, cap, k)
    err_ref = torch.zeros((1,), dtype=torch.int32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    seen = []
    for _ in range(3):
        ctx, idx, prob = batch(rng, U, n, k, max(1, U // 4), 5000)
        ref.update(ctx, idx, prob, dev_err=err_ref)
        lib.ngram_store_update_noalloc(tab, cap, k, ctx, idx, prob, dev_err=err)
        seen.append(ctx)
    torch.cuda.synchronize()
    assert int(err.item()) == int(err_ref.item()) == 0
    # which slot a new n-gram claims depends on the order of concurrent claims;
    # what a lookup returns does not: compare every stored row
    q = torch.cat(seen)
    out = []
    for t in (ref.table, tab):
        i = torch.empty((q.shape[0], k), dtype=torch.int32, device="cuda")
        p = torch.empty((q.shape[0], k), dtype=torch.float32, device="cuda")
        c = torch.empty((q.shape[0],), dtype=torch.int32, device="cuda")
        lib.ngram_store_lookup(t, cap, k, q, i, p, count_out=c)
        out.append((i, p, c))
    torch.cuda.synchronize()
    assert all(torch.equal(a, b) for a, b in zip(*out))
    # every observation was merged into its n-gram exactly once
    _, first = np.unique(q.cpu().numpy(), axis=0, return_index=True)
    assert int(out[0][2].cpu().numpy()[first].sum()) == 3 * U


def test_noalloc_allocates_nothing_and_rejects_oversize():
    k, n, cap = 10, 2, 4096
    tab = torch.empty((lib.ngram_table_bytes(cap, k),), dtype=torch.uint8, device="cuda")
    lib.ngram_table_clear(tab, cap, k)
    rng = np.random.default_rng(2)
    ctx, idx, prob = batch(rng, 2000, n, k, 500, 3000)
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.ngram_store_update_noalloc(tab, cap, k, ctx, idx, prob, dev_err=err)  # loads the module
    torch.cuda.synchronize()
    free0, _ = torch.cuda.mem_get_info()
    torch_bytes0 = torch.cuda.memory_allocated()
    for _ in range(5):
        lib.ngram_store_update_noalloc(tab, cap, k, ctx, idx, prob, dev_err=err)
    torch.cuda.synchronize()
    free1, _ = torch.cuda.mem_get_info()
    assert free1 == free0 and torch.cuda.memory_allocated() == torch_bytes0
    assert int(err.item()) == 0
    # beyond the fixed workspace: refused before anything is enqueued
    L = lib.load()
    vp = ctypes.c_void_p
    st = L.ngram_store_update_noalloc(vp(tab.data_ptr()), cap, k, vp(ctx.data_ptr()), n,
                                      vp(idx.data_ptr()), vp(prob.data_ptr()), 16385, None, None)
    assert st == lib.SD_ERR_UNSUPPORTED
