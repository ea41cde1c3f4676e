"""GPU parity of gumbel_topk (dense) and gumbel_topk_sparse against the oracle."""

import numpy as np
import pytest
import torch

import oracle
import resample_online_log_b200 as lib
import synth
from synth import gen
from tests.parity import bf16_dev, close, discrete, requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def run_dense(z, k, tau, seed, rnd, dtype="bf16"):
    rows = z.shape[0]
    t = bf16_dev(z) if dtype == "bf16" else to_dev(z.astype(np.float32))
    idx = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    sc = torch.empty((rows, k), dtype=torch.float32, device="cuda")
    lp = torch.empty((rows, k), dtype=torch.float32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.gumbel_topk(t, k, tau, seed, rnd, idx, score_out=sc, logp_out=lp, dev_err=err)
    torch.cuda.synchronize()
    return dict(idx=idx.cpu().numpy(), score=sc.cpu().numpy(), logp=lp.cpu().numpy(),
                err=int(err.item()))


def compare_dense(g, o, name):
    discrete(g["idx"], o["idx"], o["margin"][:, None], name + ".idx")
    same = np.all(g["idx"] == o["idx"], axis=1)
    close(g["score"][same], o["score"][same], 1e-4, name + ".score")
    close(g["logp"][same], o["logp"][same], 1e-5, name + ".logp")
    assert g["err"] == o["err"]


@pytest.mark.parametrize("V,k,tau,dtype", [(1000, 8, 0.6, "bf16"), (7, 7, 1.0, "bf16"),
                                           (32000, 4, 1.3, "f32"), (152064, 8, 0.6, "bf16"),
                                           (50001, 16, 0.8, "bf16"), (9, 1, 1.0, "f32")])
def test_dense_random(V, k, tau, dtype):
    rng = np.random.default_rng(V + k)
    rows = 6
    z = (rng.standard_normal((rows, V)) * 3).astype(np.float32)
    if dtype == "bf16":
        z = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(z))
    g = run_dense(z, k, tau, 3, 1, dtype)
    o = oracle.gumbel_topk(z, k, tau, 3, 1)
    compare_dense(g, o, f"dense{V}")


def test_dense_peaked_and_masked_rows():
    rng = np.random.default_rng(1)
    z = (rng.standard_normal((5, 4000)) * 2).astype(np.float32)
    z[0, 17] = 60.0                   # one dominant entry
    z[1, :] = -np.inf
    z[1, [3, 900, 2500]] = [0.5, 0.25, 0.0]   # fewer finite entries than k
    z[2, 10] = np.nan                 # non-finite row
    z[3, :] = 1.0                     # all equal: order decided by the noise alone
    z = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(z))
    g = run_dense(z, 8, 1.0, 4, 0)
    o = oracle.gumbel_topk(z, 8, 1.0, 4, 0)
    assert g["err"] == o["err"] == oracle.DEV_NONFINITE
    assert np.array_equal(g["idx"], o["idx"])
    assert list(g["idx"][1, 3:]) == [-1] * 5


def check_all_rows(z, cfg, idx, sc, lp, seed, rnd):
    """Identities every row of the whole config must satisfy (the oracle covers
    sampled rows): indices in range and distinct; logp = z[idx]/tau - lse (a
    gather of the input and the row's log-sum-exp, fp64); each score is at most
    its block's maximum M_j = log sum_{v in j} e^{z_v/tau} + G_j (block noise
    from the oracle's generator) and the first equals its block's maximum;
    scores are non-increasing along k."""
    from oracle.philox import STREAM_TOPK_BLOCK, gumbel_from_uniform, stream_words, uniform_from_bits
    rows, V = z.shape
    tau = float(np.float32(cfg.tau))  # the C ABI takes tau in fp32
    assert bool(((idx >= 0) & (idx < V)).all()), "topk: index out of range"
    srt = idx.sort(dim=1).values
    assert bool((srt[:, 1:] != srt[:, :-1]).all()), "topk: repeated index in a row"
    lse = torch.cat([torch.logsumexp(z[r0:r0 + 256].double() / tau, dim=1)
                     for r0 in range(0, rows, 256)])
    a = z.gather(1, idx.long()).double() / tau
    dl = (lp.double() - (a - lse[:, None])).abs()
    assert bool((dl <= 1e-5 * (1.0 + a.abs())).all()), f"topk: logp off by {float(dl.max()):.3e}"
    nb = (V + 127) // 128
    lam = []
    for r0 in range(0, rows, 256):
        zz = torch.full((min(256, rows - r0), nb * 128), -float("inf"), dtype=torch.float64, device=z.device)
        zz[:, :V] = z[r0:r0 + 256].double() / tau
        lam.append(torch.logsumexp(zz.view(-1, nb, 128), dim=2))
    lam = torch.cat(lam)
    G = torch.from_numpy(gumbel_from_uniform(uniform_from_bits(
        stream_words(seed, rnd, STREAM_TOPK_BLOCK, np.arange(rows), nb)))).to(z.device)
    Mj = (lam + G).gather(1, (idx.long() // 128))
    s64 = sc.double()
    assert bool((s64 <= Mj + 1e-4 * (1 + Mj.abs())).all()), "topk: a score above its block's maximum"
    assert bool(((s64[:, 0] - Mj[:, 0]).abs() <= 1e-4 * (1 + Mj[:, 0].abs())).all()), \
        "topk: the first score is not its block's maximum"
    assert bool((sc[:, 1:] <= sc[:, :-1]).all()), "topk: scores not in descending order"


def test_dense_config_sampled():
    """Whole 4096 x 152064 config on the device; sampled rows against the oracle on
    host-built rows (same bytes)."""
    from synth import device as sdev
    cfg = synth.CONFIGS["topk"]
    d = sdev.gen_config_device(cfg)
    z = d["z"]
    rows = z.shape[0]
    idx = torch.empty((rows, cfg.topk), dtype=torch.int32, device="cuda")
    sc = torch.empty((rows, cfg.topk), dtype=torch.float32, device="cuda")
    lp = torch.empty((rows, cfg.topk), dtype=torch.float32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.gumbel_topk(z, cfg.topk, cfg.tau, cfg.seed, 2, idx, score_out=sc, logp_out=lp, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_all_rows(z, cfg, idx, sc, lp, cfg.seed, 2)
    for r in [0, 1, 2047, 4095]:
        h = gen.gen_config_rows(cfg, seqs=[r])
        assert np.array_equal(z[r].float().cpu().numpy(), h["z"][0])
        o = oracle.gumbel_topk(h["z"], cfg.topk, cfg.tau, cfg.seed, 2, r0=r)
        g = dict(idx=idx[r:r + 1].cpu().numpy(), score=sc[r:r + 1].cpu().numpy(),
                 logp=lp[r:r + 1].cpu().numpy(), err=0)
        compare_dense(g, o, f"topk[{r}]")


def run_sparse(ix, pr, k, tau, seed, rnd):
    rows, L = ix.shape
    out = torch.empty((rows, k), dtype=torch.int32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.gumbel_topk_sparse(to_dev(ix.astype(np.int32)), to_dev(pr.astype(np.float32)), k, tau, seed,
                           rnd, out, dev_err=err)
    torch.cuda.synchronize()
    return out.cpu().numpy(), int(err.item())


def test_sparse_config_full():
    cfg = synth.CONFIGS["topk"]
    ix, pr = gen.sparse_rows(cfg.seed, cfg.B, cfg.sparse_L, cfg.V)
    g, err = run_sparse(ix, pr, cfg.topk, cfg.tau, cfg.seed, 0)
    o = oracle.gumbel_topk_sparse(ix, pr, cfg.topk, cfg.tau, cfg.seed, 0)
    discrete(g, o["idx"], o["margin"][:, None], "sparse.idx")
    assert err == o["err"] == 0


def test_sparse_edge_cases():
    rng = np.random.default_rng(2)
    ix = rng.integers(0, 1000, size=(6, 10))
    pr = rng.dirichlet(np.full(10, 0.3), size=6).astype(np.float32)
    pr[0, 3:] = 0.0           # only 3 stored entries, k = 5
    pr[1, 4] = np.nan         # bad row
    g, err = run_sparse(ix, pr, 5, 1.0, 7, 3)
    o = oracle.gumbel_topk_sparse(ix, pr, 5, 1.0, 7, 3)
    assert err == o["err"] == oracle.DEV_NONFINITE
    assert np.array_equal(g, o["idx"])
    assert list(g[0, 3:]) == [-1, -1]
    g, _ = run_sparse(ix[2:], pr[2:], 10, 0.5, 7, 3)     # k = L: a full permutation
    o = oracle.gumbel_topk_sparse(ix[2:], pr[2:], 10, 0.5, 7, 3)
    assert np.array_equal(g, o["idx"])


def test_dense_nan_behind_masked_entries():
    """A NaN met while every earlier entry of the thread's stream is -inf still
    marks the row non-finite."""
    rng = np.random.default_rng(12)
    z = (rng.standard_normal((3, 20000)) * 2).astype(np.float32)
    z[1, 0] = np.nan
    z[1, 1:8] = -np.inf
    z[2, 8 * 513] = np.nan          # second chunk of thread 1, first chunk all -inf
    z[2, 8:16] = -np.inf
    z[2, 8 * 513 + 1:8 * 514] = -np.inf
    z = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(z))
    g = run_dense(z, 4, 1.0, 2, 0)
    o = oracle.gumbel_topk(z, 4, 1.0, 2, 0)
    assert g["err"] == o["err"] == oracle.DEV_NONFINITE
    assert np.all(g["idx"][1:] == -1)
    compare_dense({k: v[:1] if k != "err" else 0 for k, v in g.items()},
                  {**{k: v[:1] for k, v in o.items() if k not in ("err",)}, "err": 0}, "nanrow")
