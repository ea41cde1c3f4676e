"""GPU parity of smcsd_score against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import resample_online_log_b200 as lib
import synth
from synth import gen
from tests.parity import TOL_LOGW, TOL_LSE, TOL_TV, bf16_dev, close, discrete, requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def run_score(zT, zD, x, tau, seed, rnd, dtype="bf16", logw_prev=None, ld=None,
              log_potential=None):
    B, N, R, V = zT.shape
    K = R - 1
    dev = "cuda"
    if dtype == "bf16":
        t, d = bf16_dev(zT), bf16_dev(zD)
    else:
        t, d = to_dev(zT.astype(np.float32)), to_dev(zD.astype(np.float32))
    if ld is not None and ld != V:
        tt = torch.zeros((B, N, R, ld), dtype=t.dtype, device=dev)
        dd = torch.zeros((B, N, R, ld), dtype=t.dtype, device=dev)
        tt[..., :V] = t
        dd[..., :V] = d
        t, d = tt[..., :V], dd[..., :V]
    xs = to_dev(np.asarray(x, dtype=np.int32))
    out = dict(
        logw=torch.empty((B, N), dtype=torch.float64, device=dev),
        bonus=torch.empty((B, N), dtype=torch.int32, device=dev),
        tv=torch.empty((B, N, R), dtype=torch.float32, device=dev),
        tokens=torch.empty((B, N, R), dtype=torch.int32, device=dev),
        lse=torch.empty((B, N, R, 2), dtype=torch.float64, device=dev),
        lp=torch.empty((B, N, K, 2), dtype=torch.float64, device=dev),
        err=torch.zeros((1,), dtype=torch.int32, device=dev))
    prev = None if logw_prev is None else to_dev(np.asarray(logw_prev, dtype=np.float64))
    phi = None if log_potential is None else to_dev(np.asarray(log_potential, dtype=np.float64))
    lib.smcsd_score(t, d, xs, tau, seed, rnd, out["logw"], out["bonus"], logw_prev=prev,
                    log_potential=phi, tv_out=out["tv"], tokens_out=out["tokens"], lse_out=out["lse"],
                    lp_out=out["lp"], dev_err=out["err"])
    torch.cuda.synchronize()
    res = {k: v.cpu().numpy() for k, v in out.items()}
    res["err"] = int(res["err"][0])
    return res


def compare(g, o, name):
    close(g["logw"], o["logw"], TOL_LOGW, name + ".logw")
    close(g["tv"], o["tv"], TOL_TV, name + ".tv")
    close(g["lse"], o["lse"], TOL_LSE, name + ".lse")
    close(g["lp"], o["lp"], TOL_LSE, name + ".lp")
    discrete(g["bonus"], o["bonus"], o["bonus_margin"], name + ".bonus")
    K = o["tokens"].shape[-1] - 1
    assert np.array_equal(g["tokens"][..., :K], o["tokens"][..., :K])
    assert np.array_equal(g["tokens"][..., K], g["bonus"])
    assert g["err"] == o["err"], (g["err"], o["err"])


def rand_case(rng, B, N, K, V, scale=2.0, noise=1.0):
    zT = (rng.standard_normal((B, N, K + 1, V)) * scale).astype(np.float32)
    zD = (zT + rng.standard_normal(zT.shape) * noise).astype(np.float32)
    zT = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(zT))
    zD = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(zD))
    x = rng.integers(0, V, size=(B, N, K)).astype(np.int32)
    return zT, zD, x


def test_smc_small_config_fp32():
    cfg = synth.CONFIGS["smc_small"]
    d = gen.gen_config_rows(cfg)
    g = run_score(d["zT"], d["zD"], d["draft"], cfg.tau, cfg.seed, 0, dtype="f32")
    o = oracle.smcsd_score(d["zT"], d["zD"], d["draft"], cfg.tau, cfg.seed, 0)
    compare(g, o, "smc_small")


@pytest.mark.parametrize("V,tau", [(1003, 0.8), (4096, 1.0), (33001, 0.7)])
def test_ragged_vocab_bf16(V, tau):
    rng = np.random.default_rng(V)
    zT, zD, x = rand_case(rng, 2, 3, 2, V)
    g = run_score(zT, zD, x, tau, 11, 5)
    o = oracle.smcsd_score(zT, zD, x, tau, 11, 5)
    compare(g, o, f"ragged{V}")


def test_split_v_llama_vocab_bf16():
    rng = np.random.default_rng(7)
    zT, zD, x = rand_case(rng, 1, 3, 2, 128256, scale=3.0, noise=1.5)
    g = run_score(zT, zD, x, 1.0, 3, 1)
    o = oracle.smcsd_score(zT, zD, x, 1.0, 3, 1)
    compare(g, o, "v128256")


def test_fp32_multi_tile():
    rng = np.random.default_rng(8)
    zT, zD, x = rand_case(rng, 2, 2, 3, 40000)
    g = run_score(zT, zD, x, 1.3, 4, 2, dtype="f32")
    o = oracle.smcsd_score(zT, zD, x, 1.3, 4, 2)
    compare(g, o, "f32_40000")


def test_strided_unaligned_rows():
    """ld*2 bytes is not a multiple of 16: the bulk-copy path is off, plain loads are used."""
    rng = np.random.default_rng(9)
    zT, zD, x = rand_case(rng, 2, 2, 2, 5000)
    g = run_score(zT, zD, x, 0.9, 5, 0, ld=5003)
    o = oracle.smcsd_score(zT, zD, x, 0.9, 5, 0)
    compare(g, o, "strided")


def test_padded_aligned_rows():
    rng = np.random.default_rng(10)
    zT, zD, x = rand_case(rng, 1, 4, 3, 32000)
    g = run_score(zT, zD, x, 1.0, 6, 0, ld=32768)
    o = oracle.smcsd_score(zT, zD, x, 1.0, 6, 0)
    compare(g, o, "padded")


def test_edge_cases_k0_n1_v1():
    rng = np.random.default_rng(11)
    zT, zD, x = rand_case(rng, 3, 2, 0, 700)          # K = 0: bonus only
    g = run_score(zT, zD, x, 1.0, 1, 0)
    o = oracle.smcsd_score(zT, zD, x, 1.0, 1, 0)
    compare(g, o, "K0")
    assert np.all(g["logw"] == 0.0)
    zT, zD, x = rand_case(rng, 2, 1, 3, 900)          # N = 1
    g = run_score(zT, zD, x, 1.0, 1, 0)
    compare(g, oracle.smcsd_score(zT, zD, x, 1.0, 1, 0), "N1")
    zT, zD, x = rand_case(rng, 2, 2, 2, 1)            # V = 1: point masses
    g = run_score(zT, zD, x, 1.0, 1, 0)
    compare(g, oracle.smcsd_score(zT, zD, x, 1.0, 1, 0), "V1")
    # point masses are equal distributions: TV is 0 up to the fp32 rounding of
    # the normalisation p = e * (1 / sum e) (a few ulp of 1), far inside 1e-5
    assert np.all(g["bonus"] == 0) and np.all(np.abs(g["tv"]) <= 1e-6)


def test_logw_prev_is_added():
    rng = np.random.default_rng(12)
    zT, zD, x = rand_case(rng, 2, 4, 2, 3000)
    prev = rng.standard_normal((2, 4))
    g = run_score(zT, zD, x, 1.0, 2, 9, logw_prev=prev)
    compare(g, oracle.smcsd_score(zT, zD, x, 1.0, 2, 9, logw_prev=prev), "prev")


def test_identical_rows_invariants():
    rng = np.random.default_rng(13)
    zT, _, x = rand_case(rng, 2, 4, 3, 128256)
    g = run_score(zT, zT.copy(), x, 0.7, 3, 3)
    assert np.all(g["logw"] == 0.0)
    assert np.all(g["tv"] == 0.0)


def test_ragged_vocab_padded_stride():
    """V not a multiple of the 8-entry chunk, rows padded to a 16-byte stride:
    the last chunk of every row is read entry by entry."""
    rng = np.random.default_rng(16)
    V = 33001
    zT, zD, x = rand_case(rng, 2, 5, 3, V)
    g = run_score(zT, zD, x, 0.9, 21, 2, ld=33008)
    o = oracle.smcsd_score(zT, zD, x, 0.9, 21, 2)
    compare(g, o, "ragged_padded")


def test_without_tv_output():
    """tv_out = NULL: the other outputs are unchanged."""
    rng = np.random.default_rng(17)
    B, N, K, V = 2, 6, 3, 40960
    zT, zD, x = rand_case(rng, B, N, K, V)
    g = run_score(zT, zD, x, 1.0, 5, 8)
    t, d = bf16_dev(zT), bf16_dev(zD)
    xs = to_dev(x)
    logw = torch.empty((B, N), dtype=torch.float64, device="cuda")
    bonus = torch.empty((B, N), dtype=torch.int32, device="cuda")
    lse = torch.empty((B, N, K + 1, 2), dtype=torch.float64, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.smcsd_score(t, d, xs, 1.0, 5, 8, logw, bonus, lse_out=lse, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    assert np.array_equal(logw.cpu().numpy(), g["logw"])
    assert np.array_equal(bonus.cpu().numpy(), g["bonus"])
    assert np.array_equal(lse.cpu().numpy(), g["lse"])


def test_faults_set_error_bits():
    rng = np.random.default_rng(14)
    zT, zD, x = rand_case(rng, 1, 3, 2, 2000)
    x[0, 0, 1] = 2000                       # token out of range
    zT[0, 1, 2, 17] = np.nan                # NaN in particle 1's bonus row
    zD[0, 2, :, :] = -np.inf                # particle 2: all draft rows -inf
    g = run_score(zT, zD, x, 1.0, 1, 0)
    o = oracle.smcsd_score(zT, zD, x, 1.0, 1, 0)
    assert g["err"] == o["err"] == (oracle.DEV_TOKEN_OOB | oracle.DEV_NONFINITE)
    close(g["logw"], o["logw"], TOL_LOGW, "faults.logw")
    close(g["tv"], o["tv"], TOL_TV, "faults.tv")
    assert g["bonus"][0, 1] == -1 and o["bonus"][0, 1] == -1
    discrete(g["bonus"], o["bonus"], o["bonus_margin"], "faults.bonus")


def test_reruns_bit_identical():
    rng = np.random.default_rng(15)
    zT, zD, x = rand_case(rng, 2, 8, 4, 128256)
    a = run_score(zT, zD, x, 1.0, 77, 4)
    b = run_score(zT, zD, x, 1.0, 77, 4)
    for key in ("logw", "tv", "bonus", "lse", "lp", "tokens"):
        assert np.array_equal(a[key], b[key], equal_nan=True), key


def check_all_rows(d, cfg, logw, tv, lp, lse, name):
    """Identities every row of a whole config must satisfy, checked on the device
    for all particles (the oracle comparison above covers sampled sequences):
    lp + lse equals the draft token's logit over tau (a gather of the input);
    logw is the sum over k of lp - lq; max_v z/tau <= lse <= max_v z/tau + log V;
    0 <= tv <= 1."""
    B, N, R, V, K = cfg.B, cfg.N, cfg.R, cfg.V, cfg.K
    U = B * N
    zT, zD = d["zT"].view(U, R, -1), d["zD"].view(U, R, -1)
    lp, lse = lp.view(U, K, 2), lse.view(U, R, 2)
    x = d["draft"].view(U, K, 1).long()
    tau = float(np.float32(cfg.tau))  # the C ABI takes tau in fp32
    for h, z in enumerate((zT, zD)):
        zx = z[:, :K].gather(2, x).squeeze(2).double() / tau
        got = lp[..., h] + lse[:, :K, h]
        bad = (got - zx).abs() > 1e-9 * (1.0 + zx.abs())
        assert not bad.any(), f"{name}: lp + lse != z[x]/tau at (unit, k) {bad.nonzero()[:8].tolist()}"
        mx = torch.cat([z[u0:u0 + 512].amax(2) for u0 in range(0, U, 512)]).double() / tau
        # (the slice sums are fp32, so the lower bound holds to their rounding)
        lo_ok = lse[..., h] >= mx - 1e-6 * (1.0 + mx.abs())
        hi_ok = lse[..., h] <= mx + float(np.log(V)) + 1e-6 * (1.0 + mx.abs())
        assert bool((lo_ok & hi_ok).all()), f"{name}: lse outside [max, max + log V]"
    s = (lp[..., 0] - lp[..., 1]).sum(1)
    lw = logw.view(U)
    assert bool(((lw - s).abs() <= 1e-9 * (1.0 + s.abs())).all()), f"{name}: logw != sum(lp - lq)"
    assert bool(((tv >= 0) & (tv <= 1 + 1e-6)).all()), f"{name}: tv outside [0, 1]"


@pytest.mark.parametrize("name,seqs", [("smc_batch", [0, 37]), ("smc_scale", [5, 200])])
def test_full_size_config_sampled(name, seqs):
    """Whole config on the GPU (inputs built on the device), sampled sequences checked
    against the oracle on host-built inputs; the device bytes of those sequences must
    equal the host generator's."""
    from synth import device as sdev
    cfg = synth.CONFIGS[name]
    d = sdev.gen_config_device(cfg)
    B, N, R, V, K = cfg.B, cfg.N, cfg.R, cfg.V, cfg.K
    out_logw = torch.empty((B, N), dtype=torch.float64, device="cuda")
    out_bonus = torch.empty((B, N), dtype=torch.int32, device="cuda")
    out_tv = torch.empty((B, N, R), dtype=torch.float32, device="cuda")
    out_lp = torch.empty((B, N, K, 2), dtype=torch.float64, device="cuda")
    out_lse = torch.empty((B, N, R, 2), dtype=torch.float64, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.smcsd_score(d["zT"], d["zD"], d["draft"], cfg.tau, cfg.seed, 1, out_logw, out_bonus,
                    tv_out=out_tv, lp_out=out_lp, lse_out=out_lse, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    check_all_rows(d, cfg, out_logw, out_tv, out_lp, out_lse, name)
    for b in seqs:
        h = gen.gen_config_rows(cfg, seqs=[b])
        dev_t = d["zT"][b].float().cpu().numpy()
        dev_d = d["zD"][b].float().cpu().numpy()
        assert np.array_equal(dev_t, h["zT"][0]) and np.array_equal(dev_d, h["zD"][0])
        assert np.array_equal(d["draft"][b].cpu().numpy(), h["draft"][0])
        o = oracle.smcsd_score(h["zT"], h["zD"], h["draft"], cfg.tau, cfg.seed, 1, b0=b)
        close(out_logw[b:b + 1].cpu().numpy(), o["logw"], TOL_LOGW, f"{name}[{b}].logw")
        close(out_tv[b:b + 1].cpu().numpy(), o["tv"], TOL_TV, f"{name}[{b}].tv")
        close(out_lp[b:b + 1].cpu().numpy(), o["lp"], TOL_LSE, f"{name}[{b}].lp")
        discrete(out_bonus[b:b + 1].cpu().numpy(), o["bonus"], o["bonus_margin"], f"{name}[{b}].bonus")
    del d
    torch.cuda.empty_cache()


@pytest.mark.parametrize("with_prev", [False, True])
def test_log_potential(with_prev):
    """A per-particle log-potential (reward-weighted / constrained target) adds
    to the carried weight; -inf rules a particle out without an error."""
    rng = np.random.default_rng(41)
    B, N, K, V = 3, 8, 4, 3000
    zT, zD, x = rand_case(rng, B, N, K, V)
    phi = rng.standard_normal((B, N)) * 2.0
    phi[1, 3] = -np.inf
    prev = rng.standard_normal((B, N)) if with_prev else None
    g = run_score(zT, zD, x, 0.8, 12, 3, logw_prev=prev, log_potential=phi)
    o = oracle.smcsd_score(zT, zD, x, 0.8, 12, 3, logw_prev=prev, log_potential=phi)
    assert g["logw"][1, 3] == -np.inf
    close(np.where(np.isinf(g["logw"]), 0, g["logw"]), np.where(np.isinf(o["logw"]), 0, o["logw"]),
          TOL_LOGW, "logw")
    compare({**g, "logw": np.nan_to_num(g["logw"], neginf=0)},
            {**o, "logw": np.nan_to_num(o["logw"], neginf=0)}, "potential")
    # the potential shifts nothing but the weight
    g0 = run_score(zT, zD, x, 0.8, 12, 3, logw_prev=prev)
    for k in ("tv", "lse", "lp", "bonus", "tokens"):
        assert np.array_equal(g[k], g0[k]), k
    fin = np.isfinite(phi)
    assert np.allclose((g["logw"] - g0["logw"])[fin], phi[fin], atol=1e-12, rtol=0)


def test_bonus_block_near_tie_settled_in_fp64():
    """The bonus row's two live blocks tie to fp32 precision after their block
    noise: the leader must settle the block in fp64, as the oracle does."""
    from oracle.philox import STREAM_BONUS_BLOCK, gumbel_from_uniform, stream_words, uniform_from_bits
    B, N, K, V = 1, 8, 1, 256
    rng = np.random.default_rng(77)
    zT = rng.standard_normal((B, N, K + 1, V)).astype(np.float32)
    for n in range(N):
        gam = gumbel_from_uniform(uniform_from_bits(stream_words(6, 2, STREAM_BONUS_BLOCK, n, 2)))
        zT[0, n, K, :128] = 0.5
        zT[0, n, K, 128:] = np.float32(0.5 + (gam[0] - gam[1]))
    zD = zT.copy()
    x = rng.integers(0, V, size=(B, N, K)).astype(np.int32)
    g = run_score(zT, zD, x, 1.0, 6, 2, dtype="f32")
    o = oracle.smcsd_score(zT, zD, x, 1.0, 6, 2)
    compare(g, o, "bonus-near-tie")
