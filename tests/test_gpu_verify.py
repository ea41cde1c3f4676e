"""GPU parity of sd_verify_reject against the oracle."""

import numpy as np
import pytest
import torch

import oracle
import resample_online_log_b200 as lib
import synth
from synth import gen
from tests.parity import TOL_TV, bf16_dev, close, discrete, requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def run_verify(zT, zD, x, tau, seed, rnd, dtype="bf16"):
    B, R, V = zT.shape
    K = R - 1
    if dtype == "bf16":
        t, d = bf16_dev(zT), bf16_dev(zD)
    else:
        t, d = to_dev(zT.astype(np.float32)), to_dev(zD.astype(np.float32))
    acc = torch.empty((B,), dtype=torch.int32, device="cuda")
    out = torch.empty((B, R), dtype=torch.int32, device="cuda")
    tv = torch.empty((B, K), dtype=torch.float32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.sd_verify_reject(t, d, to_dev(np.asarray(x, dtype=np.int32)), tau, seed, rnd, acc, out,
                         tv_out=tv, dev_err=err)
    torch.cuda.synchronize()
    return dict(acc=acc.cpu().numpy(), out=out.cpu().numpy(), tv=tv.cpu().numpy(),
                err=int(err.item()))


def compare(g, o, name):
    close(g["tv"], o["tv"], TOL_TV, name + ".tv")
    # accepted length: exempt when any accept decision it depends on is a near-tie
    acc_margin = np.min(np.where(np.isfinite(o["accept_margin"]), o["accept_margin"], np.inf), axis=1)
    discrete(g["acc"], o["accepted_len"], acc_margin, name + ".accepted_len")
    same = g["acc"] == o["accepted_len"]
    m = np.minimum(acc_margin, o["token_margin"])[:, None]
    discrete(g["out"][same], o["out_tokens"][same], np.broadcast_to(m, g["out"].shape)[same],
             name + ".out_tokens")
    assert g["err"] == o["err"], (g["err"], o["err"])


def test_verify_config_full():
    cfg = synth.CONFIGS["verify"]
    h = gen.gen_config_rows(cfg)
    g = run_verify(h["zT"], h["zD"], h["draft"], cfg.tau, cfg.seed, 0)
    o = oracle.sd_verify_reject(h["zT"], h["zD"], h["draft"], cfg.tau, cfg.seed, 0)
    compare(g, o, "verify")
    hist = np.stack([np.bincount(g["acc"][lo:hi], minlength=cfg.K + 1)
                     for lo, hi in ((0, 43), (43, 86), (86, 128))])
    print("accepted-length histogram by draft-noise third:\n", hist)


@pytest.mark.parametrize("V,K,tau,noise", [(1001, 3, 1.0, 1.0), (32000, 5, 0.7, 2.0),
                                           (128256, 2, 1.0, 3.0), (9, 4, 1.0, 0.5)])
def test_verify_random(V, K, tau, noise):
    rng = np.random.default_rng(V + K)
    B = 24
    zT = (rng.standard_normal((B, K + 1, V)) * 2).astype(np.float32)
    zD = (zT[:, :K] + rng.standard_normal((B, K, V)) * noise).astype(np.float32)
    zT = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(zT))
    zD = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(zD))
    # draft tokens from q (host sampler of the test; any valid ids would do)
    zd64 = zD.astype(np.float64) / tau
    q = np.exp(zd64 - zd64.max(axis=-1, keepdims=True))
    q /= q.sum(axis=-1, keepdims=True)
    x = np.array([[rng.choice(V, p=q[b, k]) for k in range(K)] for b in range(B)], dtype=np.int32)
    g = run_verify(zT, zD, x, tau, 3, V)
    o = oracle.sd_verify_reject(zT, zD, x, tau, 3, V)
    compare(g, o, f"verify{V}")


def test_verify_fp32_and_faults():
    rng = np.random.default_rng(5)
    B, K, V = 6, 3, 3000
    zT = (rng.standard_normal((B, K + 1, V)) * 2).astype(np.float32)
    zD = (zT[:, :K] + rng.standard_normal((B, K, V))).astype(np.float32)
    x = rng.integers(0, V, size=(B, K)).astype(np.int32)
    x[1, 0] = -5
    zT[2, 1, 10] = np.inf
    zD[3] = zT[3, :K]                # identical rows: everything accepted
    g = run_verify(zT, zD, x, 1.0, 8, 1, dtype="f32")
    o = oracle.sd_verify_reject(zT, zD, x, 1.0, 8, 1)
    compare(g, o, "verify_faults")
    assert g["acc"][3] == K
