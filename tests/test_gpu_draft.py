"""GPU parity of sd_draft_sample (the draft step's two-level Gumbel-max sampler)
against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import resample_online_log_b200 as lib
import synth
from synth import device as sdev
from synth import gen
from tests.parity import bf16_dev, close, discrete, requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def run_draft(zD_dev, tau, seed, rnd, row0=0):
    rows = zD_dev.shape[0]
    tok = torch.empty((rows,), dtype=torch.int32, device="cuda")
    lq = torch.empty((rows,), dtype=torch.float32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.sd_draft_sample(zD_dev, tau, seed, rnd, tok, logq_out=lq, row0=row0, dev_err=err)
    torch.cuda.synchronize()
    return tok, lq, int(err.item())


@pytest.mark.parametrize("V,tau,dtype,row0", [(1000, 1.0, "bf16", 0), (33001, 0.7, "bf16", 5),
                                              (7, 1.3, "f32", 0), (40000, 0.9, "f32", 1000)])
def test_draft_random_rows(V, tau, dtype, row0):
    rng = np.random.default_rng(V)
    z = (rng.standard_normal((12, V)) * 3).astype(np.float32)
    if dtype == "bf16":
        z = gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(z))
        d = bf16_dev(z)
    else:
        d = to_dev(z)
    tok, lq, err = run_draft(d, tau, 7, 3, row0)
    o = oracle.sd_draft_sample(z, tau, 7, 3, row0=row0)
    discrete(tok.cpu().numpy(), o["tokens"], o["margin"], f"draft{V}.tokens")
    same = tok.cpu().numpy() == o["tokens"]
    close(lq.cpu().numpy()[same], o["logq"][same], 1e-5, f"draft{V}.logq")
    assert err == o["err"] == 0


def test_draft_masked_and_bad_rows():
    z = np.full((4, 500), -np.inf, dtype=np.float32)
    z[0, [3, 250, 499]] = [1.0, 0.5, 2.0]
    z[1, 10] = np.nan
    z[2, :] = 0.0
    z[2, 77] = np.inf
    z[3, :] = 1.5
    tok, lq, err = run_draft(to_dev(z), 1.0, 2, 9)
    o = oracle.sd_draft_sample(z, 1.0, 2, 9)
    assert np.array_equal(tok.cpu().numpy(), o["tokens"])
    assert err == o["err"] == oracle.DEV_NONFINITE
    assert tok[0].item() in (3, 250, 499) and tok[1].item() == -1 and tok[2].item() == -1


def test_draft_config_rows_sampled():
    """The smc_batch draft rows of one position (64 x 16 particles, V = 128256
    bf16): all rows on the GPU, 16 sampled rows against the oracle, and on every
    row logq = the row's log-softmax at the drawn token (fp64 reference)."""
    cfg = synth.CONFIGS["smc_batch"]
    d = sdev.gen_config_device(cfg)
    zD = d["zD"][:, :, 0, :].reshape(cfg.B * cfg.N, cfg.V)
    tok, lq, err = run_draft(zD, cfg.tau, cfg.seed, 11, row0=0)
    assert err == 0
    t = tok.long()
    assert bool(((t >= 0) & (t < cfg.V)).all())
    tau = float(np.float32(cfg.tau))
    ref = torch.cat([(zD[r0:r0 + 128].double() / tau).log_softmax(dim=1)
                     .gather(1, t[r0:r0 + 128, None])[:, 0] for r0 in range(0, zD.shape[0], 128)])
    assert float((lq.double() - ref).abs().max()) <= 1e-5
    rows = np.random.default_rng(0).choice(zD.shape[0], 16, replace=False)
    h = gen.gen_config_rows(cfg, seqs=np.unique(rows // cfg.N))
    for r in rows:
        b, n = divmod(int(r), cfg.N)
        seq_pos = int(np.where(np.unique(rows // cfg.N) == b)[0][0])
        zr = h["zD"][seq_pos, n, 0][None, :]
        assert np.array_equal(zr, zD[r].float().cpu().numpy()[None, :])
        o = oracle.sd_draft_sample(zr, cfg.tau, cfg.seed, 11, row0=int(r))
        discrete(tok[r:r + 1].cpu().numpy(), o["tokens"], o["margin"], f"draft_row{r}")


@pytest.mark.parametrize("V", [1, 128, 129, 256, 300])
def test_draft_block_boundaries(V):
    rng = np.random.default_rng(V + 3)
    z = (rng.standard_normal((40, V)) * 2).astype(np.float32)
    tok, lq, err = run_draft(to_dev(z), 0.9, 1, 2)
    o = oracle.sd_draft_sample(z, 0.9, 1, 2)
    discrete(tok.cpu().numpy(), o["tokens"], o["margin"], f"draft{V}")
    assert err == 0


def test_draft_nan_behind_masked_entries():
    z = np.zeros((2, 2000), dtype=np.float32)
    z[0, 0] = np.nan
    z[0, 1:8] = -np.inf
    z[1, 520] = np.nan                     # second tile of a warp, first one masked
    z[1, 512:520] = -np.inf
    tok, lq, err = run_draft(to_dev(z), 1.0, 3, 3)
    assert err == oracle.DEV_NONFINITE and tok.cpu().tolist() == [-1, -1]


def test_draft_block_near_tie_settled_in_fp64():
    """Two live blocks whose perturbed log-masses coincide to fp32 precision:
    the fp32 bounds cannot settle the block, the fp64 path must, as the oracle."""
    from oracle.philox import STREAM_DRAFT_BLOCK, gumbel_from_uniform, stream_words, uniform_from_bits
    rows, V = 16, 256
    z = np.zeros((rows, V), dtype=np.float32)
    for r in range(rows):
        gam = gumbel_from_uniform(uniform_from_bits(stream_words(5, 8, STREAM_DRAFT_BLOCK, r, 2)))
        z[r, :128] = 1.0
        z[r, 128:] = np.float32(1.0 + (gam[0] - gam[1]))   # lambda_1 + G_1 ~= lambda_0 + G_0
    tok, lq, err = run_draft(to_dev(z), 1.0, 5, 8)
    o = oracle.sd_draft_sample(z, 1.0, 5, 8)
    discrete(tok.cpu().numpy(), o["tokens"], o["margin"], "near-tie")
    assert err == 0 and bool((tok >= 0).all())
