"""GPU parity of sd_metasd_ucb (per-sequence UCB drafter selection with the
Block Divergence / Block Efficiency reward) against the oracle, through the C ABI."""

import numpy as np
import pytest
import torch

import oracle
import resample_online_log_b200 as lib
from tests.parity import requires_gpu, to_dev

pytestmark = [pytest.mark.gpu, requires_gpu]


def gpu_round(tv, acc, arm, pulls, sums, K, kind, c, alias=False):
    B = pulls.shape[0]
    arm_d = to_dev(np.asarray(arm, np.int32))
    out = arm_d if alias else torch.empty((B,), dtype=torch.int32, device="cuda")
    rew = torch.empty((B,), dtype=torch.float64, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    lib.sd_metasd_ucb(arm_d, pulls, sums, out, K, tv=None if tv is None else to_dev(tv),
                      accepted_len=None if acc is None else to_dev(np.asarray(acc, np.int32)),
                      reward_kind=kind, c=c, reward_out=rew, dev_err=err)
    torch.cuda.synchronize()
    return out.cpu().numpy(), rew.cpu().numpy(), int(err.item())


@pytest.mark.parametrize("B,M,K,kind,c", [(1, 2, 4, lib.REWARD_BD, 2.0), (300, 5, 4, lib.REWARD_BD, 2.0),
                                          (64, 8, 6, lib.REWARD_BE, 2.0), (17, 33, 3, lib.REWARD_BD, 0.5),
                                          (200, 3, 5, lib.REWARD_BE, 0.0)])
def test_bandit_rounds_parity(B, M, K, kind, c):
    rng = np.random.default_rng(B * 31 + M)
    means = rng.uniform(0.1, 0.9, size=(B, M))
    pulls_d = torch.zeros((B, M), dtype=torch.int32, device="cuda")
    sums_d = torch.zeros((B, M), dtype=torch.float64, device="cuda")
    pulls, sums = np.zeros((B, M), np.int64), np.zeros((B, M))
    arm = np.full(B, -1)
    for rnd in range(60):
        a = np.maximum(arm, 0)
        mu = means[np.arange(B), a]
        tv = np.clip(1.0 - mu[:, None] + rng.normal(0, 0.1, (B, K + 1)), 0, 1).astype(np.float32)
        acc = rng.binomial(K, mu).astype(np.int32)
        g_arm, g_rew, g_err = gpu_round(tv, acc, arm, pulls_d, sums_d, K, kind, c)
        o = oracle.metasd_ucb_step(tv, acc, arm, pulls, sums, K, c=c, kind=kind)
        assert g_err == o["err"] == 0
        assert np.array_equal(pulls_d.cpu().numpy(), o["pulls"])
        # the reward is summed in the same order on both sides: equal bits
        assert np.array_equal(sums_d.cpu().numpy(), o["sums"])
        assert np.array_equal(np.isnan(g_rew), np.isnan(o["reward"]))
        assert np.array_equal(g_rew[~np.isnan(g_rew)], o["reward"][~np.isnan(o["reward"])])
        # the arm: exact unless two UCB indices are within rounding of each other
        sure = o["gap"] > 1e-12
        assert np.array_equal(g_arm[sure], o["arm"][sure]), rnd
        pulls, sums, arm = o["pulls"], o["sums"], g_arm.astype(np.int64)


def test_bandit_faults_and_alias():
    B, M, K = 4, 3, 2
    pulls_d = torch.ones((B, M), dtype=torch.int32, device="cuda")
    sums_d = torch.full((B, M), 0.5, dtype=torch.float64, device="cuda")
    tv = np.array([[np.nan, 0.1, 0], [0.1, 0.1, 0], [0.2, 0.2, 0], [0.0, 0.0, 0]], np.float32)
    arm = np.array([0, 3, -2, 1])
    g_arm, g_rew, g_err = gpu_round(tv, None, arm, pulls_d, sums_d, K, lib.REWARD_BD, 2.0, alias=True)
    o = oracle.metasd_ucb_step(tv, np.zeros(B, int), arm, np.ones((B, M), int), np.full((B, M), 0.5), K)
    assert g_err == o["err"] == lib.DEV_NONFINITE | lib.DEV_ARM_OOB
    assert np.array_equal(pulls_d.cpu().numpy(), o["pulls"])
    assert np.array_equal(sums_d.cpu().numpy(), o["sums"])
    assert np.array_equal(g_arm, o["arm"])
    assert np.isnan(g_rew[:3]).all() and g_rew[3] == 1.0
    # BE with an accepted length outside [0, K]
    g_arm, g_rew, g_err = gpu_round(None, [K + 1, 0, 0, 0], [0, -1, -1, -1], pulls_d, sums_d, K,
                                    lib.REWARD_BE, 2.0)
    assert g_err == lib.DEV_NONFINITE and np.isnan(g_rew).all()


def test_bandit_after_verification():
    """One MetaSD loop on the GPU: verification of the chosen drafter's block
    gives per-position TV and the accepted length; the bandit credits them."""
    rng = np.random.default_rng(3)
    B, K, V, M = 8, 4, 2000, 3
    zT = torch.from_numpy(rng.standard_normal((B, K + 1, V)).astype(np.float32) * 2).cuda()
    noise = [0.2, 1.0, 3.0]              # drafter m's logits = target + noise_m
    pulls = torch.zeros((B, M), dtype=torch.int32, device="cuda")
    sums = torch.zeros((B, M), dtype=torch.float64, device="cuda")
    arm = torch.full((B,), -1, dtype=torch.int32, device="cuda")
    tv = torch.empty((B, K), dtype=torch.float32, device="cuda")
    acc = torch.empty((B,), dtype=torch.int32, device="cuda")
    toks = torch.empty((B, K + 1), dtype=torch.int32, device="cuda")
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    for rnd in range(40):
        lib.sd_metasd_ucb(arm, pulls, sums, arm, K, tv=tv, reward_kind=lib.REWARD_BD, c=0.5,
                          dev_err=err)
        a = arm.cpu().numpy()
        zD = torch.stack([zT[b, :K] + noise[a[b]] * torch.from_numpy(
            rng.standard_normal((K, V)).astype(np.float32)).cuda() for b in range(B)])
        x = torch.from_numpy(rng.integers(0, V, (B, K)).astype(np.int32)).cuda()
        lib.sd_verify_reject(zT, zD.contiguous(), x, 1.0, 9, rnd, acc, toks, tv_out=tv, dev_err=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    p = pulls.cpu().numpy()
    assert np.all(p.sum(axis=1) == 39)
    assert np.all(p[:, 0] >= p[:, 1]) and np.all(p[:, 0] > p[:, 2])
