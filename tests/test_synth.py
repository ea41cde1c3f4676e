"""The synthetic input recipes: host determinism, shape of the data, and (GPU) the
device generator produces the same bytes as the host generator."""

import numpy as np
import pytest
import torch

import synth
from synth import gen
from tests.parity import requires_gpu


def test_host_generator_deterministic_and_peaked():
    cfg = synth.CONFIGS["smc_small"]
    a = gen.gen_config_rows(cfg, seqs=[0])
    b = gen.gen_config_rows(cfg, seqs=[0])
    assert np.array_equal(a["zT"], b["zT"]) and np.array_equal(a["draft"], b["draft"])
    z = a["zT"][0, 0].astype(np.float64)
    p = np.exp(z - z.max(axis=1, keepdims=True))
    p /= p.sum(axis=1, keepdims=True)
    assert np.all(p.max(axis=1) > 0.5)               # Zipf head carries most of the mass
    body = np.sort(z, axis=1)[:, :-50]
    assert abs(body.std() - 2.0) < 0.1 and abs(body.mean()) < 0.1


def test_head_positions_distinct_and_in_range():
    pos, rank = gen.head_positions(3, np.arange(20), 128256, 50)
    for r in range(20):
        assert len(set(pos[r])) == 50 and pos[r].max() < 128256
        assert sorted(rank[r]) == list(range(50))


def test_bf16_rounding_is_round_to_nearest_even():
    x = np.array([1.0, 1.00390625, 1.01171875, -2.5, 3.1415927, 1e-3], dtype=np.float32)
    ref = torch.from_numpy(x).to(torch.bfloat16).to(torch.float32).numpy()
    assert np.array_equal(gen.bf16_bits_to_f32(gen.f32_to_bf16_bits(x)), ref)


def test_synth_log_accuracy():
    x = np.float32(np.exp(np.linspace(-17, 3, 10001)))
    assert np.max(np.abs(gen.synth_log(x) - np.log(x.astype(np.float64)))) < 4e-6


def test_draft_tokens_follow_q():
    """The drafter stand-in samples x ~ softmax(zD / tau) (chi-square on a small row)."""
    from scipy import stats
    V, M = 12, 40000
    z = np.linspace(-1.5, 1.5, V).astype(np.float32)
    rows = np.arange(M)
    x = gen.draft_tokens_for_rows(9, rows, np.broadcast_to(z, (M, V)), 1.0)
    p = np.exp(z - z.max())
    p /= p.sum()
    _, pval = stats.chisquare(np.bincount(x, minlength=V), p * M)
    assert pval > 1e-3


@pytest.mark.gpu
@requires_gpu
@pytest.mark.parametrize("name", ["smc_small", "verify", "topk"])
def test_device_generator_matches_host(name):
    from synth import device
    cfg = synth.CONFIGS[name]
    if name == "topk":
        cfg = gen.SynthConfig(**{**cfg.__dict__, "B": 64})
    d = device.gen_config_device(cfg)
    seqs = [0, cfg.B - 1]
    h = gen.gen_config_rows(cfg, seqs=seqs)
    if name == "topk":
        assert np.array_equal(d["z"][seqs].float().cpu().numpy(), h["z"])
        return
    assert np.array_equal(d["zT"][seqs].float().cpu().numpy(), h["zT"])
    assert np.array_equal(d["zD"][seqs].float().cpu().numpy(), h["zD"])
    assert np.array_equal(d["draft"][seqs].cpu().numpy(), h["draft"])
