"""Helpers for GPU-vs-oracle parity checks.

Parity rule: continuous outputs within fixed absolute tolerances; discrete
outputs (token ids, ancestors, accepted lengths) bit-exact except decisions
whose oracle margin is below 1e-6, which are reported and must stay under
0.01% of the decisions compared.
"""

import numpy as np
import pytest
import torch

MARGIN_EXEMPT = 1e-6
EXEMPT_FRACTION = 1e-4
TOL_LOGW = 1e-4
TOL_TV = 1e-5
TOL_LSE = 1e-5

requires_gpu = pytest.mark.skipif(not torch.cuda.is_available(), reason="needs a CUDA GPU")


def discrete(gpu, ora, margin, name):
    """Asserts bit-exact discrete outputs up to exempt near-ties; returns #exempt."""
    gpu = np.asarray(gpu)
    ora = np.asarray(ora)
    margin = np.broadcast_to(np.asarray(margin, dtype=np.float64), ora.shape)
    assert gpu.shape == ora.shape, (name, gpu.shape, ora.shape)
    mism = gpu != ora
    bad = mism & ~(margin < MARGIN_EXEMPT)
    if bad.any():
        where = np.argwhere(bad)[:10]
        details = [(tuple(w), int(gpu[tuple(w)]), int(ora[tuple(w)]), float(margin[tuple(w)]))
                   for w in where]
        raise AssertionError(f"{name}: {int(bad.sum())} mismatches beyond the margin rule: {details}")
    exempt = int((mism & (margin < MARGIN_EXEMPT)).sum())
    assert exempt <= EXEMPT_FRACTION * mism.size, f"{name}: {exempt} exempt near-ties of {mism.size}"
    if exempt:
        print(f"[parity] {name}: {exempt} exempt near-tie decisions of {mism.size}")
    return exempt


def close(gpu, ora, tol, name):
    gpu = np.asarray(gpu, dtype=np.float64)
    ora = np.asarray(ora, dtype=np.float64)
    assert gpu.shape == ora.shape, (name, gpu.shape, ora.shape)
    nan_g, nan_o = np.isnan(gpu), np.isnan(ora)
    assert np.array_equal(nan_g, nan_o), f"{name}: NaN pattern differs"
    d = np.abs(gpu - ora)[~nan_o]
    worst = float(d.max()) if d.size else 0.0
    assert worst <= tol, f"{name}: max |diff| {worst:.3e} > {tol:.1e}"
    return worst


def to_dev(a, dtype=None, device="cuda"):
    t = torch.from_numpy(np.ascontiguousarray(a))
    if dtype is not None:
        t = t.to(dtype)
    return t.to(device)


def bf16_dev(a_f32, device="cuda"):
    """Host fp32 array holding bf16-exact values -> device bf16 tensor (exact)."""
    t = torch.from_numpy(np.ascontiguousarray(a_f32, dtype=np.float32))
    bt = t.to(torch.bfloat16)
    back = bt.to(torch.float32)
    same = (back == t) | (torch.isnan(back) & torch.isnan(t))
    assert bool(same.all()), "values are not bf16-exact"
    return bt.to(device)
