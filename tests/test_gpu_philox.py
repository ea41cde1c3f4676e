"""The library's device Philox4x32-10 against the oracle's NumPy implementation
(written separately from the SC'11 definition) on 10^6 counters, against the
published known-answer vectors, and the counter layout of a stream against the
oracle's stream_words.  The device code runs from libsmcsd_testing.so, built
from the same header the sampling kernels include."""

import ctypes
import os

import numpy as np
import pytest
import torch

from oracle import philox
from tests.parity import requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(os.path.dirname(HERE), "resample_online_log_b200", "libsmcsd_testing.so")


def _lib():
    L = ctypes.CDLL(LIB)
    vp = ctypes.c_void_p
    L.smcsd_testing_philox.argtypes = [vp, vp, ctypes.c_int, ctypes.c_int, vp, vp]
    L.smcsd_testing_stream.argtypes = [ctypes.c_uint64, ctypes.c_uint64, ctypes.c_uint32,
                                       ctypes.c_uint32, ctypes.c_int, vp, vp]
    return L


def _device_words(ctr, key, variant):
    n = ctr.shape[0]
    c = torch.from_numpy(ctr.astype(np.uint32).view(np.int32)).cuda()
    k = torch.from_numpy(key.astype(np.uint32).view(np.int32)).cuda()
    out = torch.empty((n, 4), dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert _lib().smcsd_testing_philox(ctypes.c_void_p(c.data_ptr()), ctypes.c_void_p(k.data_ptr()),
                                       n, variant, ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(st)) == 0
    torch.cuda.synchronize()
    return out.cpu().numpy().view(np.uint32)


@pytest.mark.parametrize("variant", [0, 1])
def test_device_philox_matches_numpy_on_a_million_counters(variant):
    rng = np.random.default_rng(2024)
    n = 1_000_000
    ctr = rng.integers(0, 2 ** 32, size=(n, 4), dtype=np.uint64)
    key = rng.integers(0, 2 ** 32, size=(n, 2), dtype=np.uint64)
    ctr[:1000, 1:] = 0            # small counters as the kernels use them
    ctr[:1000, 0] = np.arange(1000)
    got = _device_words(ctr, key, variant)
    ref = np.stack(philox.philox4x32_10(ctr[:, 0], ctr[:, 1], ctr[:, 2], ctr[:, 3],
                                        key[:, 0], key[:, 1]), axis=1).astype(np.uint32)
    assert np.array_equal(got, ref)


@pytest.mark.parametrize("variant", [0, 1])
def test_device_philox_known_answer_vectors(variant):
    rows = []
    with open(os.path.join(HERE, "golden", "philox4x32_10_kat.txt")) as f:
        for line in f:
            line = line.strip()
            if line and not line.startswith("#"):
                rows.append([int(t, 16) for t in line.split()])
    kat = np.array(rows, dtype=np.uint64)
    got = _device_words(kat[:, 0:4], kat[:, 4:6], variant)
    assert np.array_equal(got, kat[:, 6:10].astype(np.uint32))


@pytest.mark.parametrize("seed,rnd,tag,row", [(0, 0, 1, 0), (4, 7, 5, 4095),
                                              (2 ** 64 - 1, 2 ** 40 + 3, 3, 767),
                                              (123456789, 1, 6, 0)])
def test_device_stream_layout_matches_oracle(seed, rnd, tag, row):
    nblocks = 38016  # a 152064-entry row
    out = torch.empty((nblocks, 4), dtype=torch.int32, device="cuda")
    st = torch.cuda.current_stream().cuda_stream
    assert _lib().smcsd_testing_stream(seed, rnd, tag, row, nblocks, ctypes.c_void_p(out.data_ptr()),
                                       ctypes.c_void_p(st)) == 0
    torch.cuda.synchronize()
    got = out.cpu().numpy().view(np.uint32).reshape(-1)
    ref = philox.stream_words(seed, rnd, tag, row, 4 * nblocks).astype(np.uint32)
    assert np.array_equal(got, ref)
