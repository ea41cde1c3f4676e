"""The kernels' bounded mbarrier wait (bounded_wait, used by every wait of the
SMC-SD score kernel) on the GPU, run from libsmcsd_testing.so on a barrier that
nothing completes: the wait must give up after its limit, set the CTA's abort
flag and report SD_DEV_TIMEOUT with its site bits, without any fault; an
abortable wait must return at once once the flag is set; a barrier completed
in time must end the wait without an error."""

import ctypes
import os

import pytest
import torch

import resample_online_log_b200 as lib
from tests.parity import requires_gpu

pytestmark = [pytest.mark.gpu, requires_gpu]

HERE = os.path.dirname(os.path.abspath(__file__))
LIB = os.path.join(os.path.dirname(HERE), "resample_online_log_b200", "libsmcsd_testing.so")
SITE = 1 << 8
ABORT, ABORTABLE, ARRIVE = 1, 2, 4


def run_wait(limit_ns, mode, delay_ns=0):
    L = ctypes.CDLL(LIB)
    L.smcsd_testing_wait.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_uint64,
                                     ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
    err = torch.zeros((1,), dtype=torch.int32, device="cuda")
    out = torch.zeros((2,), dtype=torch.int64, device="cuda")
    s = torch.cuda.current_stream()
    assert L.smcsd_testing_wait(limit_ns, mode, delay_ns, ctypes.c_void_p(err.data_ptr()),
                                ctypes.c_void_p(out.data_ptr()), ctypes.c_void_p(s.cuda_stream)) == 0
    torch.cuda.synchronize()
    o = out.cpu().tolist()
    return int(err.item()), o[0], o[1]


@pytest.mark.parametrize("mode", [0, ABORTABLE])
def test_wait_runs_out_and_reports(mode):
    err, took, flag = run_wait(2_000_000, mode)       # 2 ms, nothing arrives
    assert err == lib.DEV_TIMEOUT | SITE
    assert flag == 1
    assert 2_000_000 <= took < 200_000_000


def test_abortable_wait_returns_once_the_cta_gave_up():
    err, took, flag = run_wait(500_000_000, ABORT | ABORTABLE)
    assert err == 0 and flag == 1 and took < 5_000_000


def test_copy_ordering_wait_ignores_the_abort_flag():
    err, took, _ = run_wait(2_000_000, ABORT)         # not abortable: waits out its own limit
    assert err == lib.DEV_TIMEOUT | SITE and took >= 2_000_000


def test_wait_completed_in_time():
    err, took, flag = run_wait(500_000_000, ABORTABLE | ARRIVE, delay_ns=1_000_000)
    assert err == 0 and flag == 0
    assert 1_000_000 <= took < 100_000_000
    # the context is still usable after a wait ran out
    run_wait(1_000_000, 0)
    x = torch.arange(10, device="cuda").sum()
    assert int(x.item()) == 45
