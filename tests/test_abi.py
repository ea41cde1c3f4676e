"""The C-ABI library loads and exports every symbol include/smcsd.h declares (no GPU)."""

import ctypes
import os
import re
import subprocess

import pytest

import resample_online_log_b200 as lib

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def declared_symbols():
    text = open(os.path.join(ROOT, "include", "smcsd.h")).read()
    return sorted(set(re.findall(r"SMCSD_API\s+[\w\s\*]+?\b(\w+)\(", text)))


def test_header_declares_the_entry_points():
    syms = declared_symbols()
    assert set(syms) == set(lib.EXPORTS), syms


def test_library_exports_every_declared_symbol():
    assert os.path.exists(lib.LIB_PATH), "build libsmcsd.so first (__graft_entry__.build())"
    out = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                         text=True, check=True).stdout
    exported = {line.split()[-1] for line in out.splitlines() if " T " in line}
    for s in declared_symbols():
        assert s in exported, s
    L = lib.load()
    for s in declared_symbols():
        assert hasattr(L, s)


def test_status_strings_and_version():
    assert lib.status_string(lib.SD_OK) == "ok"
    assert "invalid" in lib.status_string(lib.SD_ERR_INVALID_ARG)
    assert lib.version() >= 200


def test_host_argument_checks_need_no_gpu():
    L = lib.load()
    vp = ctypes.c_void_p
    # N = 0 -> invalid before anything touches CUDA
    assert L.smcsd_score(vp(1), vp(1), 1, 1, 0, 1, 10, 10, vp(1), 1.0, 0, 0, None, None, vp(1), vp(1),
                         None, None, None, None, None, None) == lib.SD_ERR_INVALID_ARG
    # tau <= 0, ld < V
    assert L.smcsd_score(vp(1), vp(1), 1, 1, 1, 1, 10, 10, vp(1), 0.0, 0, 0, None, None, vp(1), vp(1),
                         None, None, None, None, None, None) == lib.SD_ERR_INVALID_ARG
    assert L.smcsd_score(vp(1), vp(1), 1, 1, 1, 1, 10, 9, vp(1), 1.0, 0, 0, None, None, vp(1), vp(1),
                         None, None, None, None, None, None) == lib.SD_ERR_INVALID_ARG
    # B = 0 is an empty batch: OK, nothing enqueued
    assert L.smcsd_score(None, None, 1, 0, 1, 1, 10, 10, None, 1.0, 0, 0, None, None, None, None,
                         None, None, None, None, None, None) == lib.SD_OK
    # missing required outputs
    assert L.smcsd_score(vp(1), vp(1), 1, 1, 1, 1, 10, 10, vp(1), 1.0, 0, 0, None, None, None, vp(1),
                         None, None, None, None, None, None) == lib.SD_ERR_INVALID_ARG
    assert L.smcsd_resample(vp(1), 1, 0, 0, 0, None, None, vp(1), None, None) == lib.SD_ERR_INVALID_ARG
    assert L.smcsd_resample(vp(1), 1, 9000, 0, 0, None, None, vp(1), None, None) == lib.SD_ERR_UNSUPPORTED
    for bad_frac in (float("nan"), -0.5):                           # ess_frac not >= 0
        assert L.smcsd_resample_adaptive(vp(1), 1, 4, bad_frac, 0, 0, None, None, vp(1), None,
                                         None, None, None) == lib.SD_ERR_INVALID_ARG
    assert L.smcsd_resample_adaptive(vp(1), 1, 9000, 0.5, 0, 0, None, None, vp(1), None, None,
                                     None, None) == lib.SD_ERR_UNSUPPORTED
    assert L.smcsd_resample_adaptive(None, 0, 4, 0.5, 0, 0, None, None, None, None, None, None,
                                     None) == lib.SD_OK                 # empty batch
    assert L.kv_pagetable_remap(vp(16), vp(16), 1, 1, 4, vp(16), vp(1), 2, None, None, 0, None,
                                None) == lib.SD_ERR_INVALID_ARG     # tok_in without tok_out
    assert L.kv_pagetable_remap(vp(16), vp(16), 1, 1, 4, vp(16), None, 0, None, None, 0, None,
                                None) == lib.SD_ERR_INVALID_ARG     # aliasing pt_in / pt_out
    assert L.kv_pagetable_remap(vp(16), vp(16), 1, 2, 4, vp(4096), vp(256), 3, vp(264), None, 0,
                                None, None) == lib.SD_ERR_INVALID_ARG  # overlapping tok_in / tok_out
    assert L.sd_verify_reject(vp(1), vp(1), 1, 1, 0, 10, 10, vp(1), 1.0, 0, 0, vp(1), vp(1), None,
                              None, None) == lib.SD_ERR_INVALID_ARG  # K = 0
    assert L.gumbel_topk(vp(1), 1, 1, 10, 10, 11, 1.0, 0, 0, vp(1), None, None, None,
                         None) == lib.SD_ERR_INVALID_ARG            # k > V
    assert L.gumbel_topk_sparse(vp(1), vp(1), 1, 10, 11, 1.0, 0, 0, vp(1), None,
                                None) == lib.SD_ERR_INVALID_ARG     # k > L
    assert L.sd_draft_sample(vp(1), 1, 4, 10, 10, 0.0, 0, 0, 0, vp(1), None, None,
                             None) == lib.SD_ERR_INVALID_ARG        # tau <= 0
    assert L.sd_metasd_ucb(vp(1), 2, None, vp(1), 1, 4, 2, 0, 2.0, vp(1), vp(1), vp(1), None,
                           None, None) == lib.SD_ERR_INVALID_ARG    # ld_tv < K
    assert L.sd_metasd_ucb(None, 0, None, vp(1), 1, 4, 2, 1, 2.0, vp(1), vp(1), vp(1), None,
                           None, None) == lib.SD_ERR_INVALID_ARG    # BE without accepted_len
    assert L.sd_metasd_ucb(vp(1), 4, None, vp(1), 1, 4, 2, 0, -1.0, vp(1), vp(1), vp(1), None,
                           None, None) == lib.SD_ERR_INVALID_ARG    # c < 0
    assert L.sd_metasd_ucb(vp(1), 4, None, vp(1), 1, 4, 2, 2, 2.0, vp(1), vp(1), vp(1), None,
                           None, None) == lib.SD_ERR_INVALID_ARG    # unknown reward kind
    assert L.sd_metasd_ucb(None, 0, None, None, 0, 4, 2, 0, 2.0, None, None, None, None, None,
                           None) == lib.SD_OK                        # empty batch
    assert L.ngram_table_bytes(1000, 10) == 0 and L.ngram_table_bytes(16, 10) == 0   # not 2^j >= 32
    assert L.ngram_table_bytes(1024, 10) == 1024 * (8 + 4 + 80)
    assert L.ngram_table_bytes(1024, 17) == 0
    assert L.ngram_workspace_bytes(16385) == 0 and L.ngram_workspace_bytes(100) == 4 * 202
    assert L.ngram_table_clear(vp(16), 1000, 10, None) == lib.SD_ERR_INVALID_ARG
    assert L.ngram_store_update(vp(16), 1024, 10, vp(16), 4, vp(16), vp(16), 5, vp(16), 1 << 20,
                                None, None) == lib.SD_ERR_INVALID_ARG   # n > 3
    assert L.ngram_store_update(vp(16), 1024, 10, vp(16), 2, vp(16), vp(16), 5, vp(16), 40,
                                None, None) == lib.SD_ERR_INVALID_ARG   # workspace too small
    assert L.ngram_store_update(vp(16), 1024, 10, vp(16), 2, vp(16), vp(16), 20000, vp(16), 1 << 20,
                                None, None) == lib.SD_ERR_UNSUPPORTED
    assert L.ngram_store_update(vp(16), 1024, 10, None, 2, None, None, 0, None, 0, None,
                                None) == lib.SD_OK                      # empty batch
    assert L.ngram_store_lookup(vp(8), 1024, 10, vp(16), 2, 3, vp(16), vp(16), None, None,
                                None) == lib.SD_ERR_INVALID_ARG         # table not 16-byte aligned
    assert L.ngram_observe_topk(vp(16), 1, 4, 10, 10, None, 5, 10, 1.0, vp(16), vp(16), None,
                                None) == lib.SD_ERR_INVALID_ARG         # U > rows without row_ids
    assert L.ngram_observe_topk(vp(16), 1, 4, 10, 10, None, 4, 17, 1.0, vp(16), vp(16), None,
                                None) == lib.SD_ERR_INVALID_ARG         # k > 16
    assert L.sd_draft_sample(vp(1), 1, 4, 10, 10, 1.0, 0, 0, 0xFFFFFFFE, vp(1), None, None,
                             None) == lib.SD_ERR_INVALID_ARG        # row ids past 2^32
    assert L.sd_draft_sample(None, 1, 0, 10, 10, 1.0, 0, 0, 0, None, None, None,
                             None) == lib.SD_OK                     # no rows: nothing to do


def test_product_path_has_no_oracle_dependency():
    pkg = os.path.join(ROOT, "resample_online_log_b200")
    for dirpath, _, files in os.walk(pkg):
        for f in files:
            if f.endswith((".py", ".cu", ".cuh", ".h")):
                text = open(os.path.join(dirpath, f)).read()
                assert "import oracle" not in text and "from oracle" not in text, f


def test_binding_rejects_a_bad_error_word():
    """The error word is written by the kernels: a host tensor or a wrong dtype or
    size is refused before the library is called."""
    import torch
    with pytest.raises(ValueError):
        lib._check_err(torch.zeros((1,), dtype=torch.int32))          # not on a GPU
    with pytest.raises(ValueError):
        lib._check_err(torch.zeros((2,), dtype=torch.int32))
    with pytest.raises(ValueError):
        lib._check_err(torch.zeros((1,), dtype=torch.float32))
    lib._check_err(None)


def test_testing_library_exports_its_probes():
    """libsmcsd_testing.so (built beside the library, used by the GPU pins only)
    exports the device-generator probes; libsmcsd.so does not."""
    tl = os.path.join(os.path.dirname(lib.LIB_PATH), "libsmcsd_testing.so")
    assert os.path.exists(tl), "build the libraries first (__graft_entry__.build())"
    names = subprocess.run(["nm", "-D", "--defined-only", tl], capture_output=True, text=True,
                           check=True).stdout
    syms = {line.split()[-1] for line in names.splitlines() if line.strip()}
    assert {"smcsd_testing_philox", "smcsd_testing_stream", "smcsd_testing_wait"} <= syms
    main = subprocess.run(["nm", "-D", "--defined-only", lib.LIB_PATH], capture_output=True,
                          text=True, check=True).stdout
    assert "smcsd_testing" not in main
