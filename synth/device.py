"""Device-side synthetic inputs (ctypes binding of synth/libsynth.so).

Builds the same bytes as ``synth.gen`` directly in GPU memory, for inputs that
are too large to build on the host (up to ~38 GB for the largest SMC-SD round).
"""

import ctypes
import os

import numpy as np
import torch

from . import gen

_HERE = os.path.dirname(os.path.abspath(__file__))
_LIB = None


def build(verbose=False):
    import subprocess
    src = os.path.join(_HERE, "csrc", "synth.cu")
    out = os.path.join(_HERE, "libsynth.so")
    cmd = ["nvcc", "-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo",
           "-Xcompiler", "-fPIC", "-shared", "--cudart", "static", "-Xlinker", "--exclude-libs,ALL",
           "-o", out, src]
    if verbose:
        print(" ".join(cmd))
    subprocess.check_call(cmd)
    return out


def lib():
    global _LIB
    if _LIB is None:
        path = os.path.join(_HERE, "libsynth.so")
        if not os.path.exists(path):
            raise RuntimeError("synth/libsynth.so is missing: run synth.device.build()")
        L = ctypes.CDLL(path)
        L.synth_rows.restype = ctypes.c_int
        L.synth_rows.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                 ctypes.c_int64, ctypes.c_float, ctypes.c_int, ctypes.c_void_p,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_int, ctypes.c_int,
                                 ctypes.c_void_p, ctypes.c_void_p, ctypes.c_void_p]
        L.synth_draft_tokens.restype = ctypes.c_int
        L.synth_draft_tokens.argtypes = [ctypes.c_uint64, ctypes.c_int, ctypes.c_int64, ctypes.c_int,
                                         ctypes.c_int, ctypes.c_int, ctypes.c_int, ctypes.c_int64,
                                         ctypes.c_float, ctypes.c_void_p, ctypes.c_void_p,
                                         ctypes.c_void_p]
        _LIB = L
    return _LIB


def _ptr(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream():
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def gen_config_device(cfg, device="cuda", ld=None):
    """Generate a whole config on the device.

    Returns dict of torch tensors: smc -> zT, zD [B,N,K+1,V(ld)], draft [B,N,K];
    verify -> zT [B,K+1,V], zD [B,K,V], draft [B,K]; topk -> z [B,V].
    Logit tensors are uint16 bf16 bit patterns (viewed as torch.bfloat16) or fp32.
    """
    V = cfg.V
    ld = V if ld is None else ld
    bf16 = cfg.dtype == "bf16"
    tdt = torch.bfloat16 if bf16 else torch.float32
    table = torch.from_numpy(gen.normal_table()).to(device)
    L = cfg.L_head
    boosts = torch.from_numpy(gen.head_boosts(max(L, 1), cfg.sigma_z, V)).to(device)
    lib_ = lib()
    if cfg.kind == "topk":
        z = torch.empty((cfg.B, ld), dtype=tdt, device=device)
        rc = lib_.synth_rows(cfg.seed, int(bf16), cfg.B, V, ld, float(np.float32(cfg.sigma_z)), L,
                             _ptr(boosts), _ptr(table), None, 1, 0, _ptr(z), None, _stream())
        assert rc == 0, rc
        return dict(z=z[:, :V] if ld != V else z)
    R, K = cfg.R, cfg.K
    units = cfg.B * (cfg.N if cfg.kind == "smc" else 1)
    Kd = R if cfg.kind == "smc" else K
    sig = torch.tensor([cfg.sigma_d_of_seq(b) for b in range(cfg.B) for _ in range(units // cfg.B)],
                       dtype=torch.float32, device=device)
    zT = torch.empty((units * R, ld), dtype=tdt, device=device)
    zD = torch.empty((units * Kd, ld), dtype=tdt, device=device)
    rc = lib_.synth_rows(cfg.seed, int(bf16), units * R, V, ld, float(np.float32(cfg.sigma_z)), L,
                         _ptr(boosts), _ptr(table), _ptr(sig), R, Kd, _ptr(zT), _ptr(zD), _stream())
    assert rc == 0, rc
    tok = torch.empty((units * K,), dtype=torch.int32, device=device)
    inv_tau = float(np.float32(1.0 / float(np.float32(cfg.tau))))
    rc = lib_.synth_draft_tokens(cfg.seed, int(bf16), units * K, K, R, Kd, V, ld, inv_tau, _ptr(zD),
                                 _ptr(tok), _stream())
    assert rc == 0, rc
    if cfg.kind == "smc":
        shape = (cfg.B, cfg.N)
    else:
        shape = (cfg.B,)
    zT = zT.view(*shape, R, ld)
    zD = zD.view(*shape, Kd, ld)
    return dict(zT=zT, zD=zD, draft=tok.view(*shape, K), ld=ld)
