"""Python binding of libsmcsd.so, the B200 scoring / resampling library.

Argument marshalling only: every step runs in the library's CUDA kernels.
PyTorch supplies device memory and the current stream.  The functions mirror
the C entry points declared in include/smcsd.h (same names, same meaning);
they take torch tensors, check shapes / dtypes / strides, pass raw pointers
and raise ``SmcsdError`` on a non-OK status.  There is no fallback: if the
library is missing or no GPU is present, calls fail loudly.
"""

import ctypes
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libsmcsd.so")

SD_OK, SD_ERR_INVALID_ARG, SD_ERR_CUDA, SD_ERR_UNSUPPORTED = 0, 1, 2, 3
SD_F32, SD_BF16 = 0, 1
DEV_TOKEN_OOB, DEV_NONFINITE, DEV_ZERO_RESIDUAL = 1, 2, 4
DEV_PAGE_OOB, DEV_ANCESTOR_OOB, DEV_TIMEOUT, DEV_ARM_OOB, DEV_TABLE_FULL = 8, 16, 32, 64, 128
REWARD_BD, REWARD_BE = 0, 1

EXPORTS = ("smcsd_score", "smcsd_resample", "smcsd_resample_adaptive", "kv_pagetable_remap",
           "sd_verify_reject", "gumbel_topk", "gumbel_topk_sparse", "sd_draft_sample",
           "sd_metasd_ucb", "ngram_table_clear", "ngram_observe_topk", "ngram_store_update",
           "ngram_store_lookup", "ngram_store_update_noalloc", "ngram_table_bytes",
           "ngram_workspace_bytes", "sd_status_string", "sd_version")

_lib = None


class SmcsdError(RuntimeError):
    def __init__(self, name, status):
        self.status = status
        super().__init__(f"{name}: {status_string(status)} (status {status})")


def load():
    """Loads libsmcsd.so (built in-tree by resample_online_log_b200/build.py)."""
    global _lib
    if _lib is not None:
        return _lib
    if not os.path.exists(LIB_PATH):
        raise RuntimeError(f"{LIB_PATH} is missing; build it with "
                           "`python resample_online_log_b200/build.py`")
    L = ctypes.CDLL(LIB_PATH)
    vp, i32, i64, u64, f32 = (ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_uint64,
                              ctypes.c_float)
    f64 = ctypes.c_double
    L.smcsd_score.argtypes = [vp, vp, i32, i32, i32, i32, i32, i64, vp, f32, u64, u64, vp, vp, vp,
                              vp, vp, vp, vp, vp, vp, vp]
    L.smcsd_resample.argtypes = [vp, i32, i32, u64, u64, vp, vp, vp, vp, vp]
    L.smcsd_resample_adaptive.argtypes = [vp, i32, i32, f64, u64, u64, vp, vp, vp, vp, vp, vp, vp]
    L.kv_pagetable_remap.argtypes = [vp, vp, i32, i32, i32, vp, vp, i32, vp, vp, i32, vp, vp]
    L.sd_verify_reject.argtypes = [vp, vp, i32, i32, i32, i32, i64, vp, f32, u64, u64, vp, vp, vp,
                                   vp, vp]
    L.gumbel_topk.argtypes = [vp, i32, i32, i32, i64, i32, f32, u64, u64, vp, vp, vp, vp, vp]
    L.gumbel_topk_sparse.argtypes = [vp, vp, i32, i32, i32, f32, u64, u64, vp, vp, vp]
    L.sd_draft_sample.argtypes = [vp, i32, i32, i32, i64, f32, u64, u64, ctypes.c_uint32, vp, vp,
                                  vp, vp]
    L.sd_metasd_ucb.argtypes = [vp, i64, vp, vp, i32, i32, i32, i32, f64, vp, vp, vp, vp, vp, vp]
    L.ngram_table_clear.argtypes = [vp, i64, i32, vp]
    L.ngram_observe_topk.argtypes = [vp, i32, i32, i32, i64, vp, i32, i32, f32, vp, vp, vp, vp]
    L.ngram_store_update.argtypes = [vp, i64, i32, vp, i32, vp, vp, i32, vp, ctypes.c_size_t, vp,
                                     vp]
    L.ngram_store_lookup.argtypes = [vp, i64, i32, vp, i32, i32, vp, vp, vp, vp, vp]
    L.ngram_store_update_noalloc.argtypes = [vp, i64, i32, vp, i32, vp, vp, i32, vp, vp]
    L.ngram_table_bytes.argtypes = [i64, i32]
    L.ngram_table_bytes.restype = ctypes.c_size_t
    L.ngram_workspace_bytes.argtypes = [i32]
    L.ngram_workspace_bytes.restype = ctypes.c_size_t
    for name in EXPORTS[:14]:
        getattr(L, name).restype = ctypes.c_int
    L.sd_status_string.argtypes = [ctypes.c_int]
    L.sd_status_string.restype = ctypes.c_char_p
    L.sd_version.argtypes = []
    L.sd_version.restype = ctypes.c_int
    _lib = L
    return L


def status_string(status):
    return load().sd_status_string(int(status)).decode()


def version():
    return load().sd_version()


def _p(t):
    return ctypes.c_void_p(0 if t is None else t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dtype(t):
    if t.dtype == torch.bfloat16:
        return SD_BF16
    if t.dtype == torch.float32:
        return SD_F32
    raise TypeError(f"logits must be bfloat16 or float32, got {t.dtype}")


def _rows_view(t, lead):
    """Checks that t is [*lead, V] with unit stride on V and one row stride ld
    between consecutive rows; returns (V, ld)."""
    if tuple(t.shape[:-1]) != tuple(lead):
        raise ValueError(f"expected leading shape {tuple(lead)}, got {tuple(t.shape)}")
    if not t.is_cuda:
        raise ValueError("logits must be CUDA tensors")
    V = t.shape[-1]
    if t.stride(-1) != 1:
        raise ValueError("the vocabulary dimension must be contiguous")
    ld = t.stride(-2) if t.dim() >= 2 else V
    expect = ld
    for d in range(t.dim() - 2, -1, -1):
        if t.shape[d] > 1 and t.stride(d) != expect:
            raise ValueError("rows must be equally spaced (one row stride ld)")
        expect *= t.shape[d]
    return V, ld


def _check_err(dev_err):
    """The device error word: a CUDA int32 tensor of one element (or None)."""
    _want(dev_err, torch.int32, (1,), "dev_err")


def _check(name, status):
    if status != SD_OK:
        raise SmcsdError(name, status)


def _want(t, dtype, shape, name):
    if t is None:
        return
    if t.dtype != dtype or tuple(t.shape) != tuple(shape) or not t.is_contiguous() or not t.is_cuda:
        raise ValueError(f"{name}: expected contiguous CUDA {dtype} of shape {tuple(shape)}, "
                         f"got {t.dtype} {tuple(t.shape)}")


def smcsd_score(zT, zD, draft_tokens, tau, seed, round, logw_out, bonus_out, logw_prev=None,
                tv_out=None, tokens_out=None, lse_out=None, lp_out=None, dev_err=None,
                stream=None, log_potential=None):
    """zT, zD: [B, N, K+1, V] (bf16 or fp32); draft_tokens int32 [B, N, K];
    log_potential: fp64 [B, N] added to every particle's log-weight (or None)."""
    B, N, R = zT.shape[:3]
    K = R - 1
    V, ld = _rows_view(zT, (B, N, R))
    V2, ld2 = _rows_view(zD, (B, N, R))
    if zD.dtype != zT.dtype or V2 != V or ld2 != ld:
        raise ValueError("zT and zD must share dtype, V and row stride")
    _want(draft_tokens, torch.int32, (B, N, K), "draft_tokens")
    _want(logw_out, torch.float64, (B, N), "logw_out")
    _want(bonus_out, torch.int32, (B, N), "bonus_out")
    _want(logw_prev, torch.float64, (B, N), "logw_prev")
    _want(log_potential, torch.float64, (B, N), "log_potential")
    _want(tv_out, torch.float32, (B, N, R), "tv_out")
    _want(tokens_out, torch.int32, (B, N, R), "tokens_out")
    _want(lse_out, torch.float64, (B, N, R, 2), "lse_out")
    _want(lp_out, torch.float64, (B, N, K, 2), "lp_out")
    _check_err(dev_err)
    st = load().smcsd_score(_p(zT), _p(zD), _dtype(zT), B, N, K, V, ld, _p(draft_tokens),
                            float(tau), int(seed), int(round), _p(logw_prev),
                            _p(log_potential), _p(logw_out),
                            _p(bonus_out), _p(tv_out), _p(tokens_out), _p(lse_out), _p(lp_out),
                            _p(dev_err), _stream(stream))
    _check("smcsd_score", st)


def smcsd_resample(logw, seed, round, ancestors_out, w_out=None, ess_out=None, dev_err=None,
                   stream=None):
    B, N = logw.shape
    _want(logw, torch.float64, (B, N), "logw")
    _want(ancestors_out, torch.int32, (B, N), "ancestors_out")
    _want(w_out, torch.float64, (B, N), "w_out")
    _want(ess_out, torch.float64, (B,), "ess_out")
    _check_err(dev_err)
    st = load().smcsd_resample(_p(logw), B, N, int(seed), int(round), _p(w_out), _p(ess_out),
                               _p(ancestors_out), _p(dev_err), _stream(stream))
    _check("smcsd_resample", st)


def smcsd_resample_adaptive(logw, ess_frac, seed, round, ancestors_out, resampled_out=None,
                            logw_next=None, w_out=None, ess_out=None, dev_err=None, stream=None):
    """Resamples sequence b only where ESS < ess_frac * N; logw_next may be logw."""
    B, N = logw.shape
    _want(logw, torch.float64, (B, N), "logw")
    _want(ancestors_out, torch.int32, (B, N), "ancestors_out")
    _want(resampled_out, torch.int32, (B,), "resampled_out")
    _want(logw_next, torch.float64, (B, N), "logw_next")
    _want(w_out, torch.float64, (B, N), "w_out")
    _want(ess_out, torch.float64, (B,), "ess_out")
    _check_err(dev_err)
    st = load().smcsd_resample_adaptive(_p(logw), B, N, float(ess_frac), int(seed), int(round),
                                        _p(w_out), _p(ess_out), _p(ancestors_out),
                                        _p(resampled_out), _p(logw_next), _p(dev_err),
                                        _stream(stream))
    _check("smcsd_resample_adaptive", st)


def kv_pagetable_remap(pt_in, ancestors, pt_out, tok_in=None, tok_out=None, page_refcnt=None,
                       num_pages=0, dev_err=None, stream=None):
    B, N, P = pt_in.shape
    _want(pt_in, torch.int32, (B, N, P), "pt_in")
    _want(pt_out, torch.int32, (B, N, P), "pt_out")
    _want(ancestors, torch.int32, (B, N), "ancestors")
    T = 0
    if tok_in is not None:
        T = tok_in.shape[2]
        _want(tok_in, torch.int32, (B, N, T), "tok_in")
        _want(tok_out, torch.int32, (B, N, T), "tok_out")
    if page_refcnt is not None:
        _want(page_refcnt, torch.int32, (num_pages,), "page_refcnt")
    _check_err(dev_err)
    st = load().kv_pagetable_remap(_p(pt_in), _p(ancestors), B, N, P, _p(pt_out), _p(tok_in), T,
                                   _p(tok_out), _p(page_refcnt), int(num_pages), _p(dev_err),
                                   _stream(stream))
    _check("kv_pagetable_remap", st)


def sd_verify_reject(zT, zD, draft_tokens, tau, seed, round, accepted_len, out_tokens, tv_out=None,
                     dev_err=None, stream=None):
    """zT: [B, K+1, V], zD: [B, K, V]; draft_tokens int32 [B, K]."""
    B, R = zT.shape[:2]
    K = R - 1
    V, ld = _rows_view(zT, (B, R))
    V2, ld2 = _rows_view(zD, (B, K))
    if zD.dtype != zT.dtype or V2 != V or ld2 != ld:
        raise ValueError("zT and zD must share dtype, V and row stride")
    _want(draft_tokens, torch.int32, (B, K), "draft_tokens")
    _want(accepted_len, torch.int32, (B,), "accepted_len")
    _want(out_tokens, torch.int32, (B, R), "out_tokens")
    _want(tv_out, torch.float32, (B, K), "tv_out")
    _check_err(dev_err)
    st = load().sd_verify_reject(_p(zT), _p(zD), _dtype(zT), B, K, V, ld, _p(draft_tokens),
                                 float(tau), int(seed), int(round), _p(accepted_len),
                                 _p(out_tokens), _p(tv_out), _p(dev_err), _stream(stream))
    _check("sd_verify_reject", st)


def gumbel_topk(z, k, tau, seed, round, idx_out, score_out=None, logp_out=None, dev_err=None,
                stream=None):
    rows = z.shape[0]
    V, ld = _rows_view(z, (rows,))
    _want(idx_out, torch.int32, (rows, k), "idx_out")
    _want(score_out, torch.float32, (rows, k), "score_out")
    _want(logp_out, torch.float32, (rows, k), "logp_out")
    _check_err(dev_err)
    st = load().gumbel_topk(_p(z), _dtype(z), rows, V, ld, int(k), float(tau), int(seed),
                            int(round), _p(idx_out), _p(score_out), _p(logp_out), _p(dev_err),
                            _stream(stream))
    _check("gumbel_topk", st)


def gumbel_topk_sparse(idx, prob, k, tau, seed, round, idx_out, dev_err=None, stream=None):
    rows, L = idx.shape
    _want(idx, torch.int32, (rows, L), "idx")
    _want(prob, torch.float32, (rows, L), "prob")
    _want(idx_out, torch.int32, (rows, k), "idx_out")
    _check_err(dev_err)
    st = load().gumbel_topk_sparse(_p(idx), _p(prob), rows, L, int(k), float(tau), int(seed),
                                   int(round), _p(idx_out), _p(dev_err), _stream(stream))
    _check("gumbel_topk_sparse", st)


def sd_draft_sample(zD, tau, seed, round, tokens_out, logq_out=None, row0=0, dev_err=None,
                    stream=None):
    """zD: [rows, V] draft logits (bf16 or fp32); tokens_out int32 [rows]."""
    rows = zD.shape[0]
    V, ld = _rows_view(zD, (rows,))
    _want(tokens_out, torch.int32, (rows,), "tokens_out")
    _want(logq_out, torch.float32, (rows,), "logq_out")
    _check_err(dev_err)
    st = load().sd_draft_sample(_p(zD), _dtype(zD), rows, V, ld, float(tau), int(seed), int(round),
                                int(row0), _p(tokens_out), _p(logq_out), _p(dev_err),
                                _stream(stream))
    _check("sd_draft_sample", st)


def sd_metasd_ucb(arm_in, pulls, sums, arm_out, K, tv=None, accepted_len=None,
                  reward_kind=REWARD_BD, c=2.0, reward_out=None, dev_err=None, stream=None):
    """One drafter-selection round for B sequences; pulls int32 / sums fp64 [B, M]
    are updated in place.  tv: fp32 [B, >=K] (BD); accepted_len: int32 [B] (BE)."""
    B, M = pulls.shape
    _want(arm_in, torch.int32, (B,), "arm_in")
    _want(arm_out, torch.int32, (B,), "arm_out")
    _want(pulls, torch.int32, (B, M), "pulls")
    _want(sums, torch.float64, (B, M), "sums")
    _want(reward_out, torch.float64, (B,), "reward_out")
    ld = 0
    if tv is not None:
        if tv.dim() != 2 or tv.shape[0] != B or tv.dtype != torch.float32 or not tv.is_cuda \
                or tv.stride(1) != 1:
            raise ValueError(f"tv: expected CUDA float32 [{B}, >={K}] with unit inner stride")
        ld = tv.stride(0) if B > 1 else tv.shape[1]
        if tv.shape[1] < K:
            raise ValueError("tv has fewer than K columns")
    if accepted_len is not None:
        _want(accepted_len, torch.int32, (B,), "accepted_len")
    _check_err(dev_err)
    st = load().sd_metasd_ucb(_p(tv), ld, _p(accepted_len), _p(arm_in), B, int(K), M,
                              int(reward_kind), float(c), _p(pulls), _p(sums), _p(arm_out),
                              _p(reward_out), _p(dev_err), _stream(stream))
    _check("sd_metasd_ucb", st)


def ngram_table_bytes(capacity, k):
    return load().ngram_table_bytes(int(capacity), int(k))


def ngram_workspace_bytes(U):
    return load().ngram_workspace_bytes(int(U))


def _table(table, capacity, k):
    need = ngram_table_bytes(capacity, k)
    if need == 0:
        raise ValueError(f"invalid n-gram table shape: capacity={capacity}, k={k}")
    if table.dtype != torch.uint8 or table.dim() != 1 or table.numel() < need or not table.is_cuda \
            or not table.is_contiguous():
        raise ValueError(f"table: expected a contiguous CUDA uint8 buffer of >= {need} bytes")


def ngram_table_clear(table, capacity, k, stream=None):
    _table(table, capacity, k)
    _check("ngram_table_clear", load().ngram_table_clear(_p(table), int(capacity), int(k),
                                                         _stream(stream)))


def ngram_observe_topk(z, k, tau, idx_out, prob_out, row_ids=None, dev_err=None, stream=None):
    """z: [rows, V] (bf16 or fp32); row_ids int32 [U] or None (U = rows)."""
    rows = z.shape[0]
    V, ld = _rows_view(z, (rows,))
    U = rows if row_ids is None else row_ids.shape[0]
    _want(row_ids, torch.int32, (U,), "row_ids")
    _want(idx_out, torch.int32, (U, k), "idx_out")
    _want(prob_out, torch.float32, (U, k), "prob_out")
    _check_err(dev_err)
    st = load().ngram_observe_topk(_p(z), _dtype(z), rows, V, ld, _p(row_ids), U, int(k),
                                   float(tau), _p(idx_out), _p(prob_out), _p(dev_err),
                                   _stream(stream))
    _check("ngram_observe_topk", st)


def ngram_store_update(table, capacity, k, ctx, idx, prob, workspace, dev_err=None, stream=None):
    """ctx int32 [U, n]; idx int32 / prob fp32 [U, k]; workspace: CUDA uint8 of
    >= ngram_workspace_bytes(U) bytes."""
    _table(table, capacity, k)
    U, n = ctx.shape
    _want(ctx, torch.int32, (U, n), "ctx")
    _want(idx, torch.int32, (U, k), "idx")
    _want(prob, torch.float32, (U, k), "prob")
    if workspace.dtype != torch.uint8 or not workspace.is_cuda or not workspace.is_contiguous():
        raise ValueError("workspace: expected a contiguous CUDA uint8 buffer")
    _check_err(dev_err)
    st = load().ngram_store_update(_p(table), int(capacity), int(k), _p(ctx), n, _p(idx), _p(prob),
                                   U, _p(workspace), workspace.numel(), _p(dev_err),
                                   _stream(stream))
    _check("ngram_store_update", st)


def ngram_store_update_noalloc(table, capacity, k, ctx, idx, prob, dev_err=None, stream=None):
    """ngram_store_update with the library's own workspace: allocates nothing.
    Calls that overlap on the GPU race on that workspace."""
    _table(table, capacity, k)
    U, n = ctx.shape
    _want(ctx, torch.int32, (U, n), "ctx")
    _want(idx, torch.int32, (U, k), "idx")
    _want(prob, torch.float32, (U, k), "prob")
    _check_err(dev_err)
    st = load().ngram_store_update_noalloc(_p(table), int(capacity), int(k), _p(ctx), n, _p(idx),
                                           _p(prob), U, _p(dev_err), _stream(stream))
    _check("ngram_store_update_noalloc", st)


def ngram_store_lookup(table, capacity, k, ctx, idx_out, prob_out, count_out=None, dev_err=None,
                       stream=None):
    _table(table, capacity, k)
    Q, n = ctx.shape
    _want(ctx, torch.int32, (Q, n), "ctx")
    _want(idx_out, torch.int32, (Q, k), "idx_out")
    _want(prob_out, torch.float32, (Q, k), "prob_out")
    _want(count_out, torch.int32, (Q,), "count_out")
    _check_err(dev_err)
    st = load().ngram_store_lookup(_p(table), int(capacity), int(k), _p(ctx), n, Q, _p(idx_out),
                                   _p(prob_out), _p(count_out), _p(dev_err), _stream(stream))
    _check("ngram_store_lookup", st)


class NgramTable:
    """A logit n-gram store on the current CUDA device: the table buffer and an
    update workspace held as torch tensors, cleared on creation."""

    def __init__(self, capacity, k=10, max_update=16384, device="cuda"):
        self.capacity, self.k = int(capacity), int(k)
        self.table = torch.empty((ngram_table_bytes(capacity, k),), dtype=torch.uint8, device=device)
        self.workspace = torch.empty((ngram_workspace_bytes(max_update),), dtype=torch.uint8,
                                     device=device)
        ngram_table_clear(self.table, capacity, k)

    def update(self, ctx, idx, prob, dev_err=None, stream=None):
        ngram_store_update(self.table, self.capacity, self.k, ctx, idx, prob, self.workspace,
                           dev_err=dev_err, stream=stream)

    def lookup(self, ctx, idx_out, prob_out, count_out=None, dev_err=None, stream=None):
        ngram_store_lookup(self.table, self.capacity, self.k, ctx, idx_out, prob_out,
                           count_out=count_out, dev_err=dev_err, stream=stream)
