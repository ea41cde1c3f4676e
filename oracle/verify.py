"""Standard speculative-decoding verification, N = 1 (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

"Faster LLM Inference via Sequential Monte Carlo", section 1 (problem
definition) and METASD section 1 (background): a draft model proposes K tokens,
the target verifies them, the first rejection discards the rest.  The pages do
not print the rule; this is the textbook speculative-sampling rule:

  for k = 0 .. K-1 (draft token x = x_{k+1}, p = p_T row k, q = q_D row k):
      u_k ~ U(0,1) from Philox stream 2, row id b*(K+1)+k, c0 = 0, word 0
      accept iff u_k * q(x) < p(x)          (u < min(1, p/q) without a division)
  at the first reject j:
      r_v = max(p_v - q_v, 0); the emitted token is a sample of the normalised
      residual by the exact two-level Gumbel-max of ``oracle.blockdraw`` over
      log r (block noise from Philox stream 12, entry noise from stream 3, row
      id b*(K+1)+j): the 128-entry block by log sum r + G_j, then
      argmax_{v : r_v > 0} (log r_v + g_v) inside it.
      If every r_v = 0 the zero-residual error bit is raised and the token is
      drawn from p by the same draw over a = z/tau with the same streams.
  if all K are accepted: the bonus token is the two-level draw over
      a = z_T[K]/tau with block noise from stream 9 and entry noise from
      stream 1, row id b (the SMC-SD bonus sampler).
  accepted_len = j (or K); out_tokens = accepted drafts + the one drawn token,
  padded with -1 to K+1 entries; tv[b, k] = 1/2 sum_v |p_v - q_v| at all k < K
  (METASD section 2, Block Divergence built on total variation).

Edge cases: a draft token outside [0, V) is rejected (accept probability 0)
and raises the token error bit.  A non-finite target or draft row at a
position the sequence reaches stops the sequence there: accepted_len is that
position, no token is emitted at it.  The non-finite bit is raised for any
non-finite row among the K verified positions (its TV is NaN) and for the
target row K+1 when the sequence reaches it.

Parity status: the accept rule and residual are pinned by exhaustive
enumeration at V = 4, K = 2 (the emitted token law equals the target law to
1e-12); the sampler by chi-square tests (tests/test_oracle_verify.py).
"""

import numpy as np

from .blockdraw import block_gumbel_argmax
from .philox import (STREAM_ACCEPT, STREAM_BONUS, STREAM_BONUS_BLOCK, STREAM_RESIDUAL,
                     STREAM_RESIDUAL_BLOCK, row_scalar_word, uniform_from_bits)
from .score import DEV_NONFINITE, DEV_TOKEN_OOB, DEV_ZERO_RESIDUAL, row_log_softmax, total_variation


def accept_probability(p, q, x):
    """min(1, p(x)/q(x)): probability that draft token x survives verification."""
    if q[x] == 0.0:
        return 1.0
    return min(1.0, p[x] / q[x])


def residual_distribution(p, q):
    """Normalised max(p - q, 0), the law of the token drawn after a rejection."""
    r = np.maximum(np.asarray(p, dtype=np.float64) - np.asarray(q, dtype=np.float64), 0.0)
    s = r.sum()
    return r / s if s > 0 else None


def accept_uniform(seed, rnd, row_id):
    return float(uniform_from_bits(row_scalar_word(seed, rnd, STREAM_ACCEPT, row_id)))


def sd_verify_reject(zT, zD, draft_tokens, tau, seed, rnd, b0=0):
    """Verify K drafted tokens per sequence.

    zT: [B, K+1, V], zD: [B, K, V], draft_tokens: [B, K]; b0 = global index of
    the first sequence (Philox row ids use the global sequence index).
    Returns dict(accepted_len [B], out_tokens [B, K+1], tv [B, K],
                 accept_margin [B, K] (inf where no decision was taken),
                 token_margin [B], err).
    """
    zT = np.asarray(zT)
    zD = np.asarray(zD)
    draft = np.asarray(draft_tokens, dtype=np.int64)
    B, R, V = zT.shape
    K = R - 1
    assert zD.shape == (B, K, V) and draft.shape == (B, K)
    acc_len = np.zeros(B, dtype=np.int64)
    out = np.full((B, R), -1, dtype=np.int64)
    tv = np.zeros((B, K))
    acc_margin = np.full((B, K), np.inf)
    tok_margin = np.full(B, np.inf)
    err = 0
    for b in range(B):
        a, lse_t = row_log_softmax(zT[b], tau)
        d, lse_d = row_log_softmax(zD[b], tau)
        tv[b] = total_variation(a[:K], lse_t[:K], d, lse_d)
        if np.isnan(lse_t[:K]).any() or np.isnan(lse_d).any():
            err |= DEV_NONFINITE      # a NaN TV is reported even past the first rejection
        done = False
        for k in range(K):
            if np.isnan(lse_t[k]) or np.isnan(lse_d[k]):
                err |= DEV_NONFINITE
                acc_len[b] = k
                done = True
                break
            p = np.exp(a[k] - lse_t[k])
            q = np.exp(d[k] - lse_d[k])
            x = int(draft[b, k])
            u = accept_uniform(seed, rnd, (b0 + b) * R + k)
            if 0 <= x < V:
                accept = u * q[x] < p[x]
                acc_margin[b, k] = abs(u - accept_probability(p, q, x))
            else:
                err |= DEV_TOKEN_OOB
                accept = False
            if accept:
                out[b, k] = x
                continue
            r = np.maximum(p - q, 0.0)
            if (r > 0).any():
                with np.errstate(divide="ignore"):
                    w = np.where(r > 0, np.log(np.where(r > 0, r, 1.0)), -np.inf)
            else:
                err |= DEV_ZERO_RESIDUAL
                w = a[k]
            tok, mg = block_gumbel_argmax(w, seed, rnd, STREAM_RESIDUAL_BLOCK, STREAM_RESIDUAL,
                                          (b0 + b) * R + k)
            out[b, k] = tok
            tok_margin[b] = mg
            acc_len[b] = k
            done = True
            break
        if done:
            continue
        acc_len[b] = K
        if np.isnan(lse_t[K]):
            err |= DEV_NONFINITE
            continue
        tok, mg = block_gumbel_argmax(a[K], seed, rnd, STREAM_BONUS_BLOCK, STREAM_BONUS, b0 + b)
        out[b, K] = tok
        tok_margin[b] = mg
    return dict(accepted_len=acc_len, out_tokens=out, tv=tv, accept_margin=acc_margin,
                token_margin=tok_margin, err=err)
