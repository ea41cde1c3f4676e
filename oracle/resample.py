"""SMC-SD weight normalisation, ESS and systematic resampling (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

"Faster LLM Inference via Sequential Monte Carlo", section 2 (Methodology,
resampling step): low-weight particles are evicted and high-weight ones
duplicated to form the next round's N particles, following the SMC principle.
The page names no scheme; this library uses systematic resampling, run every
round (ESS is reported, not used as a trigger):

    W_j   = exp(logw_j - max logw) / sum_m exp(logw_m - max logw)
    ESS   = 1 / sum_j W_j^2
    C_j   = W_0 + ... + W_j                       (running sum, left to right)
    U_i   = (i + u0) / N,   u0 from Philox stream 4, row id = sequence b
    a_i   = min { j : C_j > U_i }   (strict), clamped to N - 1 if rounding
            leaves C_{N-1} <= U_i.

Parity status: pinned by sum W = 1, 1 <= ESS <= N, the systematic offspring
invariant (particle j gets floor(N W_j) or ceil(N W_j) copies), monotone
ancestors and a brute-force count at N = 4 over a grid of u0
(tests/test_oracle_resample.py).
"""

import numpy as np

from .philox import STREAM_RESAMPLE, row_scalar_word, uniform_from_bits
from .score import DEV_NONFINITE


def systematic_ancestors(W, u0):
    """Ancestor indices a_i = min{j : C_j > (i + u0)/N} for one sequence.

    Also returns the decision margins min(|U_i - C_{a_i}|, |U_i - C_{a_i - 1}|).
    """
    W = np.asarray(W, dtype=np.float64)
    N = W.shape[0]
    C = np.cumsum(W)
    U = (np.arange(N, dtype=np.float64) + u0) / N
    a = np.searchsorted(C, U, side="right")
    a = np.minimum(a, N - 1)
    Cprev = np.where(a > 0, C[np.maximum(a - 1, 0)], 0.0)
    margin = np.minimum(np.abs(U - C[a]), np.abs(U - Cprev))
    return a.astype(np.int64), margin


def resample_offset(seed, rnd, b):
    """u0 in (0, 1) for sequence b: word 0 of Philox stream 4, counter c0 = 0."""
    return float(uniform_from_bits(row_scalar_word(seed, rnd, STREAM_RESAMPLE, b)))


def smcsd_resample(logw, seed, rnd, b0=0):
    """Normalise log-weights, compute ESS and draw systematic ancestors.

    logw: [B, N]; b0 = global index of the first sequence (Philox row id).  Returns dict(W [B,N], ess [B], ancestors [B,N], margin [B,N], err).
    A sequence whose log-weights hold NaN or +inf, or are all -inf, gets NaN
    weights and ESS, identity ancestors, and raises the non-finite error bit.
    """
    logw = np.asarray(logw, dtype=np.float64)
    B, N = logw.shape
    W = np.zeros((B, N))
    ess = np.zeros(B)
    anc = np.zeros((B, N), dtype=np.int64)
    margin = np.full((B, N), np.inf)
    err = 0
    for b in range(B):
        lw = logw[b]
        if np.isnan(lw).any() or np.isposinf(lw).any() or np.isneginf(lw).all():
            err |= DEV_NONFINITE
            W[b] = np.nan
            ess[b] = np.nan
            anc[b] = np.arange(N)
            continue
        m = lw.max()
        w = np.exp(lw - m)
        W[b] = w / w.sum()
        ess[b] = 1.0 / np.sum(W[b] ** 2)
        anc[b], margin[b] = systematic_ancestors(W[b], resample_offset(seed, rnd, b0 + b))
    return dict(W=W, ess=ess, ancestors=anc, margin=margin, err=err)


def smcsd_resample_adaptive(logw, ess_frac, seed, rnd, b0=0):
    """Adaptive resampling: a sequence is resampled only when its ESS falls below
    ess_frac * N.

    "Faster LLM Inference via Sequential Monte Carlo", sections 2 (resampling
    step) and 5 (extensions): resampling every round is the page's scheme; the
    usual SMC refinement resamples only when the weights have degenerated, the
    effective sample size being the standard trigger.  Reading: for each
    sequence compute W and ESS as smcsd_resample does;
        resampled = ESS < ess_frac * N        (strict; ess_frac > 1: always)
        ancestors = systematic(W, u0) if resampled else the identity
        logw_next = 0 if resampled else logw  (the weights carry to the next round)
    A sequence with NaN / +inf weights, or all -inf, is not resampled: identity
    ancestors, NaN W and ESS, logw_next = logw, the non-finite error bit.

    Returns dict(W, ess, ancestors, resampled [B] int, logw_next [B, N], margin, err).
    Parity status: pinned by the never / always limits, exact ESS at the
    threshold, and the reward-weighted closed form (tests/test_oracle_resample.py).
    """
    logw = np.asarray(logw, dtype=np.float64)
    B, N = logw.shape
    r = smcsd_resample(logw, seed, rnd, b0=b0)
    resampled = np.zeros(B, dtype=np.int64)
    anc = np.tile(np.arange(N, dtype=np.int64), (B, 1))
    margin = np.full((B, N), np.inf)
    logw_next = logw.copy()
    for b in range(B):
        if np.isnan(r["ess"][b]):
            continue
        if r["ess"][b] < ess_frac * N:
            resampled[b] = 1
            anc[b] = r["ancestors"][b]
            margin[b] = r["margin"][b]
            logw_next[b] = 0.0
    return dict(W=r["W"], ess=r["ess"], ancestors=anc, resampled=resampled, logw_next=logw_next,
                margin=margin, err=r["err"])
