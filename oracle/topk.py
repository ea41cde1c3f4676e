"""Gumbel-top-k sampling without replacement, dense and sparse (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

STAND page, Methodology item 2 (Gumbel-Top-K): adding Gumbel noise to the
log-probabilities and taking the k largest indices draws k tokens without
replacement in parallel.  Methodology item 1: the n-gram store keeps only the
top-10 (index, probability) pairs per row; unstored indices have probability 0.

Dense:   s_v = z_v / tau, g_v from Philox stream 5 (row id = row), entry v;
         order entries by s_v + g_v descending, ties to the lower v; output the
         first k indices, their perturbed scores and log-probs s_v - lse(s).
Sparse:  s_l = log(prob_l) / tau (prob 0 gives -inf), g_l from Philox stream 6
         (row id = row), stored position l; same ordering (ties to lower l);
         output the global ids idx[row, l].
Entries with s = -inf are never selected: ranks with no finite entry left
are -1.  Rows holding NaN or +inf (dense) or a NaN, negative or infinite
probability (sparse), and dense rows that are all -inf, give -1 everywhere and
raise the non-finite error bit.

Parity status: pinned by a chi-square test of ordered-pair frequencies against
the Plackett-Luce law p_i p_j / (1 - p_i) at V = 6, k = 2
(tests/test_oracle_topk.py); per-seed outputs are pinned by definition only.
"""

import numpy as np

from .philox import STREAM_TOPK_DENSE, STREAM_TOPK_SPARSE, gumbel_from_uniform, stream_words, uniform_from_bits
from .score import DEV_NONFINITE, row_is_nonfinite, row_log_softmax, tau64


def _ordered_topk(score, k):
    """Indices of the k largest finite scores (ties to the lower index), padded with -1,
    plus the minimum gap between consecutive ranks 1..k+1 (inf if undefined)."""
    n = score.shape[0]
    order = np.lexsort((np.arange(n), -score))   # primary: -score, secondary: index
    finite = np.isfinite(score[order])
    take = order[:k]
    ok = finite[:k]
    sel = np.where(ok, take, -1)
    ranked = score[order[:min(k + 1, n)]]
    ranked = ranked[np.isfinite(ranked)]
    gaps = ranked[:-1] - ranked[1:]
    margin = float(gaps.min()) if gaps.size else np.inf
    return sel, margin


def gumbel_topk(z, k, tau, seed, rnd, r0=0):
    """Dense rows z [rows, V] -> dict(idx [rows,k], score [rows,k], logp [rows,k], margin [rows], err).
    r0 = global index of the first row (Philox row id)."""
    z = np.asarray(z)
    rows, V = z.shape
    idx = np.full((rows, k), -1, dtype=np.int64)
    score = np.full((rows, k), np.nan)
    logp = np.full((rows, k), np.nan)
    margin = np.full(rows, np.inf)
    err = 0
    s_all, lse = row_log_softmax(z, tau)
    bad = row_is_nonfinite(s_all)
    for r in range(rows):
        if bad[r]:
            err |= DEV_NONFINITE
            continue
        g = gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_TOPK_DENSE, r0 + r, V)))
        sc = s_all[r] + g
        sel, margin[r] = _ordered_topk(sc, k)
        idx[r] = sel
        ok = sel >= 0
        score[r, ok] = sc[sel[ok]]
        logp[r, ok] = s_all[r, sel[ok]] - lse[r]
    return dict(idx=idx, score=score, logp=logp, margin=margin, err=err)


def gumbel_topk_sparse(idx_in, prob, k, tau, seed, rnd, r0=0):
    """Sparse rows (idx [rows, L], prob [rows, L]) -> dict(idx [rows,k], margin [rows], err)."""
    idx_in = np.asarray(idx_in, dtype=np.int64)
    prob = np.asarray(prob, dtype=np.float64)
    rows, L = prob.shape
    out = np.full((rows, k), -1, dtype=np.int64)
    margin = np.full(rows, np.inf)
    err = 0
    t = tau64(tau)
    for r in range(rows):
        pr = prob[r]
        if np.isnan(pr).any() or (pr < 0).any() or np.isinf(pr).any():
            err |= DEV_NONFINITE
            continue
        with np.errstate(divide="ignore"):
            s = np.where(pr > 0, np.log(np.where(pr > 0, pr, 1.0)) / t, -np.inf)
        g = gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_TOPK_SPARSE, r0 + r, L)))
        sel, margin[r] = _ordered_topk(s + g, k)
        out[r] = np.where(sel >= 0, idx_in[r, np.maximum(sel, 0)], -1)
    return dict(idx=out, margin=margin, err=err)
