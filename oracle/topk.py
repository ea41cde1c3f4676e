"""Gumbel-top-k sampling without replacement, dense and sparse (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

STAND page, Methodology item 2 (Gumbel-Top-K): adding Gumbel noise to the
log-probabilities and taking the k largest indices draws k tokens without
replacement in parallel.  Methodology item 1: the n-gram store keeps only the
top-10 (index, probability) pairs per row; unstored indices have probability 0.

Dense:   s_v = z_v / tau.  The perturbed scores are drawn top-down over
         blocks of 128 entries (reading; the page only asks for Gumbel-top-k):
           block maxima   M_j = log sum_{v in j} e^{s_v} + G_j, G_j from Philox
                          stream 11 (row id = row, counter entry j);
           blocks kept    the k largest M_j (ties to the lower j): no entry of
                          another block can be among the k largest scores, since
                          k block maxima exceed all of its entries;
           entries        in a kept block, h_v = s_v + g_v with g_v from stream 5
                          (counter entry v), Z_j = max h_v, and the score
                          conditioned on the block's maximum being M_j,
                          S_v = -log(e^{-M_j} - e^{-Z_j} + e^{-h_v})
                          (the maximiser gets exactly M_j; Kool, van Hoof and
                          Welling, "Stochastic Beams and Where to Find Them",
                          2019, sampling Gumbels conditioned on their maximum).
         Independent Gumbels per entry have exactly this joint law, so the
         order of S is that of Gumbel-top-k: k draws without replacement.  With
         V <= 128 the order equals that of s_v + g_v (S is increasing in h).
         Output the k largest S (ties to the lower v): indices, scores S_v and
         log-probs s_v - lse(s).
Sparse:  s_l = log(prob_l) / tau (prob 0 gives -inf), g_l from Philox stream 6
         (row id = row), stored position l; same ordering (ties to lower l);
         output the global ids idx[row, l].
Entries with s = -inf are never selected: ranks with no finite entry left
are -1.  Rows holding NaN or +inf (dense) or a NaN, negative or infinite
probability (sparse), and dense rows that are all -inf, give -1 everywhere and
raise the non-finite error bit.

Parity status: pinned by chi-square tests of ordered-pair frequencies against
the Plackett-Luce law p_i p_j / (1 - p_i) at V = 6, k = 2 (one block) and
across five blocks at V = 600, k = 2; by the one-block reduction to the order
of s_v + g_v; and by the conditioned scores (the block maximiser scores
exactly M_j, the rest stay below it in the same order) (tests/test_oracle_topk.py);
per-seed outputs are pinned by definition only.
"""

import numpy as np

from .blockdraw import BLOCK, block_log_masses
from .philox import (STREAM_TOPK_BLOCK, STREAM_TOPK_DENSE, STREAM_TOPK_SPARSE, gumbel_from_uniform,
                     stream_words, uniform_from_bits)
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


def _conditioned_scores(h, M):
    """S_v = -log(e^{-M} - e^{-Z} + e^{-h_v}), Z = max h, in the stable form
    M - softplus(M - h_v + log(1 - e^{h_v - Z})); -inf entries stay -inf and
    the maximiser gets M exactly."""
    h = np.asarray(h, dtype=np.float64)
    Z = np.max(h)
    out = np.full(h.shape, -np.inf)
    live = h > -np.inf
    d = h[live] - Z
    with np.errstate(divide="ignore"):
        u = M - h[live] + np.log(-np.expm1(d))       # -inf for the maximiser
    out[live] = M - (np.maximum(u, 0.0) + np.log1p(np.exp(-np.abs(u))))
    return out


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
        s = s_all[r]
        lam = block_log_masses(s)
        nb = lam.shape[0]
        Mj = lam + gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_TOPK_BLOCK, r0 + r, nb)))
        kept, _ = _ordered_topk(Mj, k)
        Ms = np.sort(Mj[np.isfinite(Mj)])[::-1]
        mb = float(Ms[k - 1] - Ms[k]) if Ms.shape[0] > k else np.inf  # the kept set's margin
        g = gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_TOPK_DENSE, r0 + r, V)))
        sc = np.full(V, -np.inf)
        for j in kept[kept >= 0]:
            lo, hi = j * BLOCK, min((j + 1) * BLOCK, V)
            sc[lo:hi] = _conditioned_scores(s[lo:hi] + g[lo:hi], Mj[j])
        sel, me = _ordered_topk(sc, k)
        margin[r] = min(mb, me)
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
