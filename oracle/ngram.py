"""Logit n-gram store of stochastic n-gram drafting (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy / plain Python.

STAND page, Methodology item 1 (logit-based adaptive n-gram module): for every
observed n-gram the store keeps the next-token distribution, reduced to its k
most likely (index, probability) pairs; when an n-gram is seen again the
stored and the new distribution are merged by a weighted average in which an
index one side does not store counts as probability 0, and the result is cut
back to the 10 most likely entries, so memory per n-gram stays fixed.
Drafting then samples the stored distribution (item 2, Gumbel-top-k over the
stored rows).  Readings (the page leaves these open):

  * an observation is the target's sampling distribution softmax(z / tau) at
    one position; its k most likely entries (ties to the lower index) are kept
    with their probabilities under the full softmax (not renormalised), in
    fp64 and then rounded to fp32, the store's precision;
  * the weights of the average are occurrence counts: with count c stored,
        p_new(v) = (c * p_old(v) + p_obs(v)) / (c + 1)
    (the running mean of every observation seen, before truncation), computed
    in fp64 from the stored fp32 values with each operation rounded once (no
    fused multiply-add), then rounded to fp32;
  * truncation keeps the k largest rounded values, ties to the lower index,
    and stores them in that order; the count becomes c + 1;
  * several observations of one n-gram in one batch are applied in batch
    order;
  * the key is the exact n-gram (1 <= n <= 3 token ids in [0, 2^20)); a
    context with an id outside that range is not stored and raises the token
    error bit; an observation row with a NaN, infinite or negative
    probability, or a repeated index, is not stored and raises the
    non-finite error bit.

Parity status: pinned by a hand-worked merge (unstored = 0), truncation with
ties, the running-mean property over repeated observations of the same index
set, and the observed top-k against a sort of the softmax
(tests/test_oracle_ngram.py).
"""

import numpy as np

from .score import DEV_NONFINITE, DEV_TOKEN_OOB, row_is_nonfinite, row_log_softmax

KEY_MAX_ID = 1 << 20


def observe_topk(z, tau, k, rows=None):
    """The k most likely entries of softmax(z[r] / tau) per row r (or per r in
    rows): idx [U, k] int (ties to the lower index; -1 past V and in place of
    -inf entries, which have probability 0 and are not stored), prob [U, k]
    fp32 (0 where idx is -1).  Non-finite rows (NaN / +inf / all -inf) give idx -1,
    prob NaN and the non-finite error bit."""
    z = np.asarray(z)
    rows = np.arange(z.shape[0]) if rows is None else np.asarray(rows)
    U = rows.shape[0]
    idx = np.full((U, k), -1, dtype=np.int64)
    prob = np.zeros((U, k), dtype=np.float32)
    err = 0
    for u, r in enumerate(rows):
        zr = np.asarray(z[r], dtype=np.float64)
        if row_is_nonfinite(zr):
            prob[u] = np.nan
            err |= DEV_NONFINITE
            continue
        a, lse = row_log_softmax(zr, tau)
        order = np.lexsort((np.arange(zr.shape[0]), -zr))[:k]  # z order = p order
        order = order[np.isfinite(zr[order])]   # -inf entries have probability 0: not stored
        idx[u, :order.shape[0]] = order
        prob[u, :order.shape[0]] = np.exp(a[order] - lse).astype(np.float32)
    return idx, prob, err


def _row_ok(idx, prob):
    seen = set()
    for i, p in zip(idx, prob):
        if i < 0:
            continue
        if not (np.isfinite(p) and p >= 0.0) or i in seen:
            return False
        seen.add(int(i))
    return True


def merge(old_idx, old_prob, count, obs_idx, obs_prob, k):
    """One weighted-average merge of a stored row (count c) with an observation.
    Returns (idx [k], prob [k] fp32); entries -1 / 0 past the union's size."""
    old = {int(i): float(p) for i, p in zip(old_idx, old_prob) if i >= 0}
    obs = {int(i): float(p) for i, p in zip(obs_idx, obs_prob) if i >= 0}
    c = float(count)
    vals = {}
    for v in set(old) | set(obs):
        num = c * old.get(v, 0.0)          # one rounding per fp64 operation
        num = num + obs.get(v, 0.0)
        vals[v] = np.float32(num / (c + 1.0))
    keep = sorted(vals, key=lambda v: (-float(vals[v]), v))[:k]
    idx = np.full(k, -1, dtype=np.int64)
    prob = np.zeros(k, dtype=np.float32)
    for j, v in enumerate(keep):
        idx[j] = v
        prob[j] = vals[v]
    return idx, prob


class NgramStore:
    """The store as a plain map: n-gram tuple -> [count, idx [k], prob [k]]."""

    def __init__(self, n, k):
        assert 1 <= n <= 3 and 1 <= k <= 16
        self.n, self.k = n, k
        self.rows = {}

    def update(self, ctx, idx, prob):
        """Applies U observations in order; ctx [U, n], idx [U, k], prob [U, k].
        Returns the error bits."""
        err = 0
        for u in range(len(ctx)):
            key = tuple(int(t) for t in ctx[u])
            if any(t < 0 or t >= KEY_MAX_ID for t in key):
                err |= DEV_TOKEN_OOB
                continue
            if not _row_ok(idx[u], prob[u]):
                err |= DEV_NONFINITE
                continue
            c, oi, op = self.rows.get(key, (0, np.full(self.k, -1), np.zeros(self.k, np.float32)))
            ni, npr = merge(oi, op, c, idx[u], prob[u], self.k)
            self.rows[key] = (c + 1, ni, npr)
        return err

    def lookup(self, ctx):
        """Stored rows of Q contexts: idx [Q, k] (-1 if absent), prob [Q, k]
        (0 if absent), count [Q] (0 if absent)."""
        Q = len(ctx)
        idx = np.full((Q, self.k), -1, dtype=np.int64)
        prob = np.zeros((Q, self.k), dtype=np.float32)
        cnt = np.zeros(Q, dtype=np.int64)
        for q in range(Q):
            key = tuple(int(t) for t in ctx[q])
            if key in self.rows:
                cnt[q], idx[q], prob[q] = self.rows[key]
        return idx, prob, cnt
