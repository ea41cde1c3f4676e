"""Exact categorical draw by a two-level Gumbel-max (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

The pages fix that the bonus token of an SMC-SD round is a sample from the
target distribution ("Faster LLM Inference via Sequential Monte Carlo",
section 2: each round also commits one token drawn from the target at position
K+1) but not how it is drawn.  Reading: a two-level Gumbel-max over blocks of
128 consecutive vocabulary entries,

    lambda_j = log sum_{v in block j} exp(a_v)                 (a = z / tau, fp64)
    j*       = argmax_j ( lambda_j + gamma_j ),  gamma_j from the block stream,
                                                  counter entry j (ties: lower j)
    v*       = argmax_{v in block j*} ( a_v + g_v ),  g_v from the entry stream,
                                                  counter entry v (ties: lower v)

P(j* = j) = sum_{v in j} p_v (Gumbel-max over log-masses) and P(v* = v | j*) =
p_v / mass(j*) (Gumbel-max inside the block), so v* ~ softmax(a) exactly, as
one-level Gumbel-max is; only one block's entries need noise.  With V <= 128
there is one block and the draw is the one-level Gumbel-max of the entry
stream.  Blocks whose entries are all -inf have lambda = -inf and are never
chosen.

Parity status: pinned by the one-block reduction to plain Gumbel-max, a
chi-square test of 20000 draws at V = 1000 (8 blocks) against softmax, and
the block-confined case (tests/test_oracle_blockdraw.py).
"""

import numpy as np

from .philox import gumbel_from_uniform, stream_words, uniform_from_bits

BLOCK = 128


def _argmax_margin(scores):
    """First index of the largest score and its gap to the runner-up (inf if none)."""
    scores = np.asarray(scores, dtype=np.float64)
    idx = int(np.argmax(scores))
    if scores.shape[0] < 2:
        return idx, np.inf
    rest = np.delete(scores, idx)
    gap = float(scores[idx] - np.max(rest))
    return idx, (np.inf if np.isnan(gap) else gap)


def block_log_masses(a):
    """lambda_j = log sum_{v in block j} exp(a_v) for the blocks of one fp64 row."""
    a = np.asarray(a, dtype=np.float64)
    V = a.shape[0]
    nb = (V + BLOCK - 1) // BLOCK
    lam = np.full(nb, -np.inf)
    for j in range(nb):
        seg = a[j * BLOCK:(j + 1) * BLOCK]
        m = np.max(seg)
        if m > -np.inf:
            lam[j] = m + np.log(np.sum(np.exp(seg - m)))
    return lam


def block_gumbel_argmax(a, seed, rnd, tag_block, tag_entry, row_id):
    """The two-level draw over one row of a = z / tau (finite or -inf entries).

    Returns (v*, margin): margin = the smaller of the block decision's and the
    in-block decision's gap to the runner-up (inf when a decision is forced)."""
    a = np.asarray(a, dtype=np.float64)
    V = a.shape[0]
    lam = block_log_masses(a)
    nb = lam.shape[0]
    gam = gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, tag_block, row_id, nb)))
    j, mb = _argmax_margin(lam + gam)
    lo, hi = j * BLOCK, min((j + 1) * BLOCK, V)
    g = gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, tag_entry, row_id, hi)))[lo:hi]
    v, me = _argmax_margin(a[lo:hi] + g)
    return lo + v, min(mb, me)
