"""Draft step: one token per draft row sampled from q_D (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

"Faster LLM Inference via Sequential Monte Carlo", section 2 (Methodology,
draft step): the draft model extends each of the N particles by K tokens,
one position at a time; the tokens are samples from the drafter's own
distribution q_D.  STAND page, Methodology item 1: drafting samples from the
stored distribution instead of taking its argmax (stochastic drafting).
Reading (the pages give no sampler): the exact two-level Gumbel-max of
``oracle.blockdraw`` over a = zD[r] / tau -- the 128-entry block by its
log-mass plus block noise from Philox stream 10, then the entry inside it by
Gumbel-max with entry noise from stream 8 (row id = row0 + r, counter entry
j or v, ties to the lower index) -- and

    logq_r = zD[r, x_r] / tau - logsumexp_v(zD[r, v] / tau)

so that x_r ~ softmax(zD[r] / tau) exactly and logq_r is the log q_D(x) the
importance weight of the round needs.  For V <= 128 the draw is the plain
Gumbel-max argmax_v (a_v + g_v) on stream 8.  Rows with NaN or +inf, or all -inf,
give x = -1, logq = NaN and raise the non-finite error bit.

Parity status: pinned by a chi-square test of the sampled frequencies against
softmax(z / tau) at V = 16 and at V = 1000 (8 blocks), by logq against the
closed-form log-softmax, and by masked entries never being drawn
(tests/test_oracle_draft.py); per-seed outputs are pinned by definition only.
"""

import numpy as np

from .blockdraw import block_gumbel_argmax
from .philox import STREAM_DRAFT, STREAM_DRAFT_BLOCK, gumbel_from_uniform, stream_words, uniform_from_bits
from .score import DEV_NONFINITE, row_is_nonfinite, row_log_softmax


def draft_noise(seed, rnd, row_id, V):
    """Gumbel noise g_v, v < V, of the draft draw for one row (stream 8)."""
    return gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_DRAFT, row_id, V)))


def sd_draft_sample(zD, tau, seed, rnd, row0=0):
    """zD [rows, V] -> dict(tokens [rows], logq [rows], margin [rows], err)."""
    zD = np.asarray(zD)
    rows, V = zD.shape
    a, lse = row_log_softmax(zD, tau)
    bad = row_is_nonfinite(a)
    tokens = np.full(rows, -1, dtype=np.int64)
    logq = np.full(rows, np.nan)
    margin = np.full(rows, np.inf)
    err = 0
    for r in range(rows):
        if bad[r]:
            err |= DEV_NONFINITE
            continue
        x, margin[r] = block_gumbel_argmax(a[r], seed, rnd, STREAM_DRAFT_BLOCK, STREAM_DRAFT, row0 + r)
        tokens[r] = x
        logq[r] = a[r, x] - lse[r]
    return dict(tokens=tokens, logq=logq, margin=margin, err=err)
