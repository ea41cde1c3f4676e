"""SMC-SD scoring step: log-softmax, importance log-weights, TV, bonus token.

Test infrastructure only (see ``oracle/__init__``).  NumPy, fp64.

Definitions followed (all readings are listed in the project's design notes):
  * "Faster LLM Inference via Sequential Monte Carlo", section 2 (Methodology,
    scoring + resampling steps): every particle carries an importance weight in
    place of token rejection.  Reading: the log-weight of particle n is
        logw[n] = logw_prev[n] + sum_{k<K} ( log p_T(x_{k+1}) - log q_D(x_{k+1}) )
    with p_T = softmax(z_T / tau), q_D = softmax(z_D / tau) at the row that
    scores draft token x_{k+1}.  The bonus token is drawn from p_T, so its ratio
    is 1 and it does not enter the weight.
  * same page, section 2 (bonus token): each round also commits one token drawn
    from the target at position K+1.  Reading: the exact two-level Gumbel-max
    of ``oracle.blockdraw`` over a = z_T[K] / tau, block noise from Philox
    stream 9 and entry noise from stream 1, row id = b * N + n (for V <= 128:
    bonus = argmax_v (a_v + g_v), g_v from stream 1; ties to the lower v).
  * METASD page, section 2 (Block Divergence built on total-variation
    distance): per row, tv = 1/2 * sum_v | p_T(v) - q_D(v) |, reported at all
    K+1 positions.

Parity status: lse / lp / logw / tv are the fp64 definition written out and are
pinned by closed forms and invariants (tests/test_oracle_score.py).  The bonus
token is pinned by a chi-square test of Gumbel-max against softmax at V = 16
and by the two-level draw's own pins (tests/test_oracle_blockdraw.py).
"""

import numpy as np

from .blockdraw import block_gumbel_argmax
from .philox import STREAM_BONUS, STREAM_BONUS_BLOCK, gumbel_from_uniform, stream_words, uniform_from_bits

# Device error-word bits (the library's caller-visible error word uses the same values).
DEV_TOKEN_OOB = 1
DEV_NONFINITE = 2
DEV_ZERO_RESIDUAL = 4
DEV_PAGE_OOB = 8
DEV_ANCESTOR_OOB = 16


def tau64(tau):
    """Temperature as the library receives it: an fp32 value, widened exactly."""
    return float(np.float32(tau))


def row_is_nonfinite(z):
    """A row is unusable if it holds NaN or +inf, or if every entry is -inf."""
    z = np.asarray(z, dtype=np.float64)
    bad = np.isnan(z).any(axis=-1) | np.isposinf(z).any(axis=-1)
    allneg = np.isneginf(z).all(axis=-1)
    return bad | allneg


def row_log_softmax(z, tau):
    """Scaled logits a = z / tau and lse = log sum_v exp(a_v), fp64, per row.

    lse uses the max-shifted form m + log(sum exp(a - m)).  Rows that are
    non-finite (see ``row_is_nonfinite``) get lse = NaN.
    """
    a = np.asarray(z, dtype=np.float64) / tau64(tau)
    bad = row_is_nonfinite(a)
    with np.errstate(invalid="ignore", over="ignore"):
        m = np.max(a, axis=-1, keepdims=True)
        lse = m[..., 0] + np.log(np.sum(np.exp(a - m), axis=-1))
    lse = np.where(bad, np.nan, lse)
    return a, lse


def total_variation(a, lse_a, b, lse_b):
    """tv = 1/2 sum_v |exp(a_v - lse_a) - exp(b_v - lse_b)| per row (fp64)."""
    with np.errstate(invalid="ignore"):
        p = np.exp(a - lse_a[..., None])
        q = np.exp(b - lse_b[..., None])
        return 0.5 * np.sum(np.abs(p - q), axis=-1)


def gumbel_argmax(scores):
    """Index of the largest entry (first on ties) and its margin over the runner-up."""
    scores = np.asarray(scores, dtype=np.float64)
    idx = int(np.argmax(scores))
    if scores.shape[0] < 2:
        return idx, np.inf
    top2 = np.partition(scores, -2)[-2:]
    return idx, float(top2[1] - top2[0])


def bonus_noise(seed, rnd, row_id, V):
    """Gumbel noise g_v, v < V, of the bonus draw for one particle (stream 1)."""
    return gumbel_from_uniform(uniform_from_bits(stream_words(seed, rnd, STREAM_BONUS, row_id, V)))


def smcsd_score(zT, zD, draft_tokens, tau, seed, rnd, logw_prev=None, b0=0, log_potential=None):
    """Score one SMC-SD round for B sequences x N particles x (K+1) positions.

    zT, zD: [B, N, K+1, V] target / draft logits (any float dtype; widened to fp64).
    draft_tokens: [B, N, K] int, token x_{k+1} scored at row k.
    logw_prev: optional [B, N] fp64 log-weights carried from the last round.
    b0: global index of the first sequence when these B sequences are a sample
        of a larger batch (Philox row ids use the global particle index).
    log_potential: optional [B, N] fp64 extra log-potential per particle
        ("Faster LLM Inference via Sequential Monte Carlo", section 5: the
        method extends to constrained and reward-weighted decoding).  Reading:
        the target of the round becomes p_T(x) phi(x) for a caller-given
        potential phi (a reward, or 0 / 1 for a constraint), so the importance
        weight gains the factor phi: logw += log phi (-inf drops the particle).

    Returns a dict with
      lse    [B, N, K+1, 2]  (lse of target row, lse of draft row)
      lp     [B, N, K, 2]    (log p_T(x), log q_D(x)) at rows k < K
      tv     [B, N, K+1]
      logw   [B, N]
      bonus  [B, N]          (-1 when the target row K is unusable)
      tokens [B, N, K+1]     (x_1..x_K, bonus): the tokens the round commits
      bonus_margin [B, N]    (best minus runner-up perturbed score)
      err    int             (device error-word bits the library would raise)
    """
    zT = np.asarray(zT)
    zD = np.asarray(zD)
    draft_tokens = np.asarray(draft_tokens, dtype=np.int64)
    B, N, R, V = zT.shape
    K = R - 1
    assert zD.shape == zT.shape and draft_tokens.shape == (B, N, K)
    lse = np.zeros((B, N, R, 2))
    lp = np.zeros((B, N, K, 2))
    tv = np.zeros((B, N, R))
    logw = np.zeros((B, N))
    bonus = np.full((B, N), -1, dtype=np.int64)
    margin = np.full((B, N), np.inf)
    tokens = np.zeros((B, N, R), dtype=np.int64)
    err = 0
    for b in range(B):
        for n in range(N):
            a, lse_t = row_log_softmax(zT[b, n], tau)
            d, lse_d = row_log_softmax(zD[b, n], tau)
            if np.isnan(lse_t).any() or np.isnan(lse_d).any():
                err |= DEV_NONFINITE
            lse[b, n, :, 0] = lse_t
            lse[b, n, :, 1] = lse_d
            tv[b, n] = total_variation(a, lse_t, d, lse_d)
            acc = 0.0 if logw_prev is None else float(logw_prev[b, n])
            if log_potential is not None:
                acc += float(log_potential[b, n])
            for k in range(K):
                x = int(draft_tokens[b, n, k])
                if 0 <= x < V:
                    lp[b, n, k, 0] = a[k, x] - lse_t[k]
                    lp[b, n, k, 1] = d[k, x] - lse_d[k]
                else:
                    err |= DEV_TOKEN_OOB
                    lp[b, n, k, :] = np.nan
                acc += lp[b, n, k, 0] - lp[b, n, k, 1]
            logw[b, n] = acc
            tokens[b, n, :K] = draft_tokens[b, n]
            if not np.isnan(lse_t[K]):
                idx, mg = block_gumbel_argmax(a[K], seed, rnd, STREAM_BONUS_BLOCK, STREAM_BONUS,
                                              (b0 + b) * N + n)
                bonus[b, n] = idx
                margin[b, n] = mg
            tokens[b, n, K] = bonus[b, n]
    return dict(lse=lse, lp=lp, tv=tv, logw=logw, bonus=bonus, tokens=tokens,
                bonus_margin=margin, err=err)
