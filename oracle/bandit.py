"""Drafter selection by a multi-armed bandit (oracle side).

Test infrastructure only (see ``oracle/__init__``).  NumPy / plain Python, fp64.

METASD page, section 2 (Methodology): every speculative-decoding round picks
one of M drafters with a multi-armed bandit; the reward of the round is either
the number of accepted tokens (Block Efficiency, BE) or the Block Divergence
(BD), an alignment signal built on the total-variation distance between the
drafter's and the target's next-token distributions; MetaSD-UCB is an upper
confidence bound rule fed with that reward.  The page prints no formula.
Readings (the plainest ones the prose supports):

  * one bandit per sequence (the best drafter depends on the prompt);
  * rewards lie in [0, 1]:
        BD = 1 - (1/K) * sum_{k<K} TV_k    over the round's K drafted positions,
        BE = accepted_len / K;
  * the arm index is UCB1's,
        ucb_i = S_i / n_i + sqrt(c * ln(t) / n_i),   t = sum_i n_i,
    every arm not yet pulled is taken first (lowest index), ties go to the
    lowest index, c = 2 gives the textbook UCB1 bonus sqrt(2 ln t / n_i).

One call of ``metasd_ucb_step`` is one round for B sequences: the reward of the
arm each sequence used (arm_in = -1: no arm yet) updates its (pulls, sums) and
the rule picks the arm of the next round.  A reward that is not finite (a NaN
TV row, an accepted length outside [0, K]) leaves the state untouched and
raises the non-finite error bit; an arm_in outside [-1, M) raises the arm
error bit and is ignored.

Parity status: pinned by the textbook UCB1 values on a worked example, the
pull-every-arm-first rule, the BD / BE closed forms on hand-made rows, and by
the rule settling on the best of stationary Bernoulli arms
(tests/test_oracle_bandit.py).
"""

import math

import numpy as np

from .score import DEV_NONFINITE

DEV_ARM_OOB = 64
REWARD_BD, REWARD_BE = 0, 1


def block_reward(tv_row, accepted_len, K, kind):
    """Reward of one round in [0, 1]: BD from the K per-position TVs, or BE."""
    if kind == REWARD_BD:
        tv = [float(t) for t in tv_row[:K]]
        return 1.0 - sum(tv) / K
    if not 0 <= int(accepted_len) <= K:
        return math.nan      # not a block length: treated as a faulty round
    return float(accepted_len) / K


def ucb_choice(pulls, sums, c):
    """The arm UCB1 pulls next, and the gap between its index and the runner-up's
    (inf when the choice is forced: an arm not yet pulled)."""
    M = len(pulls)
    for i in range(M):
        if pulls[i] == 0:
            return i, math.inf
    t = sum(int(n) for n in pulls)
    idx = [sums[i] / pulls[i] + math.sqrt(c * math.log(t) / pulls[i]) for i in range(M)]
    best = 0
    for i in range(1, M):
        if idx[i] > idx[best]:
            best = i
    others = [idx[i] for i in range(M) if i != best]
    gap = idx[best] - max(others) if others else math.inf
    return best, gap


def metasd_ucb_step(tv, accepted_len, arm_in, pulls, sums, K, c=2.0, kind=REWARD_BD):
    """One bandit round for B sequences.

    tv [B, >=K] per-position TV of the round; accepted_len [B]; arm_in [B]
    (-1: no arm used yet); pulls [B, M] int, sums [B, M] fp64 (the state).
    Returns dict(pulls, sums, arm [B], reward [B] (NaN where none), gap [B], err).
    """
    pulls = np.array(pulls, dtype=np.int64)
    sums = np.array(sums, dtype=np.float64)
    B, M = pulls.shape
    arm_out = np.zeros(B, dtype=np.int64)
    reward = np.full(B, np.nan)
    gap = np.full(B, np.inf)
    err = 0
    for b in range(B):
        a = int(arm_in[b])
        if a >= M or a < -1:
            err |= DEV_ARM_OOB
        elif a >= 0:
            r = block_reward(tv[b], accepted_len[b], K, kind)
            if math.isfinite(r):
                pulls[b, a] += 1
                sums[b, a] += r
                reward[b] = r
            else:
                err |= DEV_NONFINITE
        arm_out[b], gap[b] = ucb_choice(pulls[b], sums[b], c)
    return dict(pulls=pulls, sums=sums, arm=arm_out, reward=reward, gap=gap, err=err)
