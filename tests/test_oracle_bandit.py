"""Pins of the drafter-selection bandit oracle (METASD page, section 2:
MetaSD-UCB fed with the Block Divergence or Block Efficiency reward)."""

import math

import numpy as np

import oracle
from oracle import REWARD_BD, REWARD_BE


def test_ucb1_worked_example():
    # Two arms: arm 0 pulled 10 times (total reward 5.0), arm 1 once (0.6).
    # t = 11; index_0 = 0.5 + sqrt(2 ln 11 / 10) = 1.192516...,
    #         index_1 = 0.6 + sqrt(2 ln 11 / 1)  = 2.789929...  -> arm 1.
    arm, gap = oracle.ucb_choice([10, 1], [5.0, 0.6], 2.0)
    assert arm == 1
    assert abs(gap - (2.789929 - 1.192516)) < 2e-6
    # With the exploration bonus off the greedy mean wins.
    arm, gap = oracle.ucb_choice([10, 1], [5.0, 0.6], 0.0)
    assert arm == 1 and abs(gap - 0.1) < 1e-12
    arm, _ = oracle.ucb_choice([10, 1], [7.0, 0.6], 0.0)
    assert arm == 0
    # c = 0.1: index_0 = 0.7 + sqrt(0.1 ln 11 / 10) = 0.854851..., index_1 = 0.6 + 0.489683 = 1.089683.
    arm, gap = oracle.ucb_choice([10, 1], [7.0, 0.6], 0.1)
    assert arm == 1 and abs(gap - (1.089683 - 0.854851)) < 2e-6


def test_unpulled_arms_come_first_and_ties_go_low():
    assert oracle.ucb_choice([3, 0, 0], [1.0, 0.0, 0.0], 2.0) == (1, math.inf)
    assert oracle.ucb_choice([3, 1, 0], [1.0, 0.0, 0.0], 2.0) == (2, math.inf)
    arm, gap = oracle.ucb_choice([4, 4, 4], [2.0, 2.0, 2.0], 2.0)
    assert arm == 0 and gap == 0.0


def test_rewards_closed_form():
    tv = np.array([0.1, 0.3, 0.2, 0.4, 0.99])   # the (K+1)-th TV is not part of the block
    assert abs(oracle.block_reward(tv, 0, 4, REWARD_BD) - 0.75) < 1e-15
    assert oracle.block_reward(tv, 3, 4, REWARD_BE) == 0.75
    assert oracle.block_reward(np.zeros(4), 0, 4, REWARD_BD) == 1.0
    assert oracle.block_reward(np.ones(4), 4, 4, REWARD_BD) == 0.0
    assert math.isnan(oracle.block_reward(tv, 5, 4, REWARD_BE))


def test_step_updates_the_used_arm_only():
    tv = np.array([[0.5, 0.5], [0.0, 0.2], [0.1, 0.1]])
    o = oracle.metasd_ucb_step(tv, [0, 0, 0], [1, -1, 0], np.zeros((3, 3), int), np.zeros((3, 3)), 2)
    assert o["pulls"].tolist() == [[0, 1, 0], [0, 0, 0], [1, 0, 0]]
    assert np.allclose(o["sums"], [[0, 0.5, 0], [0, 0, 0], [0.9, 0, 0]], atol=1e-15)
    assert o["arm"].tolist() == [0, 0, 1]
    assert np.isnan(o["reward"][1]) and o["err"] == 0


def test_faults_leave_the_state():
    tv = np.array([[np.nan, 0.1], [0.1, 0.1]])
    pulls = np.array([[1, 1], [1, 1]])
    sums = np.array([[0.5, 0.4], [0.5, 0.4]])
    o = oracle.metasd_ucb_step(tv, [0, 0], [0, 2], pulls, sums, 2)
    assert o["err"] == oracle.DEV_NONFINITE | oracle.DEV_ARM_OOB
    assert np.array_equal(o["pulls"], pulls) and np.array_equal(o["sums"], sums)
    assert o["arm"].tolist() == [0, 0]


def test_settles_on_the_best_stationary_arm():
    # Bernoulli rewards with means 0.3 / 0.5 / 0.8 fed as BD rows (TV = 1 - r):
    # UCB1 pulls the suboptimal arms O(log T) times.
    rng = np.random.default_rng(5)
    means = np.array([0.3, 0.5, 0.8])
    B, K, T = 4, 1, 1500
    pulls, sums = np.zeros((B, 3), int), np.zeros((B, 3))
    arm = np.full(B, -1)
    for _ in range(T):
        r = (rng.random(B) < means[np.maximum(arm, 0)]).astype(float)
        o = oracle.metasd_ucb_step((1.0 - r)[:, None], np.zeros(B, int), arm, pulls, sums, K)
        pulls, sums, arm = o["pulls"], o["sums"], o["arm"]
    assert np.all(pulls[:, 2] > 0.8 * T)
    # suboptimal pulls within UCB1's 8 ln T / gap^2 bound (+ 1 + pi^2 / 3)
    for i, gap in ((0, 0.5), (1, 0.3)):
        assert np.all(pulls[:, i] <= 8 * math.log(T) / gap ** 2 + 1 + math.pi ** 2 / 3)
    # BE on the same arms (accepted_len ~ Binomial(K, mean)) finds the same arm
    K = 4
    pulls, sums = np.zeros((1, 3), int), np.zeros((1, 3))
    arm = np.array([-1])
    for _ in range(T):
        acc = rng.binomial(K, means[max(arm[0], 0)], size=1)
        o = oracle.metasd_ucb_step(np.zeros((1, K)), acc, arm, pulls, sums, K, kind=REWARD_BE)
        pulls, sums, arm = o["pulls"], o["sums"], o["arm"]
    assert pulls[0, 2] > 0.7 * T
