"""Pins of the oracle's draft-selection bandit (FlashSpec, Methodology s.2:
draft choice as a K-armed bandit rewarded by the fraction of accepted draft
tokens, with UCB1 and Thompson Sampling).

Each pin is a fact fixed outside the oracle: distribution laws against
scipy, the deterministic form of the UCB1 pull bound of Auer, Cesa-Bianchi
and Fischer (2002), their expected-regret bound, and the regret ordering of
the two policies that the page reports.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
from scipy import stats

import oracle

BETA_TAG, TRIAL_TAG = 5, 6


def test_uniforms_are_uniform_on_the_open_interval():
    u = np.array([oracle.bandit_uniform(3, c, 7, 1, BETA_TAG, h) for c in range(20000)
                  for h in (0, 1)])
    assert u.min() > 0.0 and u.max() < 1.0
    assert stats.kstest(u, "uniform").pvalue > 1e-3
    # distinct counters give distinct draws; the key matters
    assert len(set(u.tolist())) == len(u)
    assert oracle.bandit_uniform(3, 0, 7, 1, BETA_TAG) != oracle.bandit_uniform(4, 0, 7, 1, BETA_TAG)


@pytest.mark.parametrize("alpha", [1.0, 1.5, 4.0, 30.0, 500.0])
def test_gamma_sampler_law(alpha):
    x = np.array([oracle.gamma_sample(alpha, 11, r, 3) for r in range(20000)])
    assert np.all(x > 0)
    assert stats.kstest(x, stats.gamma(alpha).cdf).pvalue > 1e-3
    assert math.isnan(oracle.gamma_sample(0.5, 11, 0, 0))  # shapes below 1 are not taken


@pytest.mark.parametrize("a,b", [(1.0, 1.0), (3.0, 7.0), (50.0, 20.0), (1.0, 400.0)])
def test_beta_sampler_law(a, b):
    x = np.array([oracle.beta_sample(a, b, 5, r, 2) for r in range(20000)])
    assert np.all((x > 0) & (x < 1))
    assert stats.kstest(x, stats.beta(a, b).cdf).pvalue > 1e-3


def test_trial_success_rate_is_the_reward():
    n = 40000
    for r in (0.0, 0.13, 0.5, 0.87, 1.0):
        k = sum(oracle.thompson_trial(r, 9, t, 1) for t in range(n))
        if r in (0.0, 1.0):
            assert k == r * n
        else:
            assert abs(k - r * n) < 4.5 * math.sqrt(n * r * (1 - r))


def _run(policy, means, T, seed, bernoulli=True):
    """Pseudo-regret and pull counts of a run on a Bernoulli (or exact) bandit."""
    rng = np.random.default_rng(seed)
    b = oracle.BanditOracle(len(means), policy, seed)
    best = max(means)
    regret = 0.0
    for _ in range(T):
        a = b.select()
        r = float(rng.random() < means[a]) if bernoulli else means[a]
        b.update(a, r)
        regret += best - means[a]
    return regret, b.pulls


def test_ucb1_plays_every_arm_once_then_obeys_the_deterministic_pull_bound():
    means = [0.2, 0.5, 0.45, 0.9]
    b = oracle.BanditOracle(4, "ucb1")
    order = []
    T = 5000
    last_best = None  # (n, pulls) just before the last pull of the best arm
    for _ in range(T):
        before = b.pulls.copy()
        a = b.select()
        order.append(a)
        if a == 3:
            last_best = (int(before.sum()), before)
        b.update(a, means[a])
    assert order[:4] == [0, 1, 2, 3]
    n, before = last_best
    for j, m in enumerate(means):
        d = max(means) - m
        if d > 0:
            # with exact rewards, a suboptimal arm j is chosen with n_j earlier
            # pulls only if sqrt(2 ln n / n_j) >= Delta_j: n_j <= 2 ln T / Delta^2 + 1
            assert b.pulls[j] <= 2 * math.log(T) / d ** 2 + 1
            # and whenever the best arm is chosen, sqrt(2 ln n / n_j) <=
            # Delta_j + sqrt(2 ln n / n_best): a lower bound on n_j
            lo = 2 * math.log(n) / (d + math.sqrt(2 * math.log(n) / before[3])) ** 2
            assert b.pulls[j] >= lo
    assert b.pulls[3] > 0.9 * T


def test_ucb1_regret_within_the_expected_regret_bound():
    means, T = [0.4, 0.55, 0.7], 10000
    gaps = [max(means) - m for m in means if m < max(means)]
    bound = sum(8 * math.log(T) / d for d in gaps) + (1 + math.pi ** 2 / 3) * sum(gaps)
    regs = [_run("ucb1", means, T, s)[0] for s in range(3)]
    assert np.mean(regs) < bound


def test_thompson_regret_below_ucb1_and_concentrates():
    """The page reports lower cumulative regret for Thompson Sampling than for
    UCB1 over 10,000 rounds with three arms."""
    means, T = [0.4, 0.55, 0.7], 10000
    ts = [_run("thompson", means, T, s) for s in range(3)]
    ucb = [_run("ucb1", means, T, s)[0] for s in range(3)]
    assert np.mean([r for r, _ in ts]) < np.mean(ucb)
    for _, pulls in ts:
        assert pulls[2] > 0.9 * T


def test_policies_depend_only_on_the_reward_history():
    """The selected arm sequence is a function of (seed, rewards so far): two
    runs fed the same rewards choose the same arms, whatever else happens."""
    for policy in ("ucb1", "thompson"):
        a, b = oracle.BanditOracle(3, policy, 4), oracle.BanditOracle(3, policy, 4)
        rng = np.random.default_rng(1)
        for _ in range(300):
            x, y = a.select(), b.select()
            assert x == y
            r = float(rng.random())
            a.update(x, r)
            b.update(y, r)
