"""The library's draft-selection bandit (include/sv_bandit.h, host code in
libspecverify.so) against the oracle's (FlashSpec, Methodology s.2): the
same arm at every step for the same seed and reward history, the reward of a
verified step, argument errors, and the cost of a select + update."""
from __future__ import annotations

import time

import numpy as np
import pytest

import oracle
import speculative_decoding_verification_85_b200 as sv


@pytest.mark.parametrize("policy", ["ucb1", "thompson"])
@pytest.mark.parametrize("K", [1, 2, 3, 8])
def test_same_arms_as_the_oracle(policy, K):
    rng = np.random.default_rng(K * 7 + len(policy))
    means = rng.random(K)
    for seed in (0, 12345, 2**63 + 11):
        lib_b = sv.Bandit(K, policy, seed)
        ora = oracle.BanditOracle(K, policy, seed)
        for t in range(1500):
            a, b = lib_b.select(), ora.select()
            assert a == b, (policy, K, seed, t)
            # Bernoulli rewards, and fractional ones as a verified step gives
            r = float(rng.random() < means[a]) if t % 2 else float(rng.integers(0, 6)) / 5
            lib_b.update(a, r)
            ora.update(b, r)
        pulls, sums = lib_b.stats()
        assert np.array_equal(pulls.numpy(), ora.pulls)
        assert np.array_equal(sums.numpy(), ora.sums)


def test_reward_of_a_verified_step():
    b = sv.Bandit(2, "ucb1")
    b.update_from_accept(1, np.array([4, 0, -1, 2, 5], np.int32), 5)
    pulls, sums = b.stats()
    assert pulls.tolist() == [0, 1]
    # invalid sequences (-1) carry nothing: mean of 4/5, 0, 2/5, 5/5
    assert abs(float(sums[1]) - (0.8 + 0.0 + 0.4 + 1.0) / 4) < 1e-15
    b.update_from_accept(0, np.array([-1, -1], np.int32), 5)  # nothing valid: no update
    b.update_from_accept(0, np.zeros(0, np.int32), 5)
    assert b.stats()[0].tolist() == [0, 1]


def test_argument_errors():
    with pytest.raises(sv.SpecVerifyError):
        sv.Bandit(0)
    with pytest.raises(sv.SpecVerifyError):
        sv.Bandit(2000)
    with pytest.raises(ValueError):
        sv.Bandit(2, "greedy")
    b = sv.Bandit(3, "thompson", 1)
    for arm, r in ((3, 0.5), (-1, 0.5), (0, 1.5), (0, -0.1), (0, float("nan"))):
        with pytest.raises(sv.SpecVerifyError, match="INVALID_ARG"):
            b.update(arm, r)
    with pytest.raises(sv.SpecVerifyError):
        b.update_from_accept(0, np.array([6], np.int32), 5)  # accept_len > gamma
    with pytest.raises(sv.SpecVerifyError):
        b.update_from_accept(0, np.array([1], np.int32), 0)
    assert b.stats()[0].tolist() == [0, 0, 0]  # failed calls change nothing


def test_select_update_cost(capsys):
    """Host cost of one select + update (printed; the selector runs once per
    decoding step, next to a verification of tens of microseconds)."""
    for policy in ("ucb1", "thompson"):
        b = sv.Bandit(3, policy, 5)
        n = 20000
        t0 = time.perf_counter()
        for i in range(n):
            a = b.select()
            b.update(a, 0.5)
        us = (time.perf_counter() - t0) / n * 1e6
        with capsys.disabled():
            print(f"\nbandit {policy}: {us:.2f} us per select + update (K = 3, via ctypes)")
        assert us < 200.0


# ------------------------------------------- library-only pins (no oracle)
def test_ucb1_pull_count_bound_from_the_index():
    """UCB1 with deterministic rewards (arm 0 always 0.9, arm 1 always 0.1):
    from the index mean + sqrt(2 ln n / n_j), arm 1 is pulled only while
    sqrt(2 ln n / n_1) >= 0.8 + sqrt(2 ln n / n_0), so after n pulls
    2 ln n / (0.8 + sqrt(2 ln n / n_0))^2 - 1 <= n_1 <= 2 ln n / 0.64 + 1."""
    b = sv.Bandit(2, "ucb1", 0)
    n = 10000
    for _ in range(n):
        a = b.select()
        b.update(a, 0.9 if a == 0 else 0.1)
    pulls, _ = b.stats()
    n0, n1 = int(pulls[0]), int(pulls[1])
    assert n0 + n1 == n
    lo = 2 * np.log(n) / (0.8 + np.sqrt(2 * np.log(n) / n0)) ** 2 - 1
    hi = 2 * np.log(n) / 0.64 + 1
    assert lo <= n1 <= hi, (n1, lo, hi)


def test_thompson_choice_frequency_is_the_beta_comparison():
    """Thompson Sampling with successes / failures S = (3, 2), F = (1, 2):
    each select draws Beta(S_j + 1, F_j + 1) per arm independently and picks
    the larger, so arm 0 wins with probability P(X > Y), X ~ Beta(4, 2),
    Y ~ Beta(3, 3) (numerical integral).  Rewards 1 and 0 are always a
    success and a failure."""
    from scipy import integrate, stats
    b = sv.Bandit(2, "thompson", 99)
    for arm, r in ((0, 1.0), (0, 1.0), (0, 1.0), (0, 0.0), (1, 1.0), (1, 1.0), (1, 0.0),
                   (1, 0.0)):
        b.update(arm, r)
    X, Y = stats.beta(4, 2), stats.beta(3, 3)
    p, _ = integrate.quad(lambda x: X.pdf(x) * Y.cdf(x), 0.0, 1.0)
    n = 4000
    wins = sum(b.select() == 0 for _ in range(n))
    sd = np.sqrt(p * (1 - p) / n)
    assert abs(wins / n - p) < 4.5 * sd, (wins / n, p)
    assert b.stats()[0].tolist() == [4, 4]  # select alone changes no statistics
