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
