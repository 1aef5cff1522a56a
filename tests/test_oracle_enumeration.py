"""Exact-enumeration pins of the oracle (CPU only).

The theorem on the pages (FlashSpec, Significance: Theorem 1; SpecTr-GBV,
Contributions: the method preserves the target's output law) fixes the law of
the emitted tokens: completed with target draws, it must equal target-only
sampling, prod_j P_j, in the position-wise model used here.  Enumerating every
branch of the oracle gives that law exactly, so a dropped term, a wrong sign
or a wrong index anywhere in the acceptance rule, the residual, the
multi-draft weights or the control flow shows up as a difference far above
rounding (1e-12).
"""
import numpy as np
import pytest

import oracle
from tests.oracle_enum import (Script, extend_to_full, multidraft_law, product_law,
                               row_probs, single_draft_law)
from tests import oracle_enum
from workloads import f32_to_bf16_bits


def _rows(seed, n, V, scale=1.5, dtype="f32"):
    rng = np.random.default_rng(seed)
    t = rng.normal(0, scale, (n, V)).astype(np.float32)
    return f32_to_bf16_bits(t) if dtype == "bf16" else t


def _pair(seed, gamma, V, dtype="f32", noise=1.0):
    rng = np.random.default_rng(seed)
    tg = rng.normal(0, 1.5, (gamma + 1, V)).astype(np.float32)
    dr = (tg[:gamma] + rng.normal(0, noise, (gamma, V))).astype(np.float32)
    if dtype == "bf16":
        return f32_to_bf16_bits(tg), f32_to_bf16_bits(dr)
    return tg, dr


SINGLE_CASES = [(4, 1, 1.0, "f32"), (4, 2, 0.7, "bf16"), (4, 3, 1.3, "f32"),
                (8, 2, 0.5, "bf16"), (16, 1, 1.0, "f32"), (3, 3, 2.0, "bf16"),
                (5, 2, 0.1, "f32")]


@pytest.mark.parametrize("V,gamma,T,dtype", SINGLE_CASES)
def test_single_draft_law_equals_target(V, gamma, T, dtype):
    tg, dr = _pair(V * 31 + gamma, gamma, V, dtype)
    law = single_draft_law(tg, dr, T)
    P = row_probs(tg, T)
    full = extend_to_full(law, P)
    assert abs(full.sum() - 1.0) < 1e-12
    np.testing.assert_allclose(full, product_law(P), rtol=0, atol=1e-12)


@pytest.mark.parametrize("V,gamma,T", [(4, 3, 1.0), (6, 2, 0.6)])
def test_acceptance_identity_and_geometric_law(V, gamma, T):
    """P(accept at i | accepted before) = sum_v min(p_i, q_i); hence
    P(accept_len >= i) = prod_{m<i} beta_m (the geometric accept-length law of
    Speculative Speculative Decoding, Saguaro s.1) and E[accept_len] =
    sum_i prod_{m<i} beta_m."""
    tg, dr = _pair(100 + V, gamma, V)
    law = single_draft_law(tg, dr, T)
    P, Q = row_probs(tg, T), row_probs(dr, T)
    beta = np.minimum(P[:gamma], Q).sum(axis=1)
    tail = [sum(w for (j, _), w in law.items() if j >= i) for i in range(gamma + 1)]
    for i in range(gamma + 1):
        assert abs(tail[i] - np.prod(beta[:i])) < 1e-12
    mean = sum(j * w for (j, _), w in law.items())
    assert abs(mean - sum(np.prod(beta[:i]) for i in range(1, gamma + 1))) < 1e-12


class _BiasedCoin(Script):
    def coin(self, h, tag, b, k, pos):
        return super().coin(min(1.0, 1.05 * h), tag, b, k, pos)


class _FlatCategorical(Script):
    def categorical(self, logw, tag, b, pos):
        return super().categorical(np.where(np.isfinite(logw), 0.0, -np.inf), tag, b, pos)


@pytest.mark.parametrize("script", [_BiasedCoin, _FlatCategorical])
def test_enumeration_detects_planted_mistakes(script):
    """The pin has power: a 5% bias in the acceptance coin, or a correction
    draw that ignores the residual weights, breaks the law by far more than
    the tolerance."""
    tg, dr = _pair(7, 2, 5)
    law = single_draft_law(tg, dr, 0.8, script_cls=script)
    P = row_probs(tg, 0.8)
    full = extend_to_full(law, P)
    assert np.max(np.abs(full - product_law(P))) > 1e-4


MULTI_CASES = [(2, 1, 1, 1.0), (3, 1, 2, 0.8), (4, 1, 3, 0.5), (3, 2, 1, 1.0),
               (3, 2, 2, 1.0), (4, 2, 2, 0.7), (3, 2, 3, 1.2)]


@pytest.mark.parametrize("V,L,K,T", MULTI_CASES)
def test_multidraft_law_equals_target(V, L, K, T):
    tg, dr = _pair(1000 + V * 7 + L * 3 + K, L, V)
    law = multidraft_law(tg, dr, K, T)
    P = row_probs(tg, T)
    full = extend_to_full(law, P)
    assert abs(full.sum() - 1.0) < 1e-12
    np.testing.assert_allclose(full, product_law(P), rtol=0, atol=1e-12)


def test_multidraft_hand_case_with_rejected_set():
    """A case where a draft repeats a rejected token (the set H is used):
    P0 = (.2, .5, .3), Q0 = (.5, .3, .2), K = 2, L = 1."""
    tg = np.log(np.array([[0.2, 0.5, 0.3], [0.3, 0.3, 0.4]], np.float32))
    dr = np.log(np.array([[0.5, 0.3, 0.2]], np.float32))
    law = multidraft_law(tg, dr, 2, 1.0)
    P = row_probs(tg, 1.0)
    full = extend_to_full(law, P)
    np.testing.assert_allclose(full.sum(axis=1), P[0], rtol=0, atol=1e-12)


@pytest.mark.parametrize("V,T", [(3, 1.0), (5, 0.6)])
def test_multidraft_k1_l1_is_textbook_sd(V, T):
    """K = 1, L = 1 reduces to standard speculative sampling: same joint law of
    (accept_len, tokens) as the single-draft verifier with gamma = 1."""
    tg, dr = _pair(2000 + V, 1, V)
    a = single_draft_law(tg, dr, T)
    b = multidraft_law(tg, dr, 1, T)
    assert set(a) == set(b)
    for key in a:
        assert abs(a[key] - b[key]) < 1e-12


def _mean_len(law):
    return sum(j * w for (j, _), w in law.items())


def test_block_verification_not_shorter_than_tokenwise():
    """K = 1 is single-draft greedy block verification; its expected accepted
    length is at least that of token-wise verification on the same drafts."""
    tg, dr = _pair(3001, 2, 4, noise=1.5)
    assert _mean_len(multidraft_law(tg, dr, 1, 1.0)) >= _mean_len(
        single_draft_law(tg, dr, 1.0)) - 1e-12


def test_multidraft_accept_length_monotone_in_K():
    """SpecTr-GBV, ablation on K: acceptance grows with the number of drafts."""
    tg, dr = _pair(4001, 2, 3, noise=1.5)
    means = [_mean_len(multidraft_law(tg, dr, K, 1.0)) for K in (1, 2, 3)]
    assert means[0] <= means[1] + 1e-12 <= means[2] + 2e-12
    assert means[2] > means[0]


# ------------------------------------------------ per-draft (prefix-conditioned) rows
PREFIX_CASES = [(2, 1, 2, 1.0), (3, 1, 3, 0.8), (2, 2, 2, 1.0), (3, 2, 2, 0.7), (2, 2, 3, 1.2)]


@pytest.mark.parametrize("V,L,K,T", PREFIX_CASES)
def test_per_draft_rows_law_equals_prefix_conditioned_target(V, L, K, T):
    """SpecTr-GBV, Algorithm 1 with each draft weighed by the rows of its own
    prefix: with K i.i.d. drafts from an autoregressive draft model, the
    emitted tokens (completed by the target for later positions) follow the
    autoregressive target model exactly."""
    tctx, dctx = oracle_enum.prefix_model(V, L, 3000 + 17 * V + 5 * L + K)
    law = oracle_enum.multidraft_law_prefix_model(tctx, dctx, V, L, K, T)
    want, p = oracle_enum.prefix_target_law(tctx, V, L, T)
    full = oracle_enum.extend_prefix_law(law, p, V, L)
    assert abs(full.sum() - 1.0) < 1e-12
    np.testing.assert_allclose(full, want, rtol=0, atol=1e-12)


def test_per_draft_enumeration_detects_rows_of_the_wrong_draft():
    """Planted mistake: every draft weighed with draft 0's rows.  The law
    drifts away from the target model, so the enumeration above has power."""
    V, L, K, T = 3, 2, 2, 1.0
    tctx, dctx = oracle_enum.prefix_model(V, L, 77)

    def first_drafts_rows(tc, dc, drafts, L_):
        tg, dr = oracle_enum.per_draft_rows(tc, dc, drafts, L_)
        return np.repeat(tg[:1], len(drafts), axis=0), np.repeat(dr[:1], len(drafts), axis=0)

    law = oracle_enum.multidraft_law_prefix_model(tctx, dctx, V, L, K, T, rows=first_drafts_rows)
    want, p = oracle_enum.prefix_target_law(tctx, V, L, T)
    full = oracle_enum.extend_prefix_law(law, p, V, L)
    assert np.max(np.abs(full - want)) > 1e-4


@pytest.mark.parametrize("T", [0.0, 0.4, 1.0])
@pytest.mark.parametrize("bf16", [False, True])
def test_per_draft_rows_with_equal_sets_match_shared_rows(T, bf16):
    """Per-draft rows that are K copies of the shared rows give exactly the
    shared-row result (same keyed randomness, same arithmetic)."""
    rng = np.random.default_rng(11)
    B, K, L, V = 4, 5, 4, 37
    tg = rng.normal(0, 2, (B, L + 1, V)).astype(np.float32)
    dr = (tg[:, :L] + rng.normal(0, 0.8, (B, L, V))).astype(np.float32)
    if bf16:
        tg, dr = f32_to_bf16_bits(tg), f32_to_bf16_bits(dr)
    toks = rng.integers(0, V, (B, K, L)).astype(np.int32)
    toks[:, 1:, :2] = toks[:, :1, :2]  # shared prefixes exercise the skip rules
    temps = np.full(B, T, np.float32)
    a = oracle.verify_multidraft(tg, dr, toks, temps, seed=9, step=4)
    tgk = np.ascontiguousarray(np.repeat(tg[:, None], K, axis=1))
    drk = np.ascontiguousarray(np.repeat(dr[:, None], K, axis=1))
    b = oracle.verify_multidraft(tgk, drk, toks, temps, seed=9, step=4)
    for key in ("accept_len", "tokens", "draft_index", "tie"):
        assert np.array_equal(a[key], b[key]), key
