"""Seeded Monte-Carlo and special-case pins of the full oracle (Philox path).

Enumeration pins the composition of the rules; these runs pin the randomness
machinery end to end (Philox keying, uniform conversions, Gumbel-max): the
emitted tokens over many independently keyed sequences must follow the target
law (chi-square over 10^6 trials; the KS gate of FlashSpec, Methodology s.3,
on 10,000 samples at alpha = 0.01).
"""
import numpy as np
import pytest
from hypothesis import given, settings, strategies as st
from scipy.stats import chisquare, kstest

import oracle
from tests.oracle_enum import row_probs
from workloads import bf16_bits_to_f32, f32_to_bf16_bits


def _tile(rows, B):
    return np.ascontiguousarray(np.broadcast_to(rows, (B,) + rows.shape))


def _draw_tokens(Q, n, rng):
    """n independent draft tuples x_i ~ Q_i (numpy RNG, not the verifier's)."""
    gamma, V = Q.shape
    out = np.empty((n, gamma), dtype=np.int32)
    for i in range(gamma):
        out[:, i] = rng.choice(V, size=n, p=Q[i] / Q[i].sum())
    return out


def _complete(tokens, accept_len, P, rng):
    """Extend each emitted prefix with target draws for the later positions."""
    n = tokens.shape[0]
    n_pos, V = P.shape
    full = np.empty((n, n_pos), dtype=np.int64)
    for m in range(n_pos):
        draws = rng.choice(V, size=n, p=P[m] / P[m].sum())
        keep = m <= accept_len
        full[:, m] = np.where(keep, tokens[:, m], draws)
    return full


@pytest.mark.slow
def test_single_draft_chi_square_1e6():
    V, gamma, T, n = 4, 2, 0.8, 1_000_000
    rng = np.random.default_rng(5)
    tg = f32_to_bf16_bits(rng.normal(0, 1.5, (gamma + 1, V)).astype(np.float32))
    dr = f32_to_bf16_bits((bf16_bits_to_f32(tg[:gamma]) + rng.normal(0, 1.0, (gamma, V)))
                          .astype(np.float32))
    P, Q = row_probs(tg, T), row_probs(dr, T)
    toks = _draw_tokens(Q, n, rng)
    r = oracle.verify(_tile(tg, n), _tile(dr, n), toks, np.full(n, T, np.float32),
                      seed=0, step=3, threads=8, with_logprobs=False)
    assert np.all(r["accept_len"] >= 0)
    full = _complete(r["tokens"], r["accept_len"], P, rng)
    idx = np.ravel_multi_index(full.T, (V,) * (gamma + 1))
    counts = np.bincount(idx, minlength=V ** (gamma + 1))
    expect = n * np.ravel(np.multiply.outer(np.multiply.outer(P[0], P[1]), P[2]))
    assert chisquare(counts, expect).pvalue > 1e-4
    # acceptance identity, statistically: P(accept at 0) = sum min(p0, q0)
    beta0 = np.minimum(P[0], Q[0]).sum()
    assert abs(np.mean(r["accept_len"] >= 1) - beta0) < 5 * np.sqrt(beta0 * (1 - beta0) / n)


def test_ks_gate_10000():
    """FlashSpec, Methodology s.3: KS, 10,000 samples, alpha = 0.01, comparing
    the first emitted token with the target law; a sampler that emits the
    draft's law instead must fail the same gate."""
    V, gamma, T, n = 64, 3, 1.0, 10_000
    rng = np.random.default_rng(9)
    tg = rng.normal(0, 2.0, (gamma + 1, V)).astype(np.float32)
    dr = (tg[:gamma] + rng.normal(0, 1.0, (gamma, V))).astype(np.float32)
    P, Q = row_probs(tg, T), row_probs(dr, T)
    toks = _draw_tokens(Q, n, rng)
    r = oracle.verify(_tile(tg, n), _tile(dr, n), toks, np.full(n, T, np.float32), seed=1,
                      step=0, threads=4, with_logprobs=False)
    # Continuous extension of a law on {0..V-1}: token + U(0,1) has the
    # piecewise-linear CDF below, which makes the KS statistic exact.
    below = np.concatenate([[0.0], np.cumsum(P[0])[:-1]])

    def cdf(x):
        x = np.asarray(x)
        i = np.clip(np.floor(x).astype(int), 0, V - 1)
        return np.clip(below[i] + P[0][i] * (x - i), 0.0, 1.0)

    jitter = rng.random(n)
    first = r["tokens"][:, 0] + jitter
    assert kstest(first, cdf).pvalue > 0.01
    wrong = toks[:, 0] + jitter  # the draft's law, not the target's
    assert kstest(wrong, cdf).pvalue < 0.01


@pytest.mark.slow
def test_multidraft_chi_square():
    V, L, K, T, n = 4, 2, 3, 0.6, 300_000
    rng = np.random.default_rng(21)
    tg = rng.normal(0, 1.5, (L + 1, V)).astype(np.float32)
    dr = (tg[:L] + rng.normal(0, 1.0, (L, V))).astype(np.float32)
    P, Q = row_probs(tg, T), row_probs(dr, T)
    toks = np.stack([_draw_tokens(Q, n, rng) for _ in range(K)], axis=1)
    r = oracle.verify_multidraft(_tile(tg, n), _tile(dr, n), toks, np.full(n, T, np.float32),
                                 seed=0, step=5, threads=8)
    assert np.all(r["accept_len"] >= 0)
    full = _complete(r["tokens"], r["accept_len"], P, rng)
    idx = np.ravel_multi_index(full.T, (V,) * (L + 1))
    counts = np.bincount(idx, minlength=V ** (L + 1))
    expect = n * np.ravel(np.multiply.outer(np.multiply.outer(P[0], P[1]), P[2]))
    assert chisquare(counts, expect).pvalue > 1e-4
    # the accepted prefix is the prefix of the reported draft
    for b in range(200):
        t, a = r["accept_len"][b], r["draft_index"][b]
        if t > 0:
            assert np.array_equal(r["tokens"][b, :t], toks[b, a, :t])
        else:
            assert a == -1


def test_greedy_is_argmax_matching():
    """T = 0: accept while the draft token is the target argmax (numpy argmax,
    lowest index on ties); the correction is the argmax where it stops."""
    rng = np.random.default_rng(3)
    B, gamma, V = 64, 4, 50
    tg = np.round(rng.normal(0, 1, (B, gamma + 1, V)) * 2).astype(np.float32)  # ties
    dr = tg[:, :gamma] + rng.normal(0, 0.5, (B, gamma, V)).astype(np.float32)
    gt = np.argmax(tg, axis=-1)
    toks = np.where(rng.random((B, gamma)) < 0.7, gt[:, :gamma],
                    rng.integers(0, V, (B, gamma))).astype(np.int32)
    r = oracle.verify(tg, dr, toks, np.zeros(B, np.float32))
    for b in range(B):
        j = next((i for i in range(gamma) if toks[b, i] != gt[b, i]), gamma)
        assert r["accept_len"][b] == j
        assert list(r["tokens"][b, :j]) == list(toks[b, :j])
        assert r["tokens"][b, j] == gt[b, j]
        assert np.all(r["tokens"][b, j + 1:] == -1)
        assert np.all(np.isnan(r["lp"][b]))


def test_multidraft_greedy_longest_prefix():
    rng = np.random.default_rng(4)
    B, K, L, V = 40, 3, 4, 20
    tg = rng.normal(0, 1, (B, L + 1, V)).astype(np.float32)
    dr = tg[:, :L] + rng.normal(0, 0.3, (B, L, V)).astype(np.float32)
    gt = np.argmax(tg, axis=-1)
    toks = np.where(rng.random((B, K, L)) < 0.75, gt[:, None, :L],
                    rng.integers(0, V, (B, K, L))).astype(np.int32)
    r = oracle.verify_multidraft(tg, dr, toks, np.zeros(B, np.float32))
    for b in range(B):
        lens = []
        for k in range(K):
            n = 0
            while n < L and toks[b, k, n] == gt[b, n]:
                n += 1
            lens.append(n)
        tau = max(lens)
        assert r["accept_len"][b] == tau
        assert r["draft_index"][b] == (lens.index(tau) if tau > 0 else -1)
        assert r["tokens"][b, tau] == gt[b, tau]


def test_invalid_sequences():
    rng = np.random.default_rng(8)
    B, gamma, V = 6, 3, 10
    tg = rng.normal(0, 1, (B, gamma + 1, V)).astype(np.float32)
    dr = rng.normal(0, 1, (B, gamma, V)).astype(np.float32)
    toks = rng.integers(0, V, (B, gamma)).astype(np.int32)
    temps = np.ones(B, np.float32)
    temps[0] = -1.0
    temps[1] = np.nan
    temps[2] = np.inf
    toks[3, 1] = V  # out of range
    tg[4, 2, 3] = np.nan
    r = oracle.verify(tg, dr, toks, temps)
    for b in range(5):
        assert r["accept_len"][b] == -1 and np.all(r["tokens"][b] == -1)
    assert r["accept_len"][5] >= 0


def test_keyed_by_seed_step_row_position():
    """The same inputs under the same (seed, step) give the same outputs; a new
    step or seed re-keys the draws; a sequence's outputs do not depend on the
    rest of the batch."""
    rng = np.random.default_rng(10)
    B, gamma, V = 32, 4, 40
    tg = rng.normal(0, 1, (B, gamma + 1, V)).astype(np.float32)
    dr = (tg[:, :gamma] + rng.normal(0, 1.0, (B, gamma, V))).astype(np.float32)
    toks = rng.integers(0, V, (B, gamma)).astype(np.int32)
    temps = np.ones(B, np.float32)
    a = oracle.verify(tg, dr, toks, temps, seed=5, step=9)
    b = oracle.verify(tg, dr, toks, temps, seed=5, step=9, threads=4)
    assert np.array_equal(a["tokens"], b["tokens"])
    c = oracle.verify(tg, dr, toks, temps, seed=5, step=10)
    d = oracle.verify(tg, dr, toks, temps, seed=6, step=9)
    assert not np.array_equal(a["tokens"], c["tokens"])
    assert not np.array_equal(a["tokens"], d["tokens"])
    sub = oracle.verify(tg[7:8], dr[7:8], toks[7:8], temps[7:8], seed=5, step=9)
    # row index is part of the key: a lone sequence is sequence 0 of its batch
    e = oracle.verify(np.concatenate([tg[7:8], tg[:3]]), np.concatenate([dr[7:8], dr[:3]]),
                      np.concatenate([toks[7:8], toks[:3]]), temps[:4], seed=5, step=9)
    assert np.array_equal(sub["tokens"][0], e["tokens"][0])


@settings(max_examples=60, deadline=None)
@given(B=st.integers(1, 5), gamma=st.integers(1, 6), V=st.sampled_from([1, 2, 7, 16, 33]),
       T=st.sampled_from([0.0, 0.1, 0.7, 1.0, 3.0]), bf16=st.booleans(),
       seed=st.integers(0, 2**31 - 1))
def test_oracle_invariants(B, gamma, V, T, bf16, seed):
    """FlashSpec, Methodology s.3 (property-based tests over batch sizes and
    speculation lengths): 0 <= accept_len <= gamma, the accepted tokens are the
    draft prefix, the emitted token is in range, padding is -1."""
    rng = np.random.default_rng(seed)
    tg = rng.normal(0, 2, (B, gamma + 1, V)).astype(np.float32)
    dr = (tg[:, :gamma] + rng.normal(0, 1, (B, gamma, V))).astype(np.float32)
    if bf16:
        tg, dr = f32_to_bf16_bits(tg), f32_to_bf16_bits(dr)
    toks = rng.integers(0, V, (B, gamma)).astype(np.int32)
    r = oracle.verify(tg, dr, toks, np.full(B, T, np.float32), seed=seed, step=seed % 1000)
    for b in range(B):
        j = r["accept_len"][b]
        assert 0 <= j <= gamma
        assert np.array_equal(r["tokens"][b, :j], toks[b, :j])
        assert 0 <= r["tokens"][b, j] < V
        assert np.all(r["tokens"][b, j + 1:] == -1)


@settings(max_examples=40, deadline=None)
@given(B=st.integers(1, 3), K=st.sampled_from([1, 2, 5, 32]), L=st.sampled_from([1, 2, 7, 64]),
       V=st.sampled_from([1, 2, 5, 17]), T=st.sampled_from([0.0, 0.1, 0.7, 1.0]),
       bf16=st.booleans(), seed=st.integers(0, 2**31 - 1))
def test_multidraft_oracle_invariants(B, K, L, V, T, bf16, seed):
    """SpecTr-GBV, Algorithm 1, up to the largest K and L the interface takes:
    0 <= tau <= L; with tau > 0 the output starts with the first tau tokens
    of the reported draft; the emitted token is in range; padding is -1."""
    rng = np.random.default_rng(seed)
    tg = rng.normal(0, 2, (B, L + 1, V)).astype(np.float32)
    dr = (tg[:, :L] + rng.normal(0, 1, (B, L, V))).astype(np.float32)
    if bf16:
        tg, dr = f32_to_bf16_bits(tg), f32_to_bf16_bits(dr)
    # drafts share prefixes often (small V), which exercises the skip rules
    toks = rng.integers(0, V, (B, K, L)).astype(np.int32)
    r = oracle.verify_multidraft(tg, dr, toks, np.full(B, T, np.float32), seed=seed,
                                 step=seed % 1000)
    for b in range(B):
        tau, a = int(r["accept_len"][b]), int(r["draft_index"][b])
        assert 0 <= tau <= L
        if tau > 0:
            assert 0 <= a < K
            assert np.array_equal(r["tokens"][b, :tau], toks[b, a, :tau])
        else:
            assert a == -1  # no draft's token was kept
        assert 0 <= r["tokens"][b, tau] < V
        assert np.all(r["tokens"][b, tau + 1:] == -1)
