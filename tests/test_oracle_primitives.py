"""Pins for the oracle's primitives (CPU only).

Each check compares the oracle with something other than itself: published
known-answer vectors, exact dyadic values, library routines (scipy, numpy),
or closed forms.
"""
import math
import os

import numpy as np
import pytest
from scipy.special import log_softmax

import oracle
from workloads import bf16_bits_to_f32, f32_to_bf16_bits

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def test_philox_known_answers():
    rows = []
    with open(os.path.join(GOLDEN, "philox4x32_10_kat.txt")) as f:
        for line in f:
            if line.strip() and not line.startswith("#"):
                rows.append([int(t, 16) for t in line.split()])
    assert len(rows) == 3
    for r in rows:
        out = oracle.philox4x32_10(r[0:4], r[4:6])
        assert [int(v) for v in out] == r[6:10]


def test_stream_word_keying():
    # key = (lo32(seed), hi32(seed)); counter = (c0, b, lo32(step), tag|k|pos)
    seed, step = 0x0123456789ABCDEF, 77
    for (tag, b, k, pos, c0, w) in [(1, 3, 0, 2, 2, 0), (2, 5, 0, 4, 1000, 3), (3, 0, 7, 1, 1, 0)]:
        ctr = [c0, b, step, (tag << 24) | (k << 12) | pos]
        key = [seed & 0xFFFFFFFF, seed >> 32]
        assert oracle.stream_word(seed, step, tag, b, k, pos, c0, w) == int(
            oracle.philox4x32_10(ctr, key)[w])


@pytest.mark.parametrize("x", [0, 1, 255, 256, 0x12345678, 0xFFFFFEFF, 0xFFFFFF00, 0xFFFFFFFF])
def test_uniform_conversions_exact(x):
    ua = oracle.u01_accept(x)
    assert ua == (x >> 8) / 2**24 and 0.0 <= ua < 1.0
    ug = oracle.u01_gumbel(x)
    n = 2 * (x >> 9) + 1
    assert ug == n / 2**24 and 0.0 < ug < 1.0 and n % 2 == 1
    assert np.float32(ug) == ug  # exactly representable in fp32


def test_bf16_decode():
    x = np.array([0.0, -0.0, 1.0, -2.5, 3.1415926, 1e-30, -1e30, np.inf, -np.inf], np.float32)
    bits = f32_to_bf16_bits(x)
    for b, ref in zip(bits, bf16_bits_to_f32(bits)):
        got = oracle.bf16_to_f32(int(b))
        assert (got == ref) or (math.isnan(got) and math.isnan(ref))


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
@pytest.mark.parametrize("T", [0.1, 0.7, 1.0, 2.0])
def test_row_logprobs_is_log_softmax_of_scaled_row(dtype, T):
    """FlashSpec, Methodology s.1: temperature before the log-softmax."""
    rng = np.random.default_rng(int(T * 10))
    z = rng.normal(0, 3.0, 1000).astype(np.float32)
    z[[3, 17]] = -np.inf  # probability zero entries are allowed
    row = f32_to_bf16_bits(z) if dtype == "bf16" else z
    zf = bf16_bits_to_f32(row) if dtype == "bf16" else z
    s = (zf / np.float32(T)).astype(np.float32)  # fp32 scaling
    ref = log_softmax(s.astype(np.float64))
    lp = oracle.row_logprobs(row, T)
    fin = np.isfinite(ref)
    assert np.array_equal(fin, np.isfinite(lp))
    np.testing.assert_allclose(lp[fin], ref[fin], rtol=0, atol=2e-6 * max(1.0, 1.0 / T))
    # the common bug the page warns about: log_softmax(z) / T is a different law
    wrong = log_softmax(zf.astype(np.float64)) / T
    if T != 1.0:
        assert np.max(np.abs(wrong[fin] - lp[fin])) > 1e-2
    assert abs(np.exp(lp[fin]).sum() - 1.0) < 1e-12


def test_row_invalid_cases():
    V = 16
    z = np.zeros(V, np.float32)
    z[5] = np.nan
    assert oracle.row_logprobs(z, 1.0) is None and oracle.row_argmax(z) == -1
    z = np.zeros(V, np.float32)
    z[2] = np.inf
    assert oracle.row_logprobs(z, 1.0) is None and oracle.row_argmax(z) == -1
    z = np.full(V, -np.inf, np.float32)
    assert oracle.row_logprobs(z, 1.0) is None and oracle.row_argmax(z) == -1


@pytest.mark.parametrize("seed", range(5))
def test_row_argmax_first_index(seed):
    rng = np.random.default_rng(seed)
    z = np.round(rng.normal(0, 1, 500) * 2).astype(np.float32)  # many ties
    assert oracle.row_argmax(z) == int(np.argmax(z))
    zb = f32_to_bf16_bits(z)
    assert oracle.row_argmax(zb) == int(np.argmax(bf16_bits_to_f32(zb)))


def test_residual_logw_matches_definition():
    """Speculative Speculative Decoding, Saguaro sampling: r ~ max(p - q, 0)."""
    rng = np.random.default_rng(1)
    lp = log_softmax(rng.normal(0, 2, 300))
    lq = log_softmax(rng.normal(0, 2, 300))
    lq[7] = -np.inf
    out, n = oracle.residual_logw(lp, lq)
    r = np.maximum(np.exp(lp) - np.exp(lq), 0.0)
    assert n == int(np.count_nonzero(r > 0))
    pos = r > 0
    np.testing.assert_allclose(np.exp(out[pos]), r[pos], rtol=1e-12, atol=0)
    assert np.all(out[~pos] == -np.inf)
    assert out[7] == lp[7]  # q = 0 -> residual equals p


def test_gumbel_argmax_law():
    """Gumbel-max over the keyed stream draws from softmax(logw)."""
    from scipy.stats import chisquare
    logw = np.array([0.3, -1.0, 1.2, -np.inf, 0.0, -0.4])
    p = np.exp(logw - logw.max())
    p /= p.sum()
    n = 200_000
    counts = np.zeros(logw.size)
    for b in range(n):
        y, _ = oracle.gumbel_argmax(logw, 7, 11, oracle.TAG_GUMBEL, b, 3)
        counts[y] += 1
    assert counts[3] == 0
    m = p > 0
    assert chisquare(counts[m], n * p[m]).pvalue > 1e-3


def test_gumbel_argmax_deterministic_and_keyed():
    logw = np.zeros(64)
    a = oracle.gumbel_argmax(logw, 0, 0, oracle.TAG_GUMBEL, 0, 0)[0]
    assert a == oracle.gumbel_argmax(logw, 0, 0, oracle.TAG_GUMBEL, 0, 0)[0]
    draws = {oracle.gumbel_argmax(logw, 0, s, oracle.TAG_GUMBEL, 0, 0)[0] for s in range(200)}
    assert len(draws) > 40  # different steps give different keys


def test_group_race_law():
    """The two-level race draws from the normalised weights: entry
    frequencies over three groups (the last one ragged) against w / W,
    chi-square over heavy entries at group edges and the rest of each group."""
    from scipy.stats import chisquare
    G = oracle.RACE_GROUP
    V = 2 * G + 300
    rng = np.random.default_rng(5)
    w = rng.uniform(0.0, 1.0, V) * 1e-3
    w[rng.random(V) < 0.3] = 0.0
    heavy = [0, 5, G - 1, G, 2 * G - 1, 2 * G, V - 1]
    w[heavy] = [0.4, 0.2, 0.3, 0.25, 0.1, 0.05, 0.15]
    logw = np.full(V, -np.inf)
    logw[w > 0] = np.log(w[w > 0])
    cat = np.full(V, -1)
    for i, v in enumerate(heavy):
        cat[v] = i
    for g in range(3):
        rest = np.arange(g * G, min(V, (g + 1) * G))
        rest = rest[cat[rest] < 0]
        cat[rest] = len(heavy) + g
    ncat = len(heavy) + 3
    p = np.bincount(cat, weights=w, minlength=ncat) / w.sum()
    n = 40_000
    counts = np.zeros(ncat)
    for b in range(n):
        y, _ = oracle.group_race(logw, 3, 9, oracle.TAG_GUMBEL, b, 1)
        assert w[y] > 0
        counts[cat[y]] += 1
    assert chisquare(counts, n * p).pvalue > 1e-3


def test_group_race_with_one_group_is_the_plain_race():
    """Support inside one group (or V <= RACE_GROUP): the group level has one
    candidate and the entry level uses the plain race's noise, so the draw
    equals svo_gumbel_argmax under every key."""
    G = oracle.RACE_GROUP
    rng = np.random.default_rng(6)
    V = 3 * G
    logw = np.full(V, -np.inf)
    logw[G + 17:2 * G - 3] = rng.normal(0.0, 1.5, G - 20)
    small = rng.normal(0.0, 1.0, 700)
    for s in range(300):
        assert (oracle.group_race(logw, 11, s, oracle.TAG_GUMBEL, 2, 3)[0]
                == oracle.gumbel_argmax(logw, 11, s, oracle.TAG_GUMBEL, 2, 3)[0])
        assert (oracle.group_race(small, 11, s, oracle.TAG_GUMBEL, 2, 3)[0]
                == oracle.gumbel_argmax(small, 11, s, oracle.TAG_GUMBEL, 2, 3)[0])


def test_group_race_levels_are_independent():
    """Two groups of equal total weight, one entry of each heavy: the chosen
    group must be a fair coin whatever entry the entry noise favours, i.e.
    the group choice is independent of the entry level (a shared noise
    source would tie them)."""
    G = oracle.RACE_GROUP
    V = 2 * G
    logw = np.full(V, -np.inf)
    logw[3] = 0.0
    logw[G + 3] = 0.0  # same offset within its group: same entry counter word layout
    n = 20_000
    g1 = sum(oracle.group_race(logw, 1, 2, oracle.TAG_GUMBEL, b, 0)[0] >= G for b in range(n))
    assert abs(g1 / n - 0.5) < 4.0 * math.sqrt(0.25 / n)


def test_group_race_empty_support():
    logw = np.full(3000, -np.inf)
    assert oracle.group_race(logw, 0, 0, oracle.TAG_GUMBEL, 0, 0)[0] == -1
