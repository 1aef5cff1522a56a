"""Seeded property sweep of the CUDA path against the oracle (B200 only).

Hypothesis draws the shape (B, gamma, V), the logit dtype, the temperatures
(greedy, low, unit and high, mixed within a batch), the logit scale and the
draft noise; the draws are derandomised, so every run checks the same
bounded set of cases.  Every case compares bit-exact accept lengths and token
ids (logged ties excluded) and log-probabilities within 1e-5, single-draft
and multi-draft.
"""
import pytest
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

import speculative_decoding_verification_85_b200 as sv
import workloads
from tests.parity import TieLedger, compare, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"

TEMPS = st.sampled_from([0.0, 0.05, 0.3, 0.7, 1.0, 2.5])
SETTINGS = settings(max_examples=40, deadline=None, derandomize=True, database=None,
                    suppress_health_check=list(HealthCheck))

_single = TieLedger("single-draft sweep")
_multi = TieLedger("multi-draft sweep")


@SETTINGS
@given(B=st.integers(1, 40), gamma=st.integers(1, 12),
       V=st.one_of(st.integers(1, 300), st.integers(301, 70000)),
       dtype=st.sampled_from(["bf16", "f32"]), T=st.lists(TEMPS, min_size=1, max_size=4),
       scale=st.sampled_from([0.5, 2.0, 6.0]), noise=st.sampled_from([0.0, 0.05, 0.6, 2.0]),
       seed=st.integers(0, 2**31 - 1), step=st.integers(0, 2**32 - 1))
def test_single_draft_sweep(B, gamma, V, dtype, T, scale, noise, seed, step):
    s = workloads.make_custom(B, gamma, V, dtype=dtype, seed=seed, T=T, device=DEV,
                              target_scale=scale, noise=noise)
    acc, tok, lp, lq = sv.spec_verify(s.target, s.draft, s.tokens, s.temps, seed=seed,
                                      step=step, with_logprobs=True)
    torch.cuda.synchronize()
    g = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(), "lp": lp.cpu().numpy(),
         "lq": lq.cpu().numpy()}
    _single.add(compare(g, run_oracle(s, seed, step)))


@SETTINGS
@given(B=st.integers(1, 12), K=st.integers(1, 6), L=st.integers(1, 8),
       V=st.one_of(st.integers(1, 200), st.integers(201, 40000)),
       dtype=st.sampled_from(["bf16", "f32"]), T=st.lists(TEMPS, min_size=1, max_size=3),
       noise=st.sampled_from([0.0, 0.3, 1.0]), seed=st.integers(0, 2**31 - 1),
       step=st.integers(0, 2**32 - 1))
def test_multi_draft_sweep(B, K, L, V, dtype, T, noise, seed, step):
    s = workloads.make_custom(B, L, V, dtype=dtype, seed=seed, T=T, K=K, device=DEV,
                              target_scale=2.0, noise=noise)
    acc, tok, idx = sv.spec_verify_multidraft(s.target, s.draft, s.tokens, s.temps, seed=seed,
                                              step=step)
    torch.cuda.synchronize()
    g = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
         "draft_index": idx.cpu().numpy()}
    _multi.add(compare(g, run_oracle(s, seed, step)))


def test_sweep_tie_counts():
    """Runs after the two sweeps: their excluded (tie) counts stay small."""
    _single.check(max_rate=5e-3, slack=3)
    _multi.check(max_rate=5e-3, slack=3)
