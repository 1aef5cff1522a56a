"""GPU parity on edge inputs: masked vocabularies, extreme logit magnitudes
and temperatures, drafts identical to the target (every token accepted, the
bonus draw for every sequence), many tiny rows.  The CUDA path through the C
ABI against the oracle: bit-exact accept lengths and token ids (logged ties
excluded), log-probs within 1e-5."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_85_b200 as sv
import workloads
from tests.parity import compare, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _gpu(st, seed, step):
    acc, tok, lp, lq = sv.spec_verify(st.target, st.draft, st.tokens, st.temps, seed=seed,
                                      step=step, with_logprobs=True)
    torch.cuda.synchronize()
    return {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
            "lp": lp.cpu().numpy(), "lq": lq.cpu().numpy()}


@pytest.mark.parametrize("B,gamma,V,dtype,T,scale", [
    (6, 4, 5000, "bf16", [0.7, 1.0, 0.0], 3.0),
    (5, 3, 3001, "f32", [0.01, 0.05], 20.0),
    (4, 5, 2049, "f32", [1.0, 0.4], 300.0),
])
def test_masked_vocabulary_and_extreme_scales(B, gamma, V, dtype, T, scale):
    """The upper 40% of every row is -inf (a padded vocabulary): whole tiles and
    whole Philox blocks hold nothing; the draft tokens are redrawn from the
    masked draft rows."""
    st = workloads.make_custom(B, gamma, V, dtype=dtype, seed=V, T=T, device=DEV,
                               target_scale=scale, noise=0.8)
    cut = (V * 6) // 10
    st.target[..., cut:] = float("-inf")
    st.draft[..., cut:] = float("-inf")
    g = torch.Generator(device=DEV)
    g.manual_seed(V + 1)
    toks = workloads.sample_tokens(st.draft, st.temps, 1, g)[:, 0].contiguous()
    st = workloads.Step(st.target, st.draft, toks, st.temps, 0)
    for step in (0, 3):
        compare(_gpu(st, 5, step), run_oracle(st, 5, step))


def test_identical_drafts_accept_every_token():
    """p = q at every position: every draft token is accepted and the token at
    gamma is the bonus draw from the target row gamma."""
    st = workloads.make_custom(8, 5, 4097, dtype="bf16", seed=5, T=[0.7, 1.0, 0.4], device=DEV,
                               noise=0.0)
    for step in (1, 2):
        g = _gpu(st, 2, step)
        compare(g, run_oracle(st, 2, step))
        assert (g["accept_len"] == 5).all()
        assert (g["tokens"][:, 5] >= 0).all()


def test_many_tiny_rows():
    st = workloads.make_custom(300, 3, 5, dtype="bf16", seed=9, T=[0.0, 0.4, 1.0], device=DEV)
    compare(_gpu(st, 1, 0), run_oracle(st, 1, 0))


def test_forced_rejection_near_equal_rows():
    """The residual draw where it is most fragile: the draft row equals the
    target row up to N(0, 1e-3) noise, except at the first draft token -- a
    low-probability entry boosted by +2 in the draft row, so it is rejected
    with probability about 0.86 -- and the correction token is drawn from
    max(p - q, 0), a difference of nearly equal probabilities.  Many seeds
    and steps; ties the oracle logs (its band widens with (p + q) / (p - q))
    are excluded and counted."""
    from tests.parity import TieLedger
    ledger = TieLedger("near-equal residual draws")
    B, gamma, V = 256, 2, 3001
    residual = 0
    for seed in (1, 2, 3):
        s = workloads.make_custom(B, gamma, V, dtype="f32", seed=seed, T=[1.0, 0.7], device=DEV,
                                  target_scale=2.0, noise=1e-3)
        x = s.target[:, 0].argmin(dim=-1)
        s.draft[torch.arange(B, device=DEV), 0, x] += 2.0
        s.tokens[:, 0] = x.to(torch.int32)
        for step in (0, 1):
            g = _gpu(s, seed, step)
            ledger.add(compare(g, run_oracle(s, seed, step)))
            residual += int((g["accept_len"] == 0).sum())
    assert residual > 0.7 * 6 * B  # the draws are mostly residual ones
    ledger.check(max_rate=0.05, slack=5)
