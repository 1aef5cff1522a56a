"""Single-draft kernel paths on the GPU: which kernels a shape takes, and
that the two paths give the same verification.

Small batches whose row slices fit in shared memory take the
one-cluster-per-sequence kernel; other shapes take the row kernel and the
draw kernel.  The kernels that ran are read from the CUDA profiler's
activity records.  Each path is compared with the oracle (bit-exact
accept lengths and token ids, logged ties excluded, log-probs within 1e-5),
and the same sequences verified as a small batch and as the first
sequences of a larger batch must agree (the Philox streams are keyed by the
sequence index, so they are the same streams)."""
import numpy as np
import pytest
import torch
from torch.profiler import ProfilerActivity, profile

import speculative_decoding_verification_85_b200 as sv
import workloads
from tests.parity import TieLedger, compare, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _run(target, draft, tokens, temps, seed, step):
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        acc, tok, lp, lq = sv.spec_verify(target, draft, tokens, temps, seed=seed, step=step,
                                          with_logprobs=True)
        torch.cuda.synchronize()
    names = {e.name for e in prof.events() if e.device_type == torch.autograd.DeviceType.CUDA}
    out = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
           "lp": lp.cpu().numpy(), "lq": lq.cpu().numpy()}
    return out, names


def _kernels(names):
    k = set()
    for n in names:
        for key in ("sd_cluster_kernel", "rows_kernel", "draw_kernel"):
            if key in n:
                k.add(key)
    return k


@pytest.mark.parametrize("B,gamma,V,dtype,T", [
    (1, 4, 32000, "f32", [1.0]),
    (16, 5, 32000, "bf16", [0.7, 1.0]),
    (7, 3, 5000, "bf16", [0.0, 0.4, 1.0]),
    (3, 12, 2500, "f32", [0.1, 1.0]),
    (5, 2, 700, "bf16", [1.0, 0.0]),
])
def test_small_batches_take_the_cluster_kernel(B, gamma, V, dtype, T):
    st = workloads.make_custom(B, gamma, V, dtype=dtype, seed=B * 1000 + V, T=T, device=DEV)
    led = TieLedger(f"cluster path B={B} gamma={gamma} V={V} {dtype}")
    for step in range(3):
        gpu, names = _run(st.target, st.draft, st.tokens, st.temps, 5, step)
        assert _kernels(names) == {"sd_cluster_kernel"}, names
        led.add(compare(gpu, run_oracle(st, 5, step)))
    led.check()


def test_the_two_paths_agree_on_the_same_sequences():
    B, small, gamma, V = 160, 6, 4, 32000
    st = workloads.make_custom(B, gamma, V, dtype="bf16", seed=77, T=[0.0, 0.4, 0.7, 1.0],
                               device=DEV)
    sub = workloads.Step(st.target[:small].contiguous(), st.draft[:small].contiguous(),
                         st.tokens[:small].contiguous(), st.temps[:small].contiguous(), st.step)
    led = TieLedger("cluster path vs streaming path")
    for step in range(4):
        big, names_big = _run(st.target, st.draft, st.tokens, st.temps, 9, step)
        assert _kernels(names_big) == {"rows_kernel", "draw_kernel"}, names_big
        few, names_few = _run(sub.target, sub.draft, sub.tokens, sub.temps, 9, step)
        assert _kernels(names_few) == {"sd_cluster_kernel"}, names_few
        ora = run_oracle(sub, 9, step)
        led.add(compare(few, ora))
        led.add(compare({k: v[:small] for k, v in big.items()}, ora))
        # both paths: identical outputs except where the oracle logged a tie
        tie = ora["tie"]
        for b in range(small):
            if tie[b]:
                continue
            assert few["accept_len"][b] == big["accept_len"][b]
            assert np.array_equal(few["tokens"][b], big["tokens"][b])
        np.testing.assert_allclose(few["lp"], big["lp"][:small], rtol=0, atol=2e-5)
    led.check()


@pytest.mark.parametrize("B,K,L,V,T,csize", [
    (2, 3, 4, 32000, [0.4, 1.0], 16),
    (24, 3, 4, 32000, [0.0, 0.4, 1.0], 8),
])
def test_multidraft_cluster_sizes(B, K, L, V, T, csize):
    """Multi-draft: 16-CTA clusters when the batch's clusters fit one wave,
    else 8; both against the oracle."""
    st = workloads.make_custom(B, L, V, dtype="bf16", seed=B * 7 + K, T=T, K=K, device=DEV)
    led = TieLedger(f"multi-draft {csize}-CTA clusters B={B} K={K} L={L}")
    for step in range(2):
        with profile(activities=[ProfilerActivity.CUDA]) as prof:
            acc, tok, di = sv.spec_verify_multidraft(st.target, st.draft, st.tokens, st.temps,
                                                     seed=3, step=step)
            torch.cuda.synchronize()
        names = [e.name for e in prof.events() if "md_cluster_kernel" in e.name]
        assert names and all(n.split("(")[0].rstrip(">").endswith(f" {csize}") for n in names), names
        gpu = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
               "draft_index": di.cpu().numpy()}
        led.add(compare(gpu, run_oracle(st, 3, step), check_logprobs=False))
    led.check()
