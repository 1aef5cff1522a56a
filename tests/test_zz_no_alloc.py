"""spec_verify_noalloc through the C ABI: the same results as spec_verify on
two calls in a row, with the scratch space taken from the library's fixed
array instead of a caller workspace.  Collected last on purpose; it must also
pass alone in a fresh process."""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_85_b200 as sv
import workloads
from parity import LOGP_ATOL

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def _outputs(B, g):
    return (torch.empty(B, dtype=torch.int32, device=DEV),
            torch.empty((B, g + 1), dtype=torch.int32, device=DEV),
            torch.empty((B, g), dtype=torch.float32, device=DEV),
            torch.empty((B, g), dtype=torch.float32, device=DEV))


def _same(a, b):
    acc_a, tok_a, lp_a, lq_a = (t.cpu().numpy() for t in a)
    acc_b, tok_b, lp_b, lq_b = (t.cpu().numpy() for t in b)
    assert np.array_equal(acc_a, acc_b)
    assert np.array_equal(tok_a, tok_b)
    for x, y in ((lp_a, lp_b), (lq_a, lq_b)):
        fin = np.isfinite(y)
        assert np.array_equal(np.isfinite(x), fin)
        assert np.max(np.abs(x[fin].astype(np.float64) - y[fin]), initial=0.0) <= LOGP_ATOL


def test_noalloc_matches_spec_verify_on_two_calls():
    steps = [workloads.make_custom(16, 5, 32000, dtype="bf16", seed=41, T=[0.7, 1.0, 0.0],
                                   device=DEV),
             workloads.make_custom(9, 3, 5003, dtype="f32", seed=42, T=[0.4, 1.0], device=DEV)]
    outs = [_outputs(s.target.shape[0], s.target.shape[1] - 1) for s in steps]
    refs = []
    for k, st in enumerate(steps):
        refs.append(sv.spec_verify(st.target, st.draft, st.tokens, st.temps, seed=7, step=k,
                                   with_logprobs=True))
    torch.cuda.synchronize()
    free_before = None
    for k, (st, out) in enumerate(zip(steps, outs)):
        if k == 1:
            free_before = torch.cuda.mem_get_info()[0]
        sv.spec_verify_noalloc(st.target, st.draft, st.tokens, st.temps, seed=7, step=k,
                               out_accept_len=out[0], out_tokens=out[1], out_target_logp=out[2],
                               out_draft_logp=out[3])
        torch.cuda.synchronize()
        if k == 1:
            assert torch.cuda.mem_get_info()[0] == free_before  # the call allocated nothing
        _same(out, refs[k])
