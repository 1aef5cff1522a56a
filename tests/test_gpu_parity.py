"""GPU parity: the CUDA path through the C ABI against the oracle (B200 only).

Bit-exact accept lengths and token ids (logged ties excluded), log-probs
within 1e-5, on seeded inputs: small ragged shapes that span several chunks
and a ragged tail, every workload at its full size, and the edge cases.
"""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_85_b200 as sv
import workloads
from tests.parity import TieLedger, compare, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def gpu_single(st, seed=0, step=0, ws=None, logprobs=True):
    acc, tok, lp, lq = sv.spec_verify(st.target, st.draft, st.tokens, st.temps, seed=seed,
                                      step=step, workspace=ws, with_logprobs=logprobs)
    torch.cuda.synchronize()
    out = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy()}
    if logprobs:
        out["lp"], out["lq"] = lp.cpu().numpy(), lq.cpu().numpy()
    return out


def gpu_multi(st, seed=0, step=0, ws=None):
    acc, tok, idx = sv.spec_verify_multidraft(st.target, st.draft, st.tokens, st.temps, seed=seed,
                                              step=step, workspace=ws)
    torch.cuda.synchronize()
    return {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
            "draft_index": idx.cpu().numpy()}


def widen(st, min_b=80):
    """The batch tiled to at least min_b sequences: more clusters than one wave
    holds, so the row and draw kernels take it (small batches of narrow rows
    take the one-cluster-per-sequence kernel)."""
    r = -(-min_b // st.target.shape[0])
    cat = lambda x: torch.cat([x] * r, dim=0).contiguous()  # noqa: E731
    return workloads.Step(cat(st.target), cat(st.draft), cat(st.tokens), cat(st.temps), st.step)


SMALL = [
    # B, gamma, V, dtype, temperatures
    (1, 4, 32000, "f32", 1.0),
    (3, 1, 1, "bf16", 1.0),
    (5, 2, 2, "f32", [0.0, 0.7]),
    (4, 3, 7, "bf16", [0.1, 1.0, 0.0]),
    (7, 5, 33, "f32", [0.7, 1.0]),
    (9, 8, 1000, "bf16", [0.0, 0.1, 0.4, 0.7, 1.0]),
    (6, 33, 257, "bf16", [1.0, 2.0]),
    (2, 64, 129, "f32", [0.7]),
    (17, 4, 8195, "bf16", [0.7, 1.0, 0.0]),
    (3, 5, 40003, "bf16", [0.1, 0.7, 1.0]),
    (4, 6, 20001, "f32", [0.4, 1.0]),
]


@pytest.mark.parametrize("wide", [False, True])
@pytest.mark.parametrize("B,gamma,V,dtype,T", SMALL)
def test_small_shapes(B, gamma, V, dtype, T, wide):
    if wide and V > 10000:
        pytest.skip("the wide copies of the long rows only repeat the larger tests")
    for seed in (0, 123):
        st = workloads.make_custom(B, gamma, V, dtype=dtype, seed=seed + V, T=T, device=DEV,
                                   target_scale=2.5, noise=0.8)
        if wide:
            st = widen(st)
        for step in (0, 7):
            g = gpu_single(st, seed=seed, step=step)
            o = run_oracle(st, seed, step)
            compare(g, o)


@pytest.mark.parametrize("cfg,steps", [(0, range(1)), (1, range(100)), (2, range(20)),
                                       (4, range(20))])
def test_workloads_full_size(cfg, steps):
    """Every single-draft workload at its full shape -- every step of C0 and
    C1, the first 20 steps of C2 and C4 -- through the same call and workspace
    reuse that the benchmark times."""
    c = workloads.get(cfg)
    v = sv.Verifier(DEV)
    ledger = TieLedger(c.name)
    for step in steps:
        st = workloads.make_step(c, step, device=DEV)
        acc, tok, lp, lq = v.verify(st.target, st.draft, st.tokens, st.temps, seed=0, step=step,
                                    with_logprobs=True)
        torch.cuda.synchronize()
        g = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
             "lp": lp.cpu().numpy(), "lq": lq.cpu().numpy()}
        ledger.add(compare(g, run_oracle(st, 0, step)))
    ledger.check()


def test_multidraft_full_size():
    """The multi-draft workload at its full shape, all 100 steps."""
    c = workloads.get(3)
    v = sv.Verifier(DEV)
    ledger = TieLedger(c.name)
    for step in range(100):
        st = workloads.make_step(c, step, device=DEV)
        acc, tok, idx = v.verify_multidraft(st.target, st.draft, st.tokens, st.temps, seed=0,
                                            step=step)
        torch.cuda.synchronize()
        g = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
             "draft_index": idx.cpu().numpy()}
        ledger.add(compare(g, run_oracle(st, 0, step)))
    ledger.check()


@pytest.mark.parametrize("B,K,L,V,dtype,T", [
    (4, 1, 1, 50, "f32", [1.0]),
    (5, 3, 2, 7, "bf16", [0.7, 0.1]),
    (6, 4, 5, 1000, "bf16", [0.1, 0.4, 0.7, 0.0]),
    (3, 8, 3, 4097, "f32", [1.0, 0.0]),
    (2, 2, 9, 300, "bf16", [0.5]),
])
def test_multidraft_small(B, K, L, V, dtype, T):
    for seed in (1, 2):
        st = workloads.make_custom(B, L, V, dtype=dtype, seed=seed * 31 + V, T=T, K=K, device=DEV,
                                   target_scale=2.0, noise=0.6)
        g = gpu_multi(st, seed=seed, step=3)
        compare(g, run_oracle(st, seed, 3))


@pytest.mark.parametrize("wide", [False, True])
def test_invalid_sequences(wide):
    st = workloads.make_custom(8, 4, 300, dtype="bf16", seed=5, T=1.0, device=DEV)
    st.temps[0] = -1.0
    st.temps[1] = float("nan")
    st.temps[2] = float("inf")
    st.tokens[3, 2] = 300
    st.tokens[4, 0] = -5
    st.target[5, 2, 17] = float("nan")
    st.draft[6, 1, :] = float("-inf")
    if wide:
        st = widen(st)
    g = gpu_single(st)
    o = run_oracle(st, 0, 0)
    compare(g, o)
    for b in range(st.target.shape[0]):
        if b % 8 < 7:
            assert g["accept_len"][b] == -1 and np.all(g["tokens"][b] == -1)
        else:
            assert g["accept_len"][b] >= 0


@pytest.mark.parametrize("wide", [False, True])
def test_inf_entries_and_plus_inf(wide):
    st = workloads.make_custom(6, 3, 500, dtype="f32", seed=9, T=[1.0, 0.0], device=DEV)
    st.target[0, :, ::3] = float("-inf")  # probability-zero entries
    st.draft[1, :, ::5] = float("-inf")
    st.target[2, 1, 10] = float("inf")     # invalid row
    st.target[3, 0, 4] = float("inf")      # invalid greedy row
    if wide:
        st = widen(st)
    g = gpu_single(st)
    compare(g, run_oracle(st, 0, 0))
    assert g["accept_len"][2] == -1 and g["accept_len"][3] == -1


@pytest.mark.parametrize("wide", [False, True])
def test_unaligned_rows_and_offsets(wide):
    """Rows whose start is not 16-byte aligned (odd V, sliced base pointers)."""
    for V in (31, 1001, 8193):
        st = workloads.make_custom(5, 3, V, dtype="bf16", seed=V, T=[0.7, 1.0, 0.0], device=DEV)
        if wide:
            st = widen(st)
        big_t = torch.empty(st.target.numel() + 3, dtype=st.target.dtype, device=DEV)
        big_d = torch.empty(st.draft.numel() + 5, dtype=st.draft.dtype, device=DEV)
        t = big_t[3:].view(st.target.shape)
        d = big_d[5:].view(st.draft.shape)
        t.copy_(st.target)
        d.copy_(st.draft)
        st2 = workloads.Step(t, d, st.tokens, st.temps, 0)
        compare(gpu_single(st2), run_oracle(st, 0, 0))


def test_workspace_reuse_and_determinism():
    st = workloads.make_custom(16, 5, 32000, dtype="bf16", seed=4, T=[0.7, 1.0], device=DEV)
    need = max(sv.workspace_size(16, 5, 32000, sv.BF16), sv.workspace_size(40, 7, 3000, sv.F32),
               sv.multidraft_workspace_size(3, 3, 4, 2000, sv.BF16))
    ws = torch.zeros(need, dtype=torch.uint8, device=DEV)
    a = gpu_single(st, seed=3, step=11, ws=ws)
    b = gpu_single(st, seed=3, step=11, ws=ws)
    assert np.array_equal(a["tokens"], b["tokens"]) and np.array_equal(a["lp"], b["lp"])
    # the counters sit at fixed offsets and are left at zero: calls of other
    # shapes (and the multi-draft entry point) reuse the same buffer
    st2 = workloads.make_custom(4, 2, 1000, dtype="bf16", seed=5, T=1.0, device=DEV)
    compare(gpu_single(st2, ws=ws), run_oracle(st2, 0, 0))
    st3 = workloads.make_custom(40, 7, 3000, dtype="f32", seed=6, T=[0.7, 0.0], device=DEV)
    compare(gpu_single(st3, ws=ws[: sv.workspace_size(40, 7, 3000, sv.F32)]),
            run_oracle(st3, 0, 0))
    sm = workloads.make_custom(3, 4, 2000, dtype="bf16", seed=7, T=[0.4, 0.7], K=3, device=DEV)
    compare(gpu_multi(sm, ws=ws), run_oracle(sm, 0, 0))
    compare(gpu_single(st, seed=3, step=11, ws=ws), run_oracle(st, 3, 11))


def test_host_buffer_entry_point_matches_device():
    st = workloads.make_custom(8, 4, 5000, dtype="bf16", seed=8, T=[0.7, 1.0, 0.0], device=DEV)
    dev = gpu_single(st, seed=2, step=5)
    B, g1, V = st.target.shape
    staging = torch.zeros(sv.staging_size(B, g1 - 1, V, sv.BF16), dtype=torch.uint8, device=DEV)
    h = [x.cpu().pin_memory() for x in (st.target, st.draft, st.tokens, st.temps)]
    acc, tok, lp, lq = sv.spec_verify_host(*h, staging=staging, seed=2, step=5, with_logprobs=True)
    assert np.array_equal(acc.numpy(), dev["accept_len"])
    assert np.array_equal(tok.numpy(), dev["tokens"])
    np.testing.assert_array_equal(lp.numpy(), dev["lp"])


def test_abi_errors():
    st = workloads.make_custom(2, 3, 100, dtype="bf16", seed=1, device=DEV)
    with pytest.raises(sv.SpecVerifyError, match="INVALID_ARG"):
        sv.spec_verify(st.target, st.draft, st.tokens, st.temps, step=2**32)
    small = torch.zeros(16, dtype=torch.uint8, device=DEV)
    with pytest.raises(sv.SpecVerifyError, match="WORKSPACE"):
        sv.spec_verify(st.target, st.draft, st.tokens, st.temps, workspace=small)
    with pytest.raises(ValueError):
        sv.spec_verify(st.target.cpu(), st.draft, st.tokens, st.temps)


def test_ks_gate_on_gpu_draws():
    """FlashSpec, Methodology s.3, on the CUDA path: the first emitted token
    over 10,000 independently keyed sequences follows the target law."""
    from scipy.stats import kstest
    n, gamma, V, T = 10_000, 3, 64, 1.0
    rng = np.random.default_rng(12)
    tg = rng.normal(0, 2.0, (gamma + 1, V)).astype(np.float32)
    dr = (tg[:gamma] + rng.normal(0, 1.0, (gamma, V))).astype(np.float32)
    P = np.exp(tg[0] - tg[0].max())
    P /= P.sum()
    Q = np.exp(dr - dr.max(axis=1, keepdims=True))
    Q /= Q.sum(axis=1, keepdims=True)
    toks = np.stack([rng.choice(V, size=n, p=Q[i]) for i in range(gamma)], axis=1)
    target = torch.tensor(np.broadcast_to(tg, (n,) + tg.shape).copy(), device=DEV)
    draft = torch.tensor(np.broadcast_to(dr, (n,) + dr.shape).copy(), device=DEV)
    acc, tok, _, _ = sv.spec_verify(target, draft, torch.tensor(toks, dtype=torch.int32, device=DEV),
                                    torch.full((n,), T, device=DEV), seed=4, step=1)
    first = tok[:, 0].cpu().numpy() + rng.random(n)
    below = np.concatenate([[0.0], np.cumsum(P)[:-1]])

    def cdf(x):
        i = np.clip(np.floor(x).astype(int), 0, V - 1)
        return np.clip(below[i] + P[i] * (x - i), 0.0, 1.0)

    assert kstest(first, cdf).pvalue > 0.01


def _per_draft_rows(B, K, L, V, dtype, seed, T, device):
    """A row set per draft with prefix-consistent rows: draft k's rows at
    position i depend only on its prefix x_k[0..i) (drafts that share a prefix
    see equal rows, and every draft's row 0 is the same), as a
    prefix-conditioned model gives them.  The rows of a prefix come from a
    generator seeded by (seed, b, i, prefix); each draft's tokens from its own
    generator, so the drafts are independent."""
    g = torch.Generator(device="cpu")
    g.manual_seed(seed)
    base_t = torch.randn((L + 1, V), generator=g) * 2.0
    base_d = base_t[:L] + torch.randn((L, V), generator=g) * 0.6
    temps = torch.tensor([T[b % len(T)] for b in range(B)], dtype=torch.float32)
    toks = torch.empty((B, K, L), dtype=torch.int32)
    tgt = torch.empty((B, K, L + 1, V))
    drf = torch.empty((B, K, L, V))
    for b in range(B):
        for k in range(K):
            gk = torch.Generator(device="cpu")
            gk.manual_seed((seed * 1000003 + b * 131 + k) & 0x7FFFFFFF)
            prefix = []
            for i in range(L + 1):
                gi = torch.Generator(device="cpu")
                gi.manual_seed(hash((seed, b, i) + tuple(prefix)) & 0x7FFFFFFF)
                shift = torch.randn(V, generator=gi) * 0.8
                tgt[b, k, i] = base_t[i] + shift
                if i < L:
                    drf[b, k, i] = base_d[i] + shift + torch.randn(V, generator=gi) * 0.3
                    if float(temps[b]) > 0:
                        q = torch.softmax(drf[b, k, i] / float(temps[b]), -1)
                        x = int(torch.multinomial(q, 1, generator=gk))
                    else:
                        x = int(drf[b, k, i].argmax())
                    toks[b, k, i] = x
                    prefix.append(x)
    if dtype == "bf16":
        tgt, drf = tgt.to(torch.bfloat16), drf.to(torch.bfloat16)
    return workloads.Step(tgt.contiguous().to(device), drf.contiguous().to(device),
                          toks.to(device), temps.to(device), 0)


@pytest.mark.parametrize("B,K,L,V,dtype,T", [
    (4, 1, 1, 50, "f32", [1.0]),
    (5, 3, 2, 7, "bf16", [0.7, 0.1]),
    (6, 4, 5, 1000, "bf16", [0.1, 0.4, 0.7, 0.0]),
    (8, 4, 5, 32000, "bf16", [0.1, 0.4, 0.7]),
    (3, 8, 3, 4097, "f32", [1.0, 0.0]),
])
def test_multidraft_per_draft_rows(B, K, L, V, dtype, T):
    """A row set per draft (target [B, K, L+1, V]): the CUDA path against the
    oracle's per-draft verification."""
    for seed in (1, 2):
        st = _per_draft_rows(B, K, L, V, dtype, seed * 7 + V, T, DEV)
        g = gpu_multi(st, seed=seed, step=5)
        compare(g, run_oracle(st, seed, 5))


def test_multidraft_per_draft_equal_copies_match_shared_rows():
    """K equal copies of one row set give the shared-row results bit for bit."""
    st = workloads.make_custom(6, 5, 3000, dtype="bf16", seed=77, T=[0.4, 0.7, 0.0], K=4,
                               device=DEV, target_scale=2.0, noise=0.6)
    K = st.tokens.shape[1]
    rows = workloads.Step(st.target[:, None].expand(-1, K, -1, -1).contiguous(),
                          st.draft[:, None].expand(-1, K, -1, -1).contiguous(), st.tokens,
                          st.temps, 0)
    a = gpu_multi(st, seed=3, step=9)
    b = gpu_multi(rows, seed=3, step=9)
    for key in ("accept_len", "tokens", "draft_index"):
        assert np.array_equal(a[key], b[key]), key
