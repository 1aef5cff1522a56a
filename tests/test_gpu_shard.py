"""Vocabulary-sharded verification on the GPU, against the oracle on the
whole rows.

The n ranks are emulated on one GPU: each rank's three calls run in turn on
its own column slice of the rows and its own workspace, and the two
exchanges are concatenations of the ranks' records in rank order (what an
all-gather delivers).  No kernel of one rank waits on another rank's.  Every
rank must end with the same outputs, and those are compared with the oracle
(bit-exact accept lengths and tokens, logged ties excluded, log-probs within
1e-5) and with the unsharded path on the same inputs.
"""
import numpy as np
import pytest
import torch

import speculative_decoding_verification_85_b200 as sv
import workloads
from tests.parity import TieLedger, compare, run_oracle

pytestmark = pytest.mark.gpu
DEV = "cuda:0"


def run_sharded(st, n, seed=0, step=0, bounds=None):
    """Every rank's outputs, as host arrays, in rank order."""
    B, g1, V = st.target.shape
    g = g1 - 1
    dt = sv.BF16 if st.target.dtype == torch.bfloat16 else sv.F32
    bounds = bounds or sv.vocab_shards(V, n)
    ranks = []
    for v0, Vs in bounds:
        assert Vs > 0
        t = st.target[:, :, v0:v0 + Vs].contiguous()
        d = st.draft[:, :, v0:v0 + Vs].contiguous()
        ws = torch.zeros(sv.workspace_size(B, g, Vs, dt), dtype=torch.uint8, device=DEV)
        ranks.append((v0, t, d, ws))
    stats = [sv.spec_verify_shard_stats(t, d, st.tokens, st.temps, V=V, v0=v0, workspace=ws)
             for v0, t, d, ws in ranks]
    all_stats = torch.cat(stats)
    outs, cands = [], []
    for v0, t, d, ws in ranks:
        acc, tok, lp, lq, cand = sv.spec_verify_shard_decide(
            t, d, st.tokens, st.temps, all_stats, V=V, v0=v0, nshards=len(ranks), workspace=ws,
            seed=seed, step=step, with_logprobs=True)
        outs.append((acc, tok, lp, lq))
        cands.append(cand)
    all_cands = torch.cat(cands)
    for acc, tok, _, _ in outs:
        sv.spec_verify_shard_pick(all_cands, nshards=len(ranks), out_accept_len=acc,
                                  out_tokens=tok)
    torch.cuda.synchronize()
    return [{"accept_len": a.cpu().numpy(), "tokens": t.cpu().numpy(), "lp": p.cpu().numpy(),
             "lq": q.cpu().numpy()} for a, t, p, q in outs]


def same_on_every_rank(res):
    for r in res[1:]:
        for k in ("accept_len", "tokens"):
            assert np.array_equal(r[k], res[0][k]), k
        for k in ("lp", "lq"):
            assert np.array_equal(r[k].view(np.uint32), res[0][k].view(np.uint32)), k


def unsharded(st, seed, step):
    acc, tok, lp, lq = sv.spec_verify(st.target, st.draft, st.tokens, st.temps, seed=seed,
                                      step=step, with_logprobs=True)
    torch.cuda.synchronize()
    return {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
            "lp": lp.cpu().numpy(), "lq": lq.cpu().numpy()}


CASES = [
    # B, gamma, V, dtype, temperatures, ranks
    (6, 4, 32000, "bf16", [0.0, 0.4, 0.7, 1.0], 2),
    (5, 3, 32000, "f32", [1.0, 0.1], 3),          # shards 11264, 11264, 9472
    (7, 5, 5000, "bf16", [0.7, 1.0, 0.0], 3),     # 2048, 2048, 904 (a ragged last shard)
    (4, 2, 3001, "f32", [0.4, 1.0], 2),           # odd widths: unaligned rows in the last shard
    (3, 6, 1500, "bf16", [1.0], 1),               # one rank: the whole row
    (9, 4, 20000, "bf16", [0.0], 4),              # all greedy
    (5, 64, 4096, "bf16", [0.7, 1.0], 4),         # the longest draft
]


@pytest.mark.parametrize("B,gamma,V,dtype,T,n", CASES)
def test_sharded_matches_oracle(B, gamma, V, dtype, T, n):
    st = workloads.make_custom(B, gamma, V, dtype=dtype, seed=B * 31 + V + n, T=T, device=DEV)
    led = TieLedger(f"vocab-sharded n={n} B={B} gamma={gamma} V={V} {dtype}")
    for step in range(3):
        res = run_sharded(st, n, seed=11, step=step)
        same_on_every_rank(res)
        ora = run_oracle(st, 11, step)
        led.add(compare(res[0], ora))
        # the unsharded path on the same inputs: identical outside logged ties
        one = unsharded(st, 11, step)
        for b in range(B):
            if ora["tie"][b]:
                continue
            assert one["accept_len"][b] == res[0]["accept_len"][b]
            assert np.array_equal(one["tokens"][b], res[0]["tokens"][b])
    led.check()


@pytest.mark.parametrize("cfg", ["c2", "c4"])
def test_sharded_full_size_rows(cfg):
    """A full-size vocabulary (128256 / 151936 bf16) split over 8 ranks, on a
    slice of the workload's batch; sequences sampled for the oracle."""
    st = workloads.make_step(cfg, 0, device=DEV, B=24)
    led = TieLedger(f"vocab-sharded {cfg} n=8")
    res = run_sharded(st, 8, seed=3, step=0)
    same_on_every_rank(res)
    led.add(compare(res[0], run_oracle(st, 3, 0)))
    led.check()


def test_shards_without_weight():
    """Low temperatures that leave most shards with no weight at all (their
    candidates carry none), the target's mass and the draft's in different
    shards, and q == p on whole sequences (every token accepted, the bonus
    draw)."""
    B, g, V = 8, 4, 9000
    st = workloads.make_custom(B, g, V, dtype="f32", seed=21, T=[1.0, 0.05, 0.7, 0.02],
                               device=DEV)
    st.draft[0] = st.target[0, :g]
    st.target[3, :, 8500] += 40.0  # the mass of sequence 3 sits in the last shard
    st.draft[3, :, 100] += 40.0    # ... and the draft's in the first
    st.target[7, :, 5000] += 40.0
    led = TieLedger("vocab-sharded shards without weight")
    for step in range(4):
        res = run_sharded(st, 3, seed=5, step=step)
        same_on_every_rank(res)
        led.add(compare(res[0], run_oracle(st, 5, step)))
    led.check()


def test_residual_vanishing_on_every_shard():
    """The draft row equals the target row except at the first draft token x,
    set 30 below the row's maximum and raised by 2 in the draft: x is rejected
    with probability 1 - e^-2, and max(p - q, 0) is zero in fp32 everywhere
    (the row sums agree to the last bit, p_v == q_v for v != x, q_x > p_x).
    Every shard then reports its race over p_0, and the token must be the
    oracle's two-level race over p_0 at position 0 (the fp64 residual of
    the oracle is a multiple of p_v off x, which races to the same token)."""
    import oracle
    B, g, V = 64, 2, 9000
    st = workloads.make_custom(B, g, V, dtype="f32", seed=33, T=1.0, device=DEV,
                               target_scale=2.0, noise=0.0)
    rows = torch.arange(B, device=DEV)
    x = st.target[:, 0].argmin(dim=-1)
    st.target[rows, 0, x] = st.target[:, 0].max(dim=-1).values - 30.0
    st.draft.copy_(st.target[:, :g])
    st.draft[rows, 0, x] += 2.0
    st.tokens[:, 0] = x.to(torch.int32)
    tg, _, _, _ = workloads.host_inputs(st)
    drawn = excluded = 0
    for step in range(3):
        res = run_sharded(st, 3, seed=9, step=step)
        same_on_every_rank(res)
        one = unsharded(st, 9, step)
        for b in range(B):
            if res[0]["accept_len"][b] != 0:
                continue
            assert one["accept_len"][b] == 0
            lp = oracle.row_logprobs(tg[b, 0], 1.0)
            y, gap = oracle.group_race(lp, 9, step, oracle.TAG_GUMBEL, b, 0)
            if gap < 1e-6:
                excluded += 1
                continue
            drawn += 1
            assert res[0]["tokens"][b][0] == y, (b, step)
            assert one["tokens"][b][0] == y, (b, step)
    assert drawn > B  # most sequences reject x (probability 0.86 each)
    assert excluded <= 2


def test_invalid_sequences_are_marked_on_every_rank():
    st = workloads.make_custom(8, 4, 5000, dtype="bf16", seed=6, T=1.0, device=DEV)
    st.temps[0] = -1.0
    st.temps[1] = float("nan")
    st.tokens[2, 2] = 5000           # outside the full vocabulary
    st.tokens[3, 0] = -5
    st.target[4, 2, 4500] = float("nan")  # NaN in the last shard only
    st.draft[5, 1, :] = float("-inf")
    st.target[6, 1, 10] = float("inf")    # +inf in the first shard only
    res = run_sharded(st, 3)
    same_on_every_rank(res)
    compare(res[0], run_oracle(st, 0, 0))
    for b in range(7):
        assert res[0]["accept_len"][b] == -1 and np.all(res[0]["tokens"][b] == -1)
    assert res[0]["accept_len"][7] >= 0


def test_shard_argument_errors():
    B, g, V = 2, 3, 5000
    st = workloads.make_custom(B, g, V, dtype="bf16", seed=1, device=DEV)
    ws = torch.zeros(sv.workspace_size(B, g, V, sv.BF16), dtype=torch.uint8, device=DEV)
    t = st.target[:, :, 100:2148].contiguous()
    d = st.draft[:, :, 100:2148].contiguous()
    with pytest.raises(sv.SpecVerifyError, match="multiple of 1024"):
        sv.spec_verify_shard_stats(t, d, st.tokens, st.temps, V=V, v0=100, workspace=ws)
    t = st.target[:, :, :1000].contiguous()
    d = st.draft[:, :, :1000].contiguous()
    with pytest.raises(sv.SpecVerifyError, match="every shard but the last"):
        sv.spec_verify_shard_stats(t, d, st.tokens, st.temps, V=V, v0=0, workspace=ws)
    with pytest.raises(sv.SpecVerifyError, match="must lie in"):
        sv.spec_verify_shard_stats(t, d, st.tokens, st.temps, V=V, v0=4096, workspace=ws)


def test_vocab_sharded_through_a_process_group_of_one():
    """spec_verify_vocab_sharded with its all-gathers on a real NCCL process
    group (one rank: the whole row is its shard)."""
    import socket

    import torch.distributed as dist
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{port}", rank=0,
                            world_size=1, device_id=torch.device(DEV))
    try:
        st = workloads.make_custom(6, 4, 7000, dtype="bf16", seed=44, T=[0.0, 0.7, 1.0],
                                   device=DEV)
        led = TieLedger("vocab-sharded through NCCL, one rank")
        for step in range(2):
            acc, tok, lp, lq = sv.spec_verify_vocab_sharded(st.target, st.draft, st.tokens,
                                                            st.temps, V=7000, v0=0, seed=2,
                                                            step=step, with_logprobs=True)
            torch.cuda.synchronize()
            got = {"accept_len": acc.cpu().numpy(), "tokens": tok.cpu().numpy(),
                   "lp": lp.cpu().numpy(), "lq": lq.cpu().numpy()}
            led.add(compare(got, run_oracle(st, 2, step)))
        led.check()
    finally:
        dist.destroy_process_group()


# ------------------------------------------------------------ seeded sweep
from hypothesis import HealthCheck, given, settings  # noqa: E402
from hypothesis import strategies as hs  # noqa: E402

_sweep = TieLedger("vocab-sharded sweep")


@settings(max_examples=30, deadline=None, derandomize=True, database=None,
          suppress_health_check=list(HealthCheck))
@given(B=hs.integers(1, 24), gamma=hs.integers(1, 10), V=hs.integers(1025, 60000),
       n=hs.integers(1, 6), dtype=hs.sampled_from(["bf16", "f32"]),
       T=hs.lists(hs.sampled_from([0.0, 0.05, 0.3, 0.7, 1.0, 2.5]), min_size=1, max_size=4),
       scale=hs.sampled_from([0.5, 2.0, 6.0]), noise=hs.sampled_from([0.0, 0.05, 0.6, 2.0]),
       seed=hs.integers(0, 2**31 - 1), step=hs.integers(0, 2**32 - 1))
def test_sharded_sweep(B, gamma, V, n, dtype, T, scale, noise, seed, step):
    """Shapes, shard counts (shards of whole 1024-entry groups, a ragged
    last one), dtypes, temperature mixes, logit scales and draft noise drawn
    by Hypothesis (derandomised): every rank identical, and equal to the
    oracle on the whole rows."""
    bounds = [b for b in sv.vocab_shards(V, n) if b[1] > 0]
    s = workloads.make_custom(B, gamma, V, dtype=dtype, seed=seed, T=T, device=DEV,
                              target_scale=scale, noise=noise)
    res = run_sharded(s, len(bounds), seed=seed, step=step, bounds=bounds)
    same_on_every_rank(res)
    _sweep.add(compare(res[0], run_oracle(s, seed, step)))


def test_sharded_sweep_tie_counts():
    """Runs after the sweep: its excluded (tie) count stays small."""
    _sweep.check(max_rate=5e-3, slack=3)
