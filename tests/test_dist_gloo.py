"""Multi-rank host logic of the benchmark, on CPU with gloo (world size 2).

The verification path partitions by sequence: each rank verifies its own
batch (its own inputs and Philox key), with no collective on the data path.
The only cross-rank steps are the timing barrier and the max / sum
reductions; these run here as two gloo ranks, together with the check that
the ranks' shards are distinct and that each rank's oracle result depends
only on its own shard.
"""
import os
import socket

import numpy as np
import pytest
import torch.multiprocessing as mp


def _free_port():
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    return port


def _rank_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import bench
    import oracle
    import workloads

    w, r, _ = bench._dist_init()
    assert (w, r) == (world, rank)
    bench._barrier(w, 0)
    mx = bench._max_over_ranks(float(rank + 1) * 1.5, w, torch.device("cpu"))
    sm = bench._sum_over_ranks(10.0, w, torch.device("cpu"))
    st = workloads.make_custom(3, 2, 17, dtype="bf16", seed=100000 * rank, T=0.8)
    tg, dr, tok, tm = workloads.host_inputs(st)
    res = oracle.verify(tg, dr, tok, tm, seed=rank, step=0)
    gathered = [None] * w
    dist.all_gather_object(gathered, (tg.tobytes(), res["tokens"].tolist()))
    dist.destroy_process_group()
    out[rank] = (mx, sm, gathered)


@pytest.mark.parametrize("world", [2])
def test_two_rank_reductions_and_shards(world):
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs), [p.exitcode for p in procs]
    for r in range(world):
        mx, sm, gathered = out[r]
        assert mx == 1.5 * world          # max over ranks
        assert sm == 10.0 * world         # sum over ranks (rows of all ranks)
        assert gathered[0][0] != gathered[1][0]  # distinct shards
    # rank 0's result equals a single-process run on rank 0's shard
    import oracle
    import workloads
    st = workloads.make_custom(3, 2, 17, dtype="bf16", seed=0, T=0.8)
    tg, dr, tok, tm = workloads.host_inputs(st)
    solo = oracle.verify(tg, dr, tok, tm, seed=0, step=0)
    assert out[0][2][0][1] == solo["tokens"].tolist()
    assert np.array_equal(np.array(out[1][2][0][1]), solo["tokens"])


def _gather_main(rank, world, port, out):
    os.environ.update(RANK=str(rank), WORLD_SIZE=str(world), LOCAL_RANK=str(rank),
                      MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import torch
    import torch.distributed as dist

    import speculative_decoding_verification_85_b200 as sv

    dist.init_process_group("gloo", rank=rank, world_size=world)
    local = torch.arange(48, dtype=torch.uint8) + 100 * rank
    got = sv.gather_records(local)
    dist.destroy_process_group()
    out[rank] = got.tolist()


def test_vocab_shard_exchange_is_rank_ordered():
    """The exchange between the vocabulary-shard calls: every rank receives
    all ranks' records concatenated in rank order (two gloo ranks on CPU)."""
    world = 2
    ctx = mp.get_context("spawn")
    mgr = ctx.Manager()
    out = mgr.dict()
    port = _free_port()
    procs = [ctx.Process(target=_gather_main, args=(r, world, port, out)) for r in range(world)]
    for p in procs:
        p.start()
    for p in procs:
        p.join(timeout=180)
    assert all(p.exitcode == 0 for p in procs)
    want = list(range(48)) + [100 + i for i in range(48)]
    assert out[0] == want and out[1] == want
