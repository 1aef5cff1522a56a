#!/usr/bin/env python
"""Benchmark of batched speculative-sampling verification on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl ours|reference]

One step = one spec_verify (or spec_verify_multidraft) call over one batch
of a workload: every row statistic, the acceptance decisions and the
correction/bonus draw.  Metric: verified draft rows per second (B*gamma per
step; B*K*L for the multi-draft workload), whole job over all ranks.

Timing: inputs are resident in HBM before the timed region; each step reads
its own input set from a ring of distinct sets whose total size is several
times the L2 cache, so no step finds its logits in L2.  The K timed steps are
captured once in a CUDA graph and replayed; CUDA events on the launching
stream bracket the replay, with a barrier and a synchronize on both sides; the
max over ranks is reported.  Under torchrun each rank verifies its own batch
(batch-sharded replicas, no collective on the data path: weak scaling).

e2e: the same metric through the host-buffer entry point of the C ABI: every
step copies its inputs from pinned host memory to the device, verifies, and
copies the results back.

--impl reference times the CPU oracle (the reference arm of this build) on the
host cores, on a bounded sample of each step.
"""
from __future__ import annotations

import argparse
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402
import torch  # noqa: E402

import workloads  # noqa: E402

METRIC = ("verified draft rows/s and achieved HBM GB/s vs B200 peak "
          "(spec_verify, 1 GPU)")
UNIT = "rows/s"
DEFAULT_CONFIG = "c4_b256_g4_v151936_bf16"
NOMINAL_HBM_GBS = 8000.0  # B200 HBM3e, nominal (DGX figure)
L2_BYTES = 126 * 2**20


def _peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return float(d["hbm_gbs"]), "measured"
    except Exception:
        return 6650.0, "fallback"


def _source_hash() -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "speculative_decoding_verification_85_b200", "csrc")
    for name in sorted(os.listdir(csrc)):
        with open(os.path.join(csrc, name), "rb") as f:
            h.update(name.encode())
            h.update(f.read())
    return h.hexdigest()[:16]


def step_bytes(cfg: workloads.Config, temps: torch.Tensor, accept_len=None) -> dict:
    """Bytes of logits one step must read.

    formula: B (2 gamma + 1) V sizeof + B V sizeof (every row once, plus one
    residual row per sequence).  algorithmic: the rows the method needs --
    a greedy (T = 0) sequence needs its gamma + 1 target rows and no draw; a
    sampled sequence needs all 2 gamma + 1 rows once, and then the rows of its
    draw again: two (target and draft row j) for a residual draw at j < gamma,
    one (target row gamma) for the bonus draw.  The draw rows follow from the
    step's accept lengths when they are given (otherwise one row is assumed).
    The algorithmic figure is the one used for the roofline."""
    es = 2 if cfg.dtype == "bf16" else 4
    B, g, V = cfg.B, cfg.gamma, cfg.V
    formula = B * (2 * g + 1) * V * es + B * V * es
    t = temps.cpu().numpy()
    greedy = t == 0.0
    rows = np.where(greedy, g + 1, 2 * g + 1).astype(np.int64)
    if accept_len is None or cfg.multidraft:
        draw = np.where(greedy, 0, 1)
    else:
        a = accept_len.cpu().numpy()
        draw = np.where(greedy | (a < 0), 0, np.where(a < g, 2, 1))
    algo = int(np.sum(rows + draw)) * V * es
    return {"formula": formula, "algorithmic": algo}


def gpu_ident(dev) -> str:
    """nvidia-smi's id of a torch device: its UUID ("GPU-..."), so that the
    sampler watches the GPU this process uses whatever CUDA_VISIBLE_DEVICES
    remaps (nvidia-smi ignores that variable and counts physical GPUs)."""
    u = str(torch.cuda.get_device_properties(dev).uuid)
    return u if u.startswith("GPU-") else "GPU-" + u


class ClockSampler:
    """nvidia-smi clocks and throttle reasons sampled every 200 ms, for one GPU
    named by its nvidia-smi id (UUID)."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap,"
              "utilization.gpu")

    def __init__(self, ident: str):
        self.ident = str(ident)
        self.proc = None
        self.path = None

    def command(self) -> list:
        return ["nvidia-smi", "-i", self.ident, f"--query-gpu={self.FIELDS}",
                "--format=csv,noheader,nounits", "-lms", "200"]

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(self.command(), stdout=open(self.path, "w"),
                                         stderr=subprocess.DEVNULL)
        except FileNotFoundError:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *a):
        if self.proc is not None:
            time.sleep(0.3)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self) -> dict:
        rows = []
        if self.path and os.path.exists(self.path):
            with open(self.path) as f:
                for line in f:
                    p = [x.strip() for x in line.split(",")]
                    if len(p) >= 10:
                        rows.append(p)
            os.unlink(self.path)
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0,
                    "gpu": self.ident}

        def num(x):
            try:
                return float(x)
            except ValueError:
                return float("nan")

        load = [r for r in rows if num(r[9]) > 0] or rows
        sm = [num(r[1]) for r in load]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in load for i in range(4)
                          if r[5 + i].lower().startswith("active")})
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(num(r[2]) for r in rows),
                "reasons": reasons, "samples": len(load),
                "power_w_max": max(num(r[3]) for r in rows), "gpu": self.ident}


def _dist_init():
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime

        import torch.distributed as dist
        backend = "nccl" if torch.cuda.is_available() else "gloo"
        if backend == "nccl":
            torch.cuda.set_device(local)
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    elif torch.cuda.is_available():
        torch.cuda.set_device(local)
    return world, rank, local


def _barrier(world, local):
    if world > 1:
        import torch.distributed as dist
        if torch.cuda.is_available():
            dist.barrier(device_ids=[local])
        else:
            dist.barrier()


def _max_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(x: float, world: int, device) -> float:
    if world == 1:
        return x
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def ring_size(cfg: workloads.Config) -> int:
    """Distinct resident input sets the timed steps cycle through: at least 8
    and at least 4x the L2 size in total, whatever the step count, capped
    near 24 GB of device memory."""
    es = 2 if cfg.dtype == "bf16" else 4
    per = cfg.B * (2 * cfg.gamma + 1) * cfg.V * es
    need = max(8, -(-4 * L2_BYTES // per))
    cap = max(2, int(24e9 // per))
    return int(max(2, min(need, cap)))


# ------------------------------------------------------------------- oracle
REF_SAMPLE_B = 32  # sequences per oracle step on the large workloads (bounded CPU sample)


def oracle_batch(cfg) -> int:
    """Sequences per step in the oracle's timed sample: the whole batch, or
    the first REF_SAMPLE_B sequences of it (same recipe, same temperatures)
    on the workloads whose full step would take the single-threaded oracle
    seconds."""
    return min(cfg.B, REF_SAMPLE_B)


def time_oracle(cfg, sample_steps: int, threads: int, budget_s: float, rank: int = 0):
    """Run the oracle on up to `sample_steps` steps (stopping after
    `budget_s`); return (rows/s, steps done, seconds, sequences per step)."""
    import oracle
    Bs = oracle_batch(cfg)
    rows_per = cfg.rows_per_step // cfg.B * Bs
    done, t_total, rows = 0, 0.0, 0
    for s in range(sample_steps):
        st = workloads.make_step(cfg, s + 100000 * rank, device="cpu", B=Bs)
        tg, dr, tok, tm = workloads.host_inputs(st)
        t0 = time.perf_counter()
        if cfg.multidraft:
            oracle.verify_multidraft(tg, dr, tok, tm, seed=rank, step=s, threads=threads)
        else:
            oracle.verify(tg, dr, tok, tm, seed=rank, step=s, threads=threads)
        t_total += time.perf_counter() - t0
        rows += rows_per
        done += 1
        if t_total >= budget_s:
            break
    return rows / t_total, done, t_total, Bs


def run_reference(args, cfg):
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    try:
        cores = len(os.sched_getaffinity(0))
    except AttributeError:
        cores = os.cpu_count() or 1
    threads = max(1, min(cores, oracle_batch(cfg)))
    # W untimed warm-up steps, as reported in the line
    time_oracle(cfg, args.warmup, threads, 1e9)
    value, done, secs, Bs = time_oracle(cfg, args.steps, threads, args.ref_budget)
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": done, "warmup": args.warmup, "ms_per_step": 1e3 * secs / done,
        "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
        "data": "synthetic", "config": {"workload": cfg.name, "B": cfg.B, "gamma": cfg.gamma,
                                        "V": cfg.V, "K": cfg.K or None, "logits": cfg.dtype},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": threads, "kind": "oracle",
                         "sample": f"{done} steps of {cfg.name} (requested {args.steps}), "
                                   f"{Bs} of its {cfg.B} sequences per step, "
                                   f"sequences split over {threads} host threads"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)


# ------------------------------------------------------------------ GPU arm
def run_ours(args, cfg):
    import speculative_decoding_verification_85_b200 as sv

    world, rank, local = _dist_init()
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    K, W = args.steps, args.warmup
    R = args.sets if args.sets else ring_size(cfg)
    sets = [workloads.make_step(cfg, s + 100000 * rank, device=dev) for s in range(R)]
    dt = sv.BF16 if cfg.dtype == "bf16" else sv.F32
    B, g, V = cfg.B, cfg.gamma, cfg.V
    if cfg.multidraft:
        ws_bytes = sv.multidraft_workspace_size(B, cfg.K, g, V, dt)
    else:
        ws_bytes = sv.workspace_size(B, g, V, dt)
    ws = torch.zeros(ws_bytes, dtype=torch.uint8, device=dev)
    outs = [(torch.empty(B, dtype=torch.int32, device=dev),
             torch.empty((B, g + 1), dtype=torch.int32, device=dev),
             torch.empty(B, dtype=torch.int32, device=dev)) for _ in range(R)]
    stream = torch.cuda.Stream(device=dev)
    seed = rank

    def one(i: int):
        st = sets[i % R]
        acc, tok, extra = outs[i % R]
        if cfg.multidraft:
            sv.spec_verify_multidraft(st.target, st.draft, st.tokens, st.temps, seed=seed, step=i,
                                      workspace=ws, out_accept_len=acc, out_tokens=tok,
                                      out_draft_index=extra, stream=stream)
        else:
            sv.spec_verify(st.target, st.draft, st.tokens, st.temps, seed=seed, step=i,
                           workspace=ws, out_accept_len=acc, out_tokens=tok, stream=stream)

    # warm-up (eager), then capture the K timed steps once
    with torch.cuda.stream(stream):
        for i in range(W):
            one(i)
    stream.synchronize()
    # which of this library's kernels one step launches (profiler records of
    # one more eager step): counted for gpu_launches, named in the roofline
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        with torch.cuda.stream(stream):
            one(W)
        stream.synchronize()
    step_kernels = [e.name.split("(")[0].split("<")[0].replace("void ", "").replace("sv::", "")
                    for e in prof.events()
                    if e.device_type == torch.autograd.DeviceType.CUDA and "sv::" in e.name]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(W, W + K):
            one(i)
    # kernels of this library per step, as recorded above
    launches_per_replay = K * len(step_kernels)
    with torch.cuda.stream(stream):
        graph.replay()  # warm the graph itself
    stream.synchronize()

    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_ident(dev)) as clk:
        # soak so the clocks sampled below reflect this load
        t_end = time.time() + args.soak
        while time.time() < t_end:
            with torch.cuda.stream(stream):
                graph.replay()
            stream.synchronize()
        _barrier(world, local)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            graph.replay()
            ev1.record(stream)
        torch.cuda.synchronize(dev)
        _barrier(world, local)
    ms = ev0.elapsed_time(ev1)
    ms_max = _max_over_ranks(ms, world, dev)
    clocks = clk.summary()

    # outcome statistics of the timed steps (acceptance rate alpha)
    acc_all = torch.cat([o[0] for o in outs]).float()
    valid = acc_all >= 0
    mean_len = float(acc_all[valid].mean()) if valid.any() else float("nan")

    # algorithmic bytes per step, averaged over the ring's inputs and results
    per = [step_bytes(cfg, sets[r].temps, outs[r][0]) for r in range(R)]
    bytes_info = {"formula": per[0]["formula"],
                  "algorithmic": int(round(sum(x["algorithmic"] for x in per) / R))}

    rows_total = _sum_over_ranks(cfg.rows_per_step * K, world, dev)
    value = rows_total / (ms_max / 1e3)
    peak, peak_kind = _peaks()
    algo_gbs = bytes_info["algorithmic"] / (ms / K / 1e3) / 1e9
    traffic = None
    tp = os.path.join(ROOT, "profiles", "traffic.json")
    if os.path.exists(tp):
        try:
            with open(tp) as f:
                tj = json.load(f)
            if tj.get("source_hash") == _source_hash() and tj.get("workload") == cfg.name:
                traffic = tj.get("bytes_per_launch")
        except Exception:
            traffic = None

    # ---- e2e through the host-buffer entry point (single-draft workloads):
    # every step uploads its inputs from pinned host memory, verifies and
    # downloads its outputs; two staging buffers on two streams in turn, so one
    # step's upload overlaps the previous step's verification and download
    e2e = None
    if not cfg.multidraft:
        nst = 2
        stagings = [torch.zeros(sv.staging_size(B, g, V, dt), dtype=torch.uint8, device=dev)
                    for _ in range(nst)]
        streams = [stream, torch.cuda.Stream(device=dev)]
        nh = 2
        host = []
        for s_ in range(nh):
            st = sets[s_]
            host.append([x.cpu().pin_memory() for x in (st.target, st.draft, st.tokens,
                                                        st.temps)])
        outs_h = [(torch.empty(B, dtype=torch.int32, pin_memory=True),
                   torch.empty((B, g + 1), dtype=torch.int32, pin_memory=True))
                  for _ in range(nst)]

        def e2e_step(i):
            k = i % nst
            sv.spec_verify_host(*host[i % nh], staging=stagings[k], seed=seed, step=i,
                                out_accept_len=outs_h[k][0], out_tokens=outs_h[k][1],
                                stream=streams[k], wait=False)

        for i in range(max(W, 3)):
            e2e_step(i)
        torch.cuda.synchronize(dev)
        ke = K
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        done1 = torch.cuda.Event()
        _barrier(world, local)
        torch.cuda.synchronize(dev)
        e0.record(streams[0])
        streams[1].wait_event(e0)
        for i in range(ke):
            e2e_step(i)
        done1.record(streams[1])
        streams[0].wait_event(done1)
        e1.record(streams[0])
        torch.cuda.synchronize(dev)
        _barrier(world, local)
        ems = _max_over_ranks(e0.elapsed_time(e1), world, dev)
        es = 2 if cfg.dtype == "bf16" else 4
        h2d = B * (2 * g + 1) * V * es + B * g * 4 + B * 4
        d2h = B * 4 + B * (g + 1) * 4
        e2e = {"value": _sum_over_ranks(cfg.rows_per_step * ke, world, dev) / (ems / 1e3),
               "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
               "ms_per_step": ems / ke, "h2d_gbs": h2d / (ems / ke / 1e3) / 1e9,
               "path": "spec_verify_host_async (pinned host buffers; two staging buffers "
                       "on two streams in turn)"}
        # the same bytes uploaded alone from pinned memory, no verification:
        # the host-to-device floor the end-to-end step is compared with
        hflat = torch.empty(h2d, dtype=torch.uint8, pin_memory=True)
        dst = (stagings[0][:h2d] if stagings[0].numel() >= h2d
               else torch.empty(h2d, dtype=torch.uint8, device=dev))
        with torch.cuda.stream(stream):
            for _ in range(2):
                dst.copy_(hflat, non_blocking=True)
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            e0.record(stream)
            for _ in range(ke):
                dst.copy_(hflat, non_blocking=True)
            e1.record(stream)
        torch.cuda.synchronize(dev)
        hms = _max_over_ranks(e0.elapsed_time(e1), world, dev) / ke
        e2e["h2d_only_ms_per_step"] = hms
        e2e["vs_h2d_only"] = (ems / ke) / hms
        del hflat

    # ---- CPU baseline: the oracle on a bounded sample (rank 0, N = 1 only)
    cpu = None
    if world == 1 and rank == 0 and not args.no_cpu_baseline:
        v, done, secs, Bs = time_oracle(cfg, args.cpu_steps, 1, args.cpu_budget)
        cpu = {"value": v, "unit": UNIT, "cores": 1, "kind": "oracle",
               "sample": f"{done} steps of {cfg.name}, {Bs} of its {cfg.B} sequences per "
                         f"step, single-threaded, {secs:.1f} s"}

    if rank == 0:
        line = {
            "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": K,
            "warmup": W, "ms_per_step": ms_max / K, "higher_is_better": True,
            "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
            "config": {"workload": cfg.name, "B": cfg.B, "gamma": cfg.gamma, "V": cfg.V,
                       "K": cfg.K or None, "logits": cfg.dtype,
                       "inputs": f"ring of {R} distinct resident input sets "
                                 f"({R * bytes_info['formula'] / 1e9:.2f} GB, "
                                 f"{R * bytes_info['formula'] / L2_BYTES:.1f}x L2); "
                                 "no L2 flush needed",
                       "launch": "K steps captured in one CUDA graph, replayed",
                       "parallelism": f"batch-sharded replicas x{world}"},
            "roofline": {"bound": "hbm",
                         "kernel": " + ".join(dict.fromkeys(step_kernels)) + (
                             " (the whole step)" if len(step_kernels) > 1 else
                             " (one launch per step)"),
                         "achieved": algo_gbs, "peak": peak, "unit": "GB/s",
                         "frac": algo_gbs / peak, "traffic": traffic,
                         "peak_source": (f"{peak_kind} hbm_gbs (MEASURED_PEAKS.json)"
                                         if peak_kind == "measured" else
                                         "fallback (an earlier copy-bandwidth measurement on "
                                         "this pool; MEASURED_PEAKS.json absent)"),
                         "peak_nominal": NOMINAL_HBM_GBS,
                         "frac_nominal": algo_gbs / NOMINAL_HBM_GBS,
                         "algorithmic_bytes_per_launch": bytes_info["algorithmic"],
                         "formula_bytes_per_step": bytes_info["formula"],
                         "formula_gbs": bytes_info["formula"] / (ms / K / 1e3) / 1e9,
                         "formula_frac": bytes_info["formula"] / (ms / K / 1e3) / 1e9 / peak,
                         "formula_frac_nominal":
                             bytes_info["formula"] / (ms / K / 1e3) / 1e9 / NOMINAL_HBM_GBS},
            "cpu_baseline": cpu, "e2e": e2e, "gpu_launches": launches_per_replay,
            "clocks": clocks,
            "accept": {"mean_accept_len": mean_len,
                       "alpha": mean_len / (cfg.gamma if not cfg.multidraft else cfg.gamma)},
        }
        print(json.dumps(line), flush=True)
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_vocab_shards(args, cfg):
    """--vocab-shards n: the vocabulary-sharded path as rank 0 of n runs it,
    on one GPU.  Rank 0's three calls (shard statistics, decision and shard
    race, pick) on its 1/n of every row are timed; the other ranks' records
    are computed once per input set before timing and sit in their slots of
    the two exchange buffers, which rank 0 fills in place (so the two
    all-gathers of an n-GPU run are not in the timed region).  Each input set
    is verified with a fixed step value, so every timed step repeats the
    setup's computation and its outputs are checked against the unsharded
    path."""
    import dataclasses

    import speculative_decoding_verification_85_b200 as sv

    world, rank, local = _dist_init()
    if world != 1:
        raise SystemExit("--vocab-shards times one emulated rank on one GPU")
    if cfg.multidraft:
        raise SystemExit("--vocab-shards: single-draft workloads only")
    n = args.vocab_shards
    dev = torch.device("cuda", local)
    torch.cuda.set_device(dev)
    K, W = args.steps, args.warmup
    B, g, V = cfg.B, cfg.gamma, cfg.V
    dt = sv.BF16 if cfg.dtype == "bf16" else sv.F32
    es = 2 if cfg.dtype == "bf16" else 4
    bounds = [b_ for b_ in sv.vocab_shards(V, n) if b_[1] > 0]  # ranks past V hold nothing
    n = len(bounds)
    v00, Vs0 = bounds[0]
    shard_set_bytes = B * (2 * g + 1) * Vs0 * es
    R = args.sets if args.sets else max(ring_size(cfg), -(-4 * L2_BYTES // shard_set_bytes))
    rec, crec = sv.shard_stats_bytes(B, g), sv.shard_candidate_bytes(B)
    wss = [torch.zeros(sv.workspace_size(B, g, Vs, dt), dtype=torch.uint8, device=dev)
           for _, Vs in bounds]
    stream = torch.cuda.Stream(device=dev)
    sets, differ = [], 0
    with torch.cuda.stream(stream):
        for k in range(R):
            st = workloads.make_step(cfg, k, device=dev)
            sl = [(v0, st.target[:, :, v0:v0 + Vs].contiguous(),
                   st.draft[:, :, v0:v0 + Vs].contiguous()) for v0, Vs in bounds]
            all_stats = torch.empty(n * rec, dtype=torch.uint8, device=dev)
            all_cands = torch.empty(n * crec, dtype=torch.uint8, device=dev)
            acc = torch.empty(B, dtype=torch.int32, device=dev)
            tok = torch.empty((B, g + 1), dtype=torch.int32, device=dev)
            for r, (v0, t, d) in enumerate(sl):
                sv.spec_verify_shard_stats(t, d, st.tokens, st.temps, V=V, v0=v0, workspace=wss[r],
                                           out_stats=all_stats[r * rec:(r + 1) * rec],
                                           stream=stream)
            for r, (v0, t, d) in enumerate(sl):
                a_r = acc if r == 0 else torch.empty_like(acc)
                t_r = tok if r == 0 else torch.empty_like(tok)
                sv.spec_verify_shard_decide(t, d, st.tokens, st.temps, all_stats, V=V, v0=v0,
                                            nshards=n, workspace=wss[r], seed=0, step=k,
                                            out_accept_len=a_r, out_tokens=t_r,
                                            out_candidate=all_cands[r * crec:(r + 1) * crec],
                                            stream=stream)
            sv.spec_verify_shard_pick(all_cands, nshards=n, out_accept_len=acc, out_tokens=tok,
                                      stream=stream)
            a1, t1, _, _ = sv.spec_verify(st.target, st.draft, st.tokens, st.temps, seed=0,
                                          step=k, stream=stream)
            stream.synchronize()
            differ += int(((a1 != acc) | (t1 != tok).any(dim=1)).sum())
            sets.append((sl[0][1], sl[0][2], st.tokens, st.temps, all_stats, all_cands, acc, tok))
            del st, sl
    torch.cuda.empty_cache()

    def one(i: int):
        k = i % R
        t, d, x, temps, all_stats, all_cands, acc, tok = sets[k]
        sv.spec_verify_shard_stats(t, d, x, temps, V=V, v0=v00, workspace=wss[0],
                                   out_stats=all_stats[:rec], stream=stream)
        sv.spec_verify_shard_decide(t, d, x, temps, all_stats, V=V, v0=v00, nshards=n,
                                    workspace=wss[0], seed=0, step=k, out_accept_len=acc,
                                    out_tokens=tok, out_candidate=all_cands[:crec], stream=stream)
        sv.spec_verify_shard_pick(all_cands, nshards=n, out_accept_len=acc, out_tokens=tok,
                                  stream=stream)

    with torch.cuda.stream(stream):
        for i in range(W):
            one(i)
    stream.synchronize()
    from torch.profiler import ProfilerActivity, profile
    with profile(activities=[ProfilerActivity.CUDA]) as prof:
        with torch.cuda.stream(stream):
            one(W)
        stream.synchronize()
    step_kernels = [e.name.split("(")[0].split("<")[0].replace("void ", "").replace("sv::", "")
                    for e in prof.events()
                    if e.device_type == torch.autograd.DeviceType.CUDA and "sv::" in e.name]
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for i in range(W, W + K):
            one(i)
    with torch.cuda.stream(stream):
        graph.replay()
    stream.synchronize()
    ev0, ev1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(gpu_ident(dev)) as clk:
        t_end = time.time() + args.soak
        while time.time() < t_end:
            with torch.cuda.stream(stream):
                graph.replay()
            stream.synchronize()
        torch.cuda.synchronize(dev)
        with torch.cuda.stream(stream):
            ev0.record(stream)
            graph.replay()
            ev1.record(stream)
        torch.cuda.synchronize(dev)
    ms = ev0.elapsed_time(ev1)
    # rank 0's algorithmic bytes: its slice of every needed row and draw row
    scfg = dataclasses.replace(cfg, V=Vs0)
    algo = int(round(sum(step_bytes(scfg, s_[3], s_[6])["algorithmic"] for s_ in sets) / R))
    gbs = algo / (ms / K / 1e3) / 1e9
    peak, peak_kind = _peaks()
    line = {
        "metric": METRIC, "value": cfg.rows_per_step * K / (ms / 1e3), "unit": UNIT,
        "n_gpus": 1, "steps": K, "warmup": W, "ms_per_step": ms / K, "higher_is_better": True,
        "scaling": "strong", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": cfg.name, "vocab_shards": n, "rank": 0, "shard": [v00, Vs0],
                   "timed": "rank 0's three calls on its 1/n of every row; the other ranks' "
                            "records gathered before timing (the two all-gathers are not "
                            "timed: one GPU)",
                   "inputs": f"ring of {R} input sets ({R * shard_set_bytes / 1e9:.2f} GB of "
                             f"rank 0's rows, {R * shard_set_bytes / L2_BYTES:.1f}x L2)",
                   "launch": "K steps captured in one CUDA graph, replayed"},
        "roofline": {"bound": "hbm", "kernel": " + ".join(dict.fromkeys(step_kernels)),
                     "achieved": gbs, "peak": peak, "unit": "GB/s", "frac": gbs / peak,
                     "traffic": None, "peak_source": peak_kind,
                     "algorithmic_bytes_per_launch": algo},
        "gpu_launches": K * len(step_kernels), "clocks": clk.summary(), "e2e": None,
        "cpu_baseline": None,
        "check": {"sequences": R * B, "differ_from_unsharded": differ},
    }
    print(json.dumps(line), flush=True)
    del graph


def main():
    ap = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=None)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--config", default=DEFAULT_CONFIG)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--soak", type=float, default=1.5, help="seconds of untimed load before timing")
    ap.add_argument("--cpu-steps", type=int, default=200)
    ap.add_argument("--cpu-budget", type=float, default=10.0)
    ap.add_argument("--ref-budget", type=float, default=60.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--batch", type=int, default=None,
                    help="run the workload with this many sequences instead of its own B "
                         "(small profiling captures; not a bench line)")
    ap.add_argument("--sets", type=int, default=None,
                    help="distinct input sets in the ring (default: at least 4x L2)")
    ap.add_argument("--vocab-shards", type=int, default=None,
                    help="time rank 0 of this many vocabulary shards on one GPU (not the "
                         "bench line)")
    args = ap.parse_args()
    cfg = workloads.get(args.config)
    if args.batch is not None and args.batch != cfg.B:
        import dataclasses
        cfg = dataclasses.replace(cfg, B=args.batch, name=f"{cfg.name}@B{args.batch}")
    if args.steps is None:
        args.steps = 1000 if cfg.index in (1, 3) else (200 if cfg.index == 2 else
                                                         (100 if cfg.index == 4 else 1000))
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        run_reference(args, cfg)
    elif args.vocab_shards:
        run_vocab_shards(args, cfg)
    else:
        run_ours(args, cfg)


if __name__ == "__main__":
    main()
