#!/usr/bin/env python
"""Benchmark of the HySparse2 hot path on B200.

One step = one decode step of a hybrid block on the long-decode workload (8 sequences, a
262,144-token MQA K/V cache each, 64 query heads, head_dim 128): the full-attention layer
with top-1024 + last-128 selection (hs2_full_attn_select, Lq = 1), then 4 sparse layers that
reuse K, V and the indices with their own queries (hs2_sparse_attn). Throughput is steps/s
of the whole job. Inputs (1.07 GB of K+V per GPU) are larger than L2, so no flush is needed.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl hs2|reference] [--no-prefill]

Multi-GPU: one process per GPU (torchrun); every rank runs its own independent batch
(weak scaling, no data-path collective); the timed region is bracketed by barriers and the
reported time is the max over ranks.

--impl reference times the fp64 CPU oracle (the only other implementation of the path) on
this host's cores, on a bounded sample of the same workload, extrapolated to a step.
"""
from __future__ import annotations

import argparse
import ctypes
import csv
import io
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import synth  # noqa: E402

METRIC = "sparse-attn decode steps/s @256k; full-attn+top-k prefill tok/s; % roofline"
WORKLOAD = "decode_256k"
PREFILL_WORKLOAD = "prefill_32k"


def _peaks():
    try:
        with open(os.path.join(ROOT, "MEASURED_PEAKS.json")) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p["bf16_tflops_sustained"], "source": "measured"}
    except Exception:
        return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


def _traffic(kernel: str):
    """dram bytes per launch from a committed ncu capture, if it is still for this source."""
    try:
        with open(os.path.join(ROOT, "profiles", "traffic.json")) as f:
            t = json.load(f)[kernel]
        import hashlib
        src = open(os.path.join(ROOT, t["source"]), "rb").read()
        if hashlib.sha256(src).hexdigest() != t["source_sha256"]:
            return None
        return t["dram_bytes_per_launch"]
    except Exception:
        return None


class ClockSampler:
    """nvidia-smi clocks / throttle reasons, sampled every 50 ms by a reader thread; summary()
    keeps the samples taken between start_region() and end_region()."""

    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.rows = []          # (monotonic time, csv line)
        self.t_start = None
        self.t_end = None
        self._first = threading.Event()
        self._thread = None

    def _reader(self):
        for line in self.proc.stdout:
            self.rows.append((time.monotonic(), line))
            self._first.set()

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "50"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self._thread = threading.Thread(target=self._reader, daemon=True)
            self._thread.start()
            self._first.wait(timeout=5.0)   # sampling is running before the timed region opens
        except Exception:
            self.proc = None
        return self

    def start_region(self):
        self.t_start = time.monotonic()

    def end_region(self):
        self.t_end = time.monotonic()
        # one more sample after the region, so a region shorter than the interval still has one
        n = len(self.rows)
        t0 = time.monotonic()
        while self.proc is not None and len(self.rows) == n and time.monotonic() - t0 < 0.5:
            time.sleep(0.01)

    def __exit__(self, *a):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            if self._thread is not None:
                self._thread.join(timeout=2)

    def summary(self):
        lines = [ln for (t, ln) in self.rows
                 if self.t_start is None or (t >= self.t_start and (self.t_end is None or t <= self.t_end + 0.06))]
        if not lines:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unavailable"], "samples": 0}
        rows = [r for r in csv.reader(io.StringIO("".join(lines))) if len(r) >= 9]
        sm = [float(r[1]) for r in rows if r[1].strip().replace(".", "").isdigit()]
        smax = [float(r[2]) for r in rows if r[2].strip().replace(".", "").isdigit()]
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[5 + i].strip().lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * (max(sm) if sm else 1)]
        return {"sm_mhz": statistics.median(loaded) if loaded else None, "sm_max_mhz": max(smax) if smax else None,
                "reasons": reasons, "samples": len(rows)}


# ----------------------------------------------------------------------------------------------
# CPU oracle timing (cpu_baseline leg and --impl reference)
# ----------------------------------------------------------------------------------------------
def oracle_decode_sample(g: synth.SyntheticInputs, keys: int, seq: int = 0, want=False):
    """Oracle on sequence `seq` truncated to its last `keys` cache rows: full layer + sparse layers.
    Returns the time, and with want=True also the full layer's oracle result (idx, score)."""
    import oracle
    wl = g.wl
    k = np.ascontiguousarray(g.k[seq:seq + 1, -keys:])
    v = np.ascontiguousarray(g.v[seq:seq + 1, -keys:])
    q = np.ascontiguousarray(g.q[seq:seq + 1])
    t0 = time.perf_counter()
    r = oracle.full_attn_select(q, k, v, wl.scale, wl.window, wl.topk, want_score=want)
    idx = r["idx"].reshape(1, 1, -1)
    for layer in range(wl.n_sparse):
        oracle.sparse_attn(np.ascontiguousarray(g.q_sparse(layer)[seq:seq + 1]), k, v, idx, wl.scale)
    dt = time.perf_counter() - t0
    return (dt, r) if want else dt


def oracle_keys_for_budget(g, budget_s: float) -> int:
    """Largest cache sample (power of two, <= Lk) whose oracle step fits in budget_s."""
    wl = g.wl
    keys = min(wl.Lk, 16384)
    t = oracle_decode_sample(g, keys)
    per_key = t / keys
    fit = int(budget_s / max(per_key, 1e-12))
    keys = max(2048, min(wl.Lk, 1 << int(math.floor(math.log2(max(fit, 2048))))))
    return keys


def selection_check(gpu_idx, results, wl):
    """Swap count of the GPU's decode selection against the oracle's (whole sequences only):
    the acceptance rule of the parity tests (tests/parity.py), on the bench's own inputs."""
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import check_selection
    if not results:
        return None
    seqs = sorted(results)
    st = check_selection(np.stack([gpu_idx[b] for b in seqs]), np.stack([results[b]["idx"][0] for b in seqs]),
                         np.stack([results[b]["score"][0] for b in seqs]), np.full(len(seqs), wl.Lk - 1),
                         wl.window, wl.topk)
    return {"sequences": len(seqs), "swaps": st.swaps, "max_swap_rel": st.max_swap_rel, "ok": st.ok(),
            "rule": "sets equal except swaps whose fp64 oracle scores differ by <= 1e-5 relative"}


def cpu_baseline(g, budget_s=20.0, min_s=10.0, gpu_idx=None):
    """The oracle on the host cores, on a bounded sample of the bench workload: whole sequences
    (or the last `keys` rows of each when one is too slow), as many as fit in about 10-20 s.
    With gpu_idx ([B, S] of the timed run, same inputs) the sequences the oracle ran whole also
    give the selection's swap count."""
    import oracle
    wl = g.wl
    keys = oracle_keys_for_budget(g, budget_s)
    total, n = 0.0, 0
    results = {}
    while n < 3 * wl.B and (n == 0 or total < min_s):
        want = gpu_idx is not None and keys == wl.Lk and n < wl.B
        r = oracle_decode_sample(g, keys, seq=n % wl.B, want=want)
        if want:
            r, res = r
            results[n % wl.B] = res
        total += r
        n += 1
    step_s = total / n * (wl.Lk / keys) * wl.B
    base = {"value": 1.0 / step_s, "unit": "steps/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": f"{n} sequence passes (sequences 0..{min(n, wl.B) - 1} of {wl.B}), last {keys} of {wl.Lk} "
                      f"cache rows each, full layer + {wl.n_sparse} sparse layers, {total:.1f} s; scaled "
                      f"x{wl.Lk // keys} rows x{wl.B} sequences / {n} passes"
                      + ("" if keys == wl.Lk and n >= wl.B else " (extrapolated)")}
    sel = selection_check(gpu_idx, results, wl) if gpu_idx is not None else None
    return base, sel


def run_reference(args):
    """The reference arm: the fp64 oracle as it stands on this host's cores. One step is the whole
    decode step of the bench workload (every sequence's full layer and sparse layers) when that
    fits the per-step share of a ~150 s budget; otherwise a bounded sample of it (the first
    sequence, or the last `keys` rows of its cache) scaled to a step, said so in the line."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return 0
    import oracle
    wl = synth.WORKLOADS[WORKLOAD]
    g = synth.SyntheticInputs(wl, seed=args.seed)
    n_runs = args.steps + args.warmup
    per_step_budget = max(0.5, 150.0 / max(n_runs, 1))
    t_seq = oracle_decode_sample(g, wl.Lk)               # one whole sequence (also a warm-up)
    if t_seq * wl.B <= per_step_budget:
        keys, seqs = wl.Lk, list(range(wl.B))              # the whole step, no extrapolation
    elif t_seq <= per_step_budget:
        keys, seqs = wl.Lk, [0]
    else:
        keys, seqs = oracle_keys_for_budget(g, per_step_budget), [0]

    def one_step():
        return sum(oracle_decode_sample(g, keys, seq=b) for b in seqs)

    for _ in range(args.warmup):
        one_step()
    total = 0.0
    for _ in range(args.steps):
        total += one_step()
    sample_s = total / max(args.steps, 1)
    scale_up = (wl.Lk / keys) * (wl.B / len(seqs))
    step_s = sample_s * scale_up
    value = 1.0 / step_s
    sample = (f"per step: all {wl.B} sequences, whole {wl.Lk}-row caches, full layer + {wl.n_sparse} sparse "
              f"layers (no extrapolation)" if scale_up == 1.0 else
              f"per step: sequence 0 of {wl.B}, last {keys} of {wl.Lk} cache rows, scaled x{wl.Lk // keys} rows "
              f"x{wl.B // len(seqs)} sequences (extrapolated)")
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": args.gpus,
        "steps": args.steps, "warmup": args.warmup, "ms_per_step": step_s * 1e3, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": f"{wl.name}: B={wl.B} sequences per GPU, {wl.Lk}-token MQA K/V cache, "
                               f"H={wl.H}, d={wl.d}, window {wl.window} + top-{wl.topk}, "
                               f"{wl.n_sparse} sparse layers per step"},
        "cpu_baseline": {"value": value, "unit": "steps/s", "cores": oracle.default_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "steps/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------------------------
# GPU arm
# ----------------------------------------------------------------------------------------------
def _dist_init():
    """Rank setup from the torchrun environment. NCCL on GPUs; gloo when there is no GPU (the
    multi-rank host logic is tested that way on CPU)."""
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    gpu = torch.cuda.is_available()
    if gpu:
        torch.cuda.set_device(local)
    if world > 1 and not dist.is_initialized():
        import datetime
        timeout = datetime.timedelta(seconds=120)
        if gpu:
            dist.init_process_group("nccl", timeout=timeout, device_id=torch.device("cuda", local))
        else:
            dist.init_process_group("gloo", timeout=timeout)
    return world, rank, local


def _reduce_device():
    import torch
    import torch.distributed as dist
    return "cpu" if dist.get_backend() == "gloo" else "cuda"


def _barrier(world):
    import torch
    import torch.distributed as dist
    if world > 1:
        dist.barrier()
    if torch.cuda.is_available():
        torch.cuda.synchronize()


def _max_over_ranks(x: float, world: int) -> float:
    """The slowest rank's value: every multi-GPU time is the max over ranks."""
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def _sum_over_ranks(x: float, world: int) -> float:
    import torch
    import torch.distributed as dist
    if world == 1:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=_reduce_device())
    dist.all_reduce(t, op=dist.ReduceOp.SUM)
    return float(t.item())


def _throughput(world: int, steps: int, ms_max: float) -> float:
    """Whole-job steps/s: every rank runs `steps` steps of its own batch (weak scaling), timed by
    the slowest rank."""
    return world * steps / (ms_max / 1e3)


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=1000)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--impl", default="hs2", choices=["hs2", "reference"])
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-prefill", action="store_true")
    ap.add_argument("--no-ragged", action="store_true", help="skip the ragged-batch decode clause")
    ap.add_argument("--no-fp8", action="store_true", help="skip the FP8 (e4m3) K/V cache decode clause")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true", help="skip the decode_32k, decode_1m and tiny_prefill clauses")
    ap.add_argument("--no-v1", action="store_true", help="skip the HySparse (v1) block-level decode clause")
    ap.add_argument("--fp8-only", action="store_true",
                    help="time only the FP8-cache decode step (--steps/--warmup; small profiling cases with --batch)")
    ap.add_argument("--no-backward", action="store_true", help="skip the training-shape backward clause")
    ap.add_argument("--eager", action="store_true", help="time eager launches instead of one CUDA graph of the steps")
    ap.add_argument("--batch", type=int, default=0, help="override sequences per GPU (small profiling cases)")
    ap.add_argument("--cache", type=int, default=0, help="override cache length (small profiling cases)")
    ap.add_argument("--prefill-only", action="store_true", help="time only the prefill full-attention + selection")
    ap.add_argument("--prefill-len", type=int, default=0, help="override the prefill length (profiling cases)")
    ap.add_argument("--sparse-layers", type=int, default=-1, help="prefill-only: sparse layers to time after it")
    args = ap.parse_args()
    if args.warmup < 3:
        args.warmup = 3
    if args.impl == "reference":
        return run_reference(args)
    if args.prefill_only:
        return run_prefill_only(args)
    if args.fp8_only:
        return run_fp8_only(args)
    return run_gpu(args)


def run_fp8_only(args):
    """The FP8-cache decode step alone on the decode workload (or a reduced --batch/--cache case);
    one JSON line."""
    import torch
    import long_context_mqa_b200 as hs2
    world, rank, local = _dist_init()
    dev = torch.device("cuda", local)
    wl = synth.WORKLOADS[WORKLOAD]
    if args.batch or args.cache:
        wl = wl.with_(name=f"{WORKLOAD}_b{args.batch or wl.B}_n{args.cache or wl.Lk}", B=args.batch or wl.B,
                      Lk=args.cache or wl.Lk)
    g = synth.SyntheticInputs(wl, seed=args.seed + rank)
    q, k, v = _bf16(g.q, dev), _bf16(g.k, dev), _bf16(g.v, dev)
    qs = [_bf16(g.q_sparse(i), dev) for i in range(wl.n_sparse)]
    res = bench_fp8(args, world, wl, hs2, q, k, v, qs, _peaks(), steps=max(1, args.steps), warmup=args.warmup)
    if rank == 0:
        print(json.dumps({"fp8_kv": res}), flush=True)
    return 0


def run_prefill_only(args):
    """Prefill full attention + selection (and optionally its sparse layers) alone; one JSON line."""
    import torch
    world, rank, local = _dist_init()
    dev = torch.device("cuda", local)
    res = bench_prefill(args, world, dev, _peaks(), reps=max(1, args.steps), warmup=args.warmup)
    if rank == 0:
        print(json.dumps({"prefill": res}), flush=True)
    return 0


def _bf16(bits, device):
    import torch
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).to(device)


def run_gpu(args):
    import torch
    import long_context_mqa_b200 as hs2
    world, rank, local = _dist_init()
    dev = torch.device("cuda", local)
    peaks = _peaks()
    wl = synth.WORKLOADS[WORKLOAD]
    if args.batch or args.cache:   # reduced case for profiler captures; never the reported workload
        wl = wl.with_(name=f"{WORKLOAD}_b{args.batch or wl.B}_n{args.cache or wl.Lk}", B=args.batch or wl.B,
                      Lk=args.cache or wl.Lk)
    g = synth.SyntheticInputs(wl, seed=args.seed + rank)   # each rank: its own independent batch
    q = _bf16(g.q, dev)
    k = _bf16(g.k, dev)
    v = _bf16(g.v, dev)
    qs = [_bf16(g.q_sparse(i), dev) for i in range(wl.n_sparse)]
    S = wl.window + wl.topk
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, 1, wl.H), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.B, 1, S), dtype=torch.int32, device=dev)
    outs = [torch.empty_like(q) for _ in range(wl.n_sparse)]
    ws_full = torch.zeros(hs2.full_attn_select_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d), dtype=torch.uint8,
                          device=dev)
    ws_sp_bytes = hs2.sparse_attn_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d, S)
    ws_sp = [torch.zeros(ws_sp_bytes, dtype=torch.uint8, device=dev) for _ in range(wl.n_sparse)]
    stream = torch.cuda.current_stream()

    def step():
        # one hybrid block: the full-attention layer selects, then its sparse layers run one after
        # another (in the model each sparse layer's query comes from the previous layer's output)
        hs2.full_attn_select(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws_full)
        for i in range(wl.n_sparse):
            hs2.sparse_attn(qs[i], k, v, idx, scale=wl.scale, out=outs[i], workspace=ws_sp[i])

    # ---------------- device-resident throughput: the K timed steps run as one CUDA graph (the
    # library's timing events around the dec_fused launches become nodes of that graph). An event
    # between two launches cuts their programmatic-launch overlap, so the events bracket the
    # dec_fused launch of every PROF_EVERY-th step only.
    PROF_EVERY = 8

    def timed_steps():
        for i in range(args.steps):
            hs2.profile_enable("dec_fused" if i % PROF_EVERY == 0 else None)
            step()
        hs2.profile_enable(None)

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    graph, graph_note = None, None
    launches0 = hs2.kernel_launches()
    if not args.eager:
        try:
            graph = torch.cuda.CUDAGraph()
            with torch.cuda.graph(graph):
                timed_steps()
            graph.replay()            # upload and warm the graph (untimed)
            torch.cuda.synchronize()
        except Exception as e:       # fall back to eager launches, said so in the line
            hs2.profile_enable(None)
            hs2.profile_read("dec_fused")
            graph, graph_note = None, f"eager (graph capture failed: {e})"
            torch.cuda.synchronize()
    launches = hs2.kernel_launches() - launches0
    with ClockSampler(local) as clocks:
        _barrier(world)
        if graph is None:
            launches0 = hs2.kernel_launches()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        clocks.start_region()
        e0.record(stream)
        if graph is not None:
            graph.replay()
        else:
            timed_steps()
        e1.record(stream)
        e1.synchronize()
        clocks.end_region()
        if graph is None:
            launches = hs2.kernel_launches() - launches0
        _barrier(world)
    ms_total = _max_over_ranks(e0.elapsed_time(e1), world)
    dec_ms, dec_n = hs2.profile_read("dec_fused")
    # the dominant kernel's launch time: 50 single launches, each timed by CUDA events, with the
    # clocks sampled over them
    with ClockSampler(local) as dclocks:
        dclocks.start_region()
        dec_times = time_launches(hs2, "dec_fused", step, 50)
        dclocks.end_region()
    # per-kernel breakdown (separate short run with every launch timed by CUDA events)
    hs2.profile_enable("*")
    n_brk = min(args.steps, 50)
    for _ in range(n_brk):
        step()
    torch.cuda.synchronize()
    hs2.profile_enable(None)
    breakdown = {}
    for name in ("dec_fused", "dec_redo", "sel_collect", "sel_rescore", "sel_final", "sparse_attn"):
        kms, kn = hs2.profile_read(name)
        if kn:
            breakdown[name] = kms / n_brk
    status = hs2.read_device_status(ws_full)
    status_sp = max(hs2.read_device_status(w) for w in ws_sp)
    ms_per_step = ms_total / args.steps
    value = _throughput(world, args.steps, ms_total)
    # the decode sparse layers' gathers: B rows x S selected K and V rows per layer
    sparse_gather = None
    if "sparse_attn" in breakdown:
        per_layer_ms = breakdown["sparse_attn"] / wl.n_sparse
        gb = wl.B * (wl.window + wl.topk) * wl.d * 2 * 2
        sparse_gather = {"achieved": gb / (per_layer_ms / 1e3) / 1e9, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                         "frac": gb / (per_layer_ms / 1e3) / 1e9 / peaks["hbm_gbs"], "bytes_per_layer": gb,
                         "ms_per_layer": per_layer_ms,
                         "note": "4.7 MB per layer: latency-bound (a dependent chain of gather, S, softmax, PV "
                                 "and cluster merge); at the HBM peak the bytes would take 0.7 us"}

    # ---------------- roofline of the dominant kernel (the fused decode kernel)
    ncand = wl.Lk - wl.window
    dec_bytes = wl.B * wl.Lk * wl.d * 2 * 2 + wl.B * ncand * 4   # K + V once from HBM, scores written
    roofline = dec_roofline(dec_times, dec_bytes, peaks, traffic=_traffic("dec_fused"), clocks=dclocks.summary())
    roofline["in_graph_avg_launch_ms"] = dec_ms / max(dec_n, 1)
    roofline["in_graph_launches_timed"] = dec_n
    step_bytes = (wl.B * wl.Lk * wl.d * 4 + (1 + wl.n_sparse) * wl.B * wl.H * wl.d * 4
                  + wl.n_sparse * wl.B * S * wl.d * 4 + wl.B * S * 4)
    step_roof = {"bound": "hbm", "algorithmic_bytes": step_bytes,
                 "achieved_gbs": step_bytes / (ms_per_step / 1e3) / 1e9,
                 "frac": step_bytes / (ms_per_step / 1e3) / 1e9 / peaks["hbm_gbs"]}

    # ---------------- end to end through the public API, host buffers. Per step: the full layer's
    # query and the new token's K/V rows go up from pinned memory first (the decode kernel needs
    # them), the rows join the cache; the sparse layers' queries go up on a copy stream while the
    # full layer runs; each layer's result (the full layer's output and indices, then each sparse
    # layer's output) comes back on the copy stream as soon as that layer is done, so only the
    # last layer's download follows the last kernel; the caller then waits for all of them.
    qn = q.numel()
    rown = wl.B * wl.d                                   # one new K (or V) row per sequence
    h_in0 = torch.empty(qn + 2 * rown, dtype=torch.bfloat16).pin_memory()
    h_in0[:qn].copy_(q.reshape(-1).cpu())
    pin = lambda a: torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16)
    h_in0[qn:qn + rown].copy_(pin(g.k[:, -1, :]).reshape(-1))
    h_in0[qn + rown:].copy_(pin(g.v[:, -1, :]).reshape(-1))
    h_in1 = torch.empty(qn * wl.n_sparse, dtype=torch.bfloat16).pin_memory()
    for i in range(wl.n_sparse):
        h_in1[qn * i:qn * (i + 1)].copy_(qs[i].reshape(-1).cpu())
    d_in0 = torch.empty_like(h_in0, device=dev)
    d_in1 = torch.empty_like(h_in1, device=dev)
    q_e = d_in0[:qn].view(q.shape)
    krow_e = d_in0[qn:qn + rown].view(wl.B, 1, wl.d)
    vrow_e = d_in0[qn + rown:].view(wl.B, 1, wl.d)
    qs_e = [d_in1[qn * i:qn * (i + 1)].view(q.shape) for i in range(wl.n_sparse)]
    on = out.numel()
    n_out0 = on * 2 + idx.numel() * 4                    # bytes: the full layer's output, the indices
    d_out0 = torch.empty(n_out0, dtype=torch.uint8, device=dev)
    h_out0 = torch.empty(n_out0, dtype=torch.uint8).pin_memory()
    out_e = d_out0[:on * 2].view(torch.bfloat16).view(out.shape)
    idx_e = d_out0[on * 2:].view(torch.int32).view(idx.shape)
    outs_e = [torch.empty_like(out) for _ in range(wl.n_sparse)]
    h_outs = [torch.empty(out.shape, dtype=torch.bfloat16).pin_memory() for _ in range(wl.n_sparse)]
    h2d = (h_in0.numel() + h_in1.numel()) * 2
    # the new token's K/V rows go from the upload buffer into row Lk - 1 of every sequence (pitch
    # Lk * d elements) by one 2-D device copy each, through the runtime torch already loaded
    cudart = ctypes.CDLL("libcudart.so.12")
    cudart.cudaMemcpy2DAsync.argtypes = [ctypes.c_void_p, ctypes.c_size_t, ctypes.c_void_p, ctypes.c_size_t,
                                         ctypes.c_size_t, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
    cudart.cudaMemcpyAsync.argtypes = [ctypes.c_void_p, ctypes.c_void_p, ctypes.c_size_t, ctypes.c_int, ctypes.c_void_p]
    up0 = (d_in0.data_ptr(), h_in0.data_ptr(), h_in0.numel() * 2, 1)  # cudaMemcpyHostToDevice
    last = wl.n_sparse - 1
    down_last = (h_outs[last].data_ptr(), outs_e[last].data_ptr(), outs_e[last].numel() * 2, 2)  # DeviceToHost
    copies_done = torch.cuda.Event()
    row_bytes, pitch = wl.d * 2, wl.Lk * wl.d * 2
    appends = ((k.data_ptr() + (wl.Lk - 1) * row_bytes, krow_e.data_ptr()),
               (v.data_ptr() + (wl.Lk - 1) * row_bytes, vrow_e.data_ptr()))
    d2d = 3  # cudaMemcpyDeviceToDevice
    step_done = torch.cuda.Event()
    d2h = n_out0 + wl.n_sparse * on * 2
    copy_stream = torch.cuda.Stream(device=dev)
    ev_in1 = torch.cuda.Event()
    ev_layer = [torch.cuda.Event() for _ in range(1 + wl.n_sparse)]

    def e2e_step():
        sp = stream.cuda_stream
        if cudart.cudaMemcpyAsync(*up0, sp):
            raise RuntimeError("cudaMemcpyAsync failed")
        for dst, src in appends:                         # the new token's K/V rows join the cache
            if cudart.cudaMemcpy2DAsync(dst, pitch, src, row_bytes, row_bytes, wl.B, d2d, sp):
                raise RuntimeError("cudaMemcpy2DAsync failed")
        hs2.full_attn_select(q_e, k, v, scale=wl.scale, out=out_e, lse=lse, idx=idx_e, workspace=ws_full)
        ev_layer[0].record(stream)
        with torch.cuda.stream(copy_stream):
            d_in1.copy_(h_in1, non_blocking=True)
            ev_in1.record(copy_stream)
            copy_stream.wait_event(ev_layer[0])
            h_out0.copy_(d_out0, non_blocking=True)
        stream.wait_event(ev_in1)
        for i in range(wl.n_sparse):
            hs2.sparse_attn(qs_e[i], k, v, idx_e, scale=wl.scale, out=outs_e[i], workspace=ws_sp[i])
            if i == last:  # the last layer's output comes back on its own stream, right after it
                if cudart.cudaMemcpyAsync(*down_last, sp):
                    raise RuntimeError("cudaMemcpyAsync failed")
                break
            ev_layer[i + 1].record(stream)
            with torch.cuda.stream(copy_stream):
                copy_stream.wait_event(ev_layer[i + 1])
                h_outs[i].copy_(outs_e[i], non_blocking=True)
        copies_done.record(copy_stream)
        step_done.record(stream)
        while not (step_done.query() and copies_done.query()):  # the caller waits for the results
            pass

    # enough steps that a single host hiccup (a page fault, a scheduler tick) does not set the number
    e2e_steps = max(200, min(args.steps, 1000))
    for _ in range(10):
        e2e_step()
    _barrier(world)
    f0, f1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    f0.record(stream)
    for _ in range(e2e_steps):
        e2e_step()
    f1.record(stream)
    f1.synchronize()
    _barrier(world)
    e2e_ms = _max_over_ranks(f0.elapsed_time(f1), world)
    e2e_value = _throughput(world, e2e_steps, e2e_ms)

    # ---------------- ragged decode (a batch of different cache lengths in the same buffers)
    ragged = None
    if not args.no_ragged:
        ragged = bench_ragged(args, world, wl, hs2, q, k, v, qs, peaks)

    # ---------------- the same decode step over an FP8 (e4m3) K/V cache
    fp8 = None
    if not args.no_fp8:
        fp8 = bench_fp8(args, world, wl, hs2, q, k, v, qs, peaks)

    # ---------------- the HySparse (v1) block-level step at the same budget
    v1 = None
    if not args.no_v1:
        v1 = bench_v1(args, world, wl, hs2, q, k, v, qs, peaks, value)

    # ---------------- prefill (secondary clause of the metric)
    prefill = None
    if not args.no_prefill:
        prefill = bench_prefill(args, world, dev, peaks)

    # ---------------- backward of a hybrid block at the training shape
    backward = None
    if not args.no_backward:
        backward = bench_backward(args, world, dev, peaks)

    # ---------------- the other configurations of the method's synthetic workloads
    configs = None
    if not args.no_configs:
        gpu_idx = idx.reshape(wl.B, S).cpu().numpy()
        configs = {}
        for name in ("decode_32k", "decode_1m"):
            configs[name] = bench_decode_config(args, world, rank, dev, peaks, name)
        configs["tiny_prefill"] = bench_tiny(args, world, rank, dev, peaks)
    else:
        gpu_idx = None

    launches_total = int(_sum_over_ranks(launches, world))
    if rank == 0:
        cpu, sel = None, None
        if world == 1 and not args.no_cpu_baseline:
            cpu, sel = cpu_baseline(g, gpu_idx=gpu_idx)
        line = {
            "metric": METRIC, "value": value, "unit": "steps/s", "n_gpus": world, "steps": args.steps,
            "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
            "config": {"workload": f"{wl.name}: B={wl.B} sequences per GPU, {wl.Lk}-token MQA K/V cache, "
                                   f"H={wl.H}, d={wl.d}, window {wl.window} + top-{wl.topk}, "
                                   f"{wl.n_sparse} sparse layers per step",
                       "global_batch": wl.B * world, "seq_len": wl.Lk, "parallelism": f"dp{world} (replicas)",
                       "l2": "inputs larger than L2 (1.07 GB K+V per GPU), no flush",
                       "launch": (f"the {args.steps} timed steps replayed as one CUDA graph" if graph is not None
                                  else (graph_note or "eager launches"))},
            "roofline": roofline, "step_roofline": step_roof, "kernel_ms_per_step": breakdown,
            "sparse_gather": sparse_gather,
            "e2e": {"value": e2e_value, "unit": "steps/s", "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h,
                    "steps": e2e_steps, "note": "public Python API; per step from pinned memory: the full layer's query and the new token's K/V rows (one copy; the rows then written into the cache by a 2-D device copy each), the sparse layers' queries (one copy on a second stream, overlapping the full layer); each layer's results copied back on that stream once the layer is done; the step ends when the last copy has landed (polled)"},
            "gpu_launches": launches_total, "clocks": clocks.summary(),
            "device_status": [status, status_sp], "cpu_baseline": cpu, "selection_check": sel,
            "ragged": ragged, "fp8_kv": fp8, "v1": v1, "prefill": prefill, "backward": backward, "configs": configs,
        }
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return 0


def time_launches(hs2, kernel: str, fn, n: int = 50):
    """CUDA-event duration of each of n launches of `kernel`: fn() runs one step eagerly with the
    library's events around that kernel's launch, and the step is waited for before the next (the
    launch list then has one entry per step). Returns the per-launch times in ms."""
    import torch
    times = []
    for _ in range(n):
        hs2.profile_enable(kernel)
        fn()
        hs2.profile_enable(None)
        ms, k = hs2.profile_read(kernel)
        if k:
            times.append(ms / k)
    torch.cuda.synchronize()
    return times


def dec_roofline(times_ms, dec_bytes, peaks, kernel="dec_fused", traffic=None, clocks=None):
    med = statistics.median(times_ms)
    gbs = dec_bytes / (med / 1e3) / 1e9
    r = {"kernel": kernel, "bound": "hbm", "achieved": gbs, "peak": peaks["hbm_gbs"], "unit": "GB/s",
         "frac": gbs / peaks["hbm_gbs"], "traffic": traffic, "peak_source": peaks["source"],
         "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_ms": med, "mean_launch_ms": statistics.fmean(times_ms),
         "min_launch_ms": min(times_ms), "max_launch_ms": max(times_ms), "launches_timed": len(times_ms),
         "timed_launches_note": "median of CUDA-event durations of single launches, one per eagerly launched "
                                "step (each step waited for)"}
    if clocks is not None:
        r["clocks_during_launches"] = clocks
    return r


def bench_decode_config(args, world, rank, dev, peaks, name, steps=200, warmup=5):
    """A decode workload other than the headline one (decode_32k, decode_1m): the same step (one
    hs2_full_attn_select with Lq = 1, then the sparse layers) replayed as one CUDA graph of
    `steps` steps; the fused decode kernel's roofline from >= 25 single-launch timings; the
    sparse layer's time; the oracle's cpu_baseline and swap count on the same inputs."""
    import torch
    import long_context_mqa_b200 as hs2
    wl = synth.WORKLOADS[name]
    g = synth.SyntheticInputs(wl, seed=args.seed + rank)
    q, k, v = _bf16(g.q, dev), _bf16(g.k, dev), _bf16(g.v, dev)
    qs = [_bf16(g.q_sparse(i), dev) for i in range(wl.n_sparse)]
    S = wl.window + wl.topk
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, 1, wl.H), dtype=torch.float32, device=dev)
    idx = torch.empty((wl.B, 1, S), dtype=torch.int32, device=dev)
    outs = [torch.empty_like(q) for _ in range(wl.n_sparse)]
    ws = torch.zeros(hs2.full_attn_select_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d), dtype=torch.uint8, device=dev)
    ws_sp = [torch.zeros(hs2.sparse_attn_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d, S), dtype=torch.uint8,
                         device=dev) for _ in range(wl.n_sparse)]
    stream = torch.cuda.current_stream()

    def step():
        hs2.full_attn_select(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws)
        for i in range(wl.n_sparse):
            hs2.sparse_attn(qs[i], k, v, idx, scale=wl.scale, out=outs[i], workspace=ws_sp[i])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            step()
    graph.replay()
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with ClockSampler(dev.index or 0) as clocks:
        clocks.start_region()
        e0.record(stream)
        graph.replay()
        e1.record(stream)
        e1.synchronize()
        clocks.end_region()
    _barrier(world)
    ms = _max_over_ranks(e0.elapsed_time(e1), world)
    del graph
    times = time_launches(hs2, "dec_fused", step, 30)
    hs2.profile_enable("sparse_attn")
    for _ in range(10):
        step()
    torch.cuda.synchronize()
    hs2.profile_enable(None)
    sp_ms, sp_n = hs2.profile_read("sparse_attn")
    status = [hs2.read_device_status(ws), max(hs2.read_device_status(w) for w in ws_sp)]
    dec_bytes = wl.B * wl.Lk * wl.d * 2 * 2 + wl.B * (wl.Lk - wl.window) * 4
    res = {"workload": f"{wl.name}: B={wl.B} sequences, {wl.Lk}-token MQA K/V cache, H={wl.H}, d={wl.d}, "
                       f"window {wl.window} + top-{wl.topk}, {wl.n_sparse} sparse layers per step",
           "value": _throughput(world, steps, ms), "unit": "steps/s", "ms_per_step": ms / steps,
           "tok_per_s": _throughput(world, steps, ms) * wl.B, "launch": f"{steps} steps replayed as one CUDA graph",
           "clocks": clocks.summary(),
           "roofline": dec_roofline(times, dec_bytes, peaks),
           "sparse_layer_ms": sp_ms / max(sp_n, 1), "device_status": status}
    gb = wl.B * S * wl.d * 2 * 2
    res["sparse_gather"] = {"achieved": gb / (res["sparse_layer_ms"] / 1e3) / 1e9, "unit": "GB/s",
                            "peak": peaks["hbm_gbs"], "bytes_per_layer": gb,
                            "frac": gb / (res["sparse_layer_ms"] / 1e3) / 1e9 / peaks["hbm_gbs"],
                            "note": "CUDA events around each sparse layer launch (eager): latency-bound"}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        res["cpu_baseline"], res["selection_check"] = cpu_baseline(g, budget_s=15.0, min_s=8.0,
                                                                   gpu_idx=idx.reshape(wl.B, S).cpu().numpy())
    del q, k, v, qs, out, outs, ws, ws_sp
    torch.cuda.empty_cache()
    return res


def bench_tiny(args, world, rank, dev, peaks, reps=50):
    """The tiny prefill workload (L = 2048, 16 heads, head_dim 64): one step = the full layer with
    selection over every row, then one sparse layer. Latency-bound at this size; reported as
    tok/s with the executed tensor flops against the dense bf16 peak. The oracle runs the same
    step in full (every row) for the cpu_baseline and the swap count."""
    import torch
    import long_context_mqa_b200 as hs2
    wl = synth.WORKLOADS["tiny_prefill"]
    g = synth.SyntheticInputs(wl, seed=args.seed + rank)
    q, k, v = _bf16(g.q, dev), _bf16(g.k, dev), _bf16(g.v, dev)
    q1 = _bf16(g.q_sparse(0), dev)
    S = wl.window + wl.topk
    out = torch.empty_like(q)
    out1 = torch.empty_like(q)
    lse = torch.empty((1, wl.Lq, wl.H), dtype=torch.float32, device=dev)
    idx = torch.empty((1, wl.Lq, S), dtype=torch.int32, device=dev)
    ws = torch.zeros(hs2.full_attn_select_workspace_bytes(1, wl.Lq, wl.Lk, wl.H, wl.d), dtype=torch.uint8, device=dev)
    ws1 = torch.zeros(hs2.sparse_attn_workspace_bytes(1, wl.Lq, wl.Lk, wl.H, wl.d, S), dtype=torch.uint8, device=dev)
    s = torch.cuda.current_stream()

    def step():
        hs2.full_attn_select(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws)
        hs2.sparse_attn(q1, k, v, idx, scale=wl.scale, out=out1, workspace=ws1)

    for _ in range(5):
        step()
    torch.cuda.synchronize()
    launch = f"{reps} steps replayed as one CUDA graph"
    try:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(reps):
                step()
        graph.replay()
        torch.cuda.synchronize()
    except Exception as e:
        graph, launch = None, f"eager launches (graph capture failed: {e})"
        torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    if graph is not None:
        graph.replay()
    else:
        for _ in range(reps):
            step()
    e1.record(s)
    e1.synchronize()
    _barrier(world)
    ms = _max_over_ranks(e0.elapsed_time(e1), world) / reps
    del graph
    hs2.profile_enable("*")
    for _ in range(20):
        step()
    torch.cuda.synchronize()
    hs2.profile_enable(None)
    kern = {}
    for name in ("fa_fwd", "score_select", "sparse_attn"):
        kms, kn = hs2.profile_read(name)
        if kn:
            kern[name] = kms / kn
    L = wl.Lq
    P = L * (L + 1) / 2
    sel_pairs = sum(min(t + 1, S) for t in range(L))
    flops = 6 * wl.H * wl.d * P + 4 * wl.H * wl.d * sel_pairs
    tf = flops / (ms / 1e3) / 1e12
    res = {"workload": f"tiny_prefill: L={L}, H={wl.H}, d={wl.d}, scale 1/8, full layer with selection + 1 sparse "
                       f"layer per step", "tok_per_s": world * L / (ms / 1e3), "ms_per_step": ms, "launch": launch,
           "kernel_ms": kern,
           "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": tf / peaks["bf16_tflops"], "peak_source": peaks["source"] + " burst",
                        "flops": "executed 6*H*d*L(L+1)/2 (full layer) + 4*H*d*sum_t min(t+1, S) (sparse layer)",
                        "note": "latency-bound at this size (a few waves of small tiles)"},
           "device_status": [hs2.read_device_status(ws), hs2.read_device_status(ws1)]}
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        import oracle
        t0 = time.perf_counter()
        r = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, wl.window, wl.topk, want_score=True)
        oracle.sparse_attn(g.q_sparse(0), g.k, g.v, r["idx"].reshape(1, L, S), wl.scale)
        dt = time.perf_counter() - t0
        res["cpu_baseline"] = {"value": L / dt, "unit": "tok/s", "cores": oracle.default_threads(), "kind": "oracle",
                               "sample": f"the whole step (all {L} rows, full layer + 1 sparse layer), {dt:.1f} s, "
                                         f"no extrapolation (the oracle also keeps every row's score vector)"}
        sys.path.insert(0, os.path.join(ROOT, "tests"))
        from parity import check_selection
        st = check_selection(idx.reshape(L, S).cpu().numpy(), r["idx"], r["score"], np.arange(L), wl.window, wl.topk)
        res["selection_check"] = {"rows": st.rows, "swaps": st.swaps, "max_swap_rel": st.max_swap_rel, "ok": st.ok()}
    return res


def bench_v1(args, world, wl, hs2, q, k, v, qs, peaks, token_value, steps=200, warmup=5):
    """The HySparse (v1) decode step on the headline inputs, at the same budget as the token-level
    step (1,024 tokens by score + the 128-token window): hs2_full_attn_select_v1 (16 blocks of 64
    tokens), then the sparse layers as hs2_sparse_attn_v1 (block branch + window branch, mixed by
    a seeded gate in [0, 1] per (sequence, head)), one CUDA graph; device-timed like the main line."""
    import torch
    S = 16 * 64 + wl.window
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, 1, wl.H), dtype=torch.float32, device=q.device)
    idx = torch.empty((wl.B, 1, S), dtype=torch.int32, device=q.device)
    outs = [torch.empty_like(q) for _ in range(wl.n_sparse)]
    rng = np.random.default_rng(7)
    gates = [torch.from_numpy(rng.uniform(0.0, 1.0, size=(wl.B, 1, wl.H)).astype(np.float32)).to(q.device)
             for _ in range(wl.n_sparse)]
    ws = torch.zeros(hs2.full_attn_select_v1_workspace_bytes(wl.B, wl.Lk, wl.H, wl.d), dtype=torch.uint8,
                     device=q.device)
    ws_sp = [torch.zeros(hs2.sparse_attn_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d, S), dtype=torch.uint8,
                         device=q.device) for _ in range(wl.n_sparse)]
    stream = torch.cuda.current_stream()

    def step():
        hs2.full_attn_select_v1(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws)
        for i in range(wl.n_sparse):
            hs2.sparse_attn_v1(qs[i], k, v, idx, gates[i], scale=wl.scale, out=outs[i], workspace=ws_sp[i])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            step()
    graph.replay()
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    e1.synchronize()
    _barrier(world)
    ms = _max_over_ranks(e0.elapsed_time(e1), world)
    del graph
    hs2.profile_enable("*")
    for _ in range(20):
        step()
    torch.cuda.synchronize()
    hs2.profile_enable(None)
    kern = {}
    for name in ("dec_fused", "dec_redo", "blk_score", "blk_final", "sparse_attn"):
        kms, kn = hs2.profile_read(name)
        if kn:
            kern[name] = kms / 20
    value = _throughput(world, steps, ms)
    return {"workload": f"{wl.name} inputs, HySparse (v1): 16 blocks of 64 tokens by block score + a gated "
                        f"{wl.window}-token window branch, {wl.n_sparse} gated sparse layers per step (the same "
                        f"1,152-token budget as the token-level step)",
            "value": value, "unit": "steps/s", "ms_per_step": ms / steps,
            "vs_token_level": value / token_value if token_value else None,
            "kernel_ms_per_step": kern, "device_status": [hs2.read_device_status(ws),
                                                          max(hs2.read_device_status(w) for w in ws_sp)]}


def bench_backward(args, world, dev, peaks, reps=3):
    """Backward of one hybrid block at the training shape (prefill_32k: L = 32,768, 64 heads,
    d = 128): the full layer's hs2_full_attn_bwd and the sparse layers' hs2_sparse_attn_bwd (each
    over the full layer's selection with its own Q), adding into one pair of fp32 dK, dV buffers.
    Reported as tok/s of the block's backward and the tensor rate of each kernel family."""
    import torch
    import long_context_mqa_b200 as hs2
    wl = synth.WORKLOADS[PREFILL_WORKLOAD]
    g = synth.SyntheticInputs(wl, seed=args.seed)
    q, k, v = _bf16(g.q, dev), _bf16(g.k, dev), _bf16(g.v, dev)
    out, lse, idx = hs2.full_attn_select(q, k, v, scale=wl.scale)
    S = wl.window + wl.topk
    qs = [_bf16(g.q_sparse(i), dev) for i in range(wl.n_sparse)]
    fw = [hs2.sparse_attn(qs[i], k, v, idx, scale=wl.scale, want_lse=True) for i in range(wl.n_sparse)]
    dos = [_bf16(g.grad_out(i), dev) for i in range(wl.n_sparse + 1)]
    dq = torch.empty_like(q)
    dqs = [torch.empty_like(q) for _ in range(wl.n_sparse)]
    dk = torch.zeros((1, wl.Lk, wl.d), dtype=torch.float32, device=dev)
    dv = torch.zeros_like(dk)
    ws = torch.zeros(hs2.attn_bwd_workspace_bytes(1, wl.Lq, wl.Lk, wl.H, wl.d), dtype=torch.uint8, device=dev)

    def block_bwd():
        dk.zero_()
        dv.zero_()
        hs2.full_attn_bwd(q, k, v, out, lse, dos[0], scale=wl.scale, dq=dq, dk=dk, dv=dv, workspace=ws)
        for i in range(wl.n_sparse):
            hs2.sparse_attn_bwd(qs[i], k, v, idx, fw[i][0], fw[i][1], dos[i + 1], scale=wl.scale, dq=dqs[i], dk=dk,
                                dv=dv, workspace=ws)

    block_bwd()
    torch.cuda.synchronize()
    _barrier(world)
    s = torch.cuda.current_stream()
    hs2.profile_enable("*")
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        block_bwd()
    e1.record(s)
    e1.synchronize()
    hs2.profile_enable(None)
    ms = _max_over_ranks(e0.elapsed_time(e1), world) / reps
    kern = {}
    for name in ("bwd_prep", "bwd_dq", "bwd_dkdv", "sparse_bwd"):
        kms, kn = hs2.profile_read(name)
        if kn:
            kern[name] = kms / reps
    P = wl.Lq * (wl.Lq + 1) / 2
    dq_fl, kv_fl = 6 * wl.H * wl.d * P, 8 * wl.H * wl.d * P      # executed: S, dP recomputed by both
    sel_pairs = sum(min(t + 1, S) for t in range(wl.Lq))
    sp_fl = 10 * wl.H * wl.d * sel_pairs                          # per sparse layer: S, dP, dQ, dK, dV
    res = {"workload": f"{wl.name}: backward of one hybrid block (full layer + {wl.n_sparse} sparse layers), "
                       f"L={wl.Lq}, H={wl.H}, d={wl.d}; dK, dV accumulated over the layers",
           "tok_per_s": world * wl.Lq / (ms / 1e3), "ms": ms, "kernel_ms": kern,
           "status": hs2.read_device_status(ws)}
    if "bwd_dq" in kern and "bwd_dkdv" in kern:
        full_ms = kern["bwd_dq"] + kern["bwd_dkdv"]
        tf = (dq_fl + kv_fl) / (full_ms / 1e3) / 1e12
        res["full_roofline"] = {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                "frac": tf / peaks["bf16_tflops"],
                                "flops": "executed 14*H*d*L(L+1)/2 (dq kernel: S, dP, dQ; dkdv kernel: S^T, dP^T, dV, dK)",
                                "algorithmic_tflops": 10 * wl.H * wl.d * P / (full_ms / 1e3) / 1e12,
                                "dq_tflops": dq_fl / (kern["bwd_dq"] / 1e3) / 1e12,
                                "dkdv_tflops": kv_fl / (kern["bwd_dkdv"] / 1e3) / 1e12}
    if "sparse_bwd" in kern:
        per = kern["sparse_bwd"] / wl.n_sparse
        tf = sp_fl / (per / 1e3) / 1e12
        res["sparse_roofline"] = {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                  "frac": tf / peaks["bf16_tflops"], "ms_per_layer": per,
                                  "flops": "10*H*d*sum_t min(t+1, S) per layer"}
    if world == 1 and not args.no_cpu_baseline and int(os.environ.get("RANK", "0")) == 0:
        import oracle
        rows = np.concatenate([np.arange(8) + int((i + 0.5) * wl.Lq / 8) - 4 for i in range(8)])
        t0 = time.perf_counter()
        oracle.attn_bwd(g.q, g.k, g.v, g.grad_out(0), wl.scale, rows=rows, want_kv=False)
        dt = time.perf_counter() - t0
        # the dQ rows' share of the full layer's backward: the K/V side repeats the same row work
        est = dt * wl.Lq / rows.size * 2.0
        res["cpu_baseline"] = {"value": wl.Lq / est, "unit": "tok/s", "cores": oracle.default_threads(),
                               "kind": "oracle", "sample": f"the full layer's dQ on {rows.size} rows (8 evenly spaced "
                               f"strata), {dt:.1f} s, x{wl.Lq // rows.size} rows x2 for the key-side pass of the same "
                               f"work (extrapolated; the sparse layers are not included)"}
    del q, k, v, out, lse, idx, qs, fw, dos, dq, dqs, dk, dv
    torch.cuda.empty_cache()
    return res


RAGGED_FRACTIONS = (1.0, 0.75, 0.5, 0.375, 0.25, 0.125, 0.0625, 0.015625)


def bench_ragged(args, world, wl, hs2, q, k, v, qs, peaks, steps=200, warmup=5):
    """Decode steps over a ragged batch: sequence b keeps the first lens[b] rows of the bench's
    cache (lengths from the full cache down to 1/64 of it), one hs2_full_attn_select_ragged plus
    the sparse layers per step, as one CUDA graph; device-timed like the main line."""
    import torch
    lens = [max(1, int(wl.Lk * RAGGED_FRACTIONS[b % len(RAGGED_FRACTIONS)])) for b in range(wl.B)]
    S = wl.window + wl.topk
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, 1, wl.H), dtype=torch.float32, device=q.device)
    idx = torch.empty((wl.B, 1, S), dtype=torch.int32, device=q.device)
    outs = [torch.empty_like(q) for _ in range(wl.n_sparse)]
    ws = torch.zeros(hs2.full_attn_select_ragged_workspace_bytes(lens, wl.Lk, wl.H, wl.d), dtype=torch.uint8,
                     device=q.device)
    ws_sp = [torch.zeros(hs2.sparse_attn_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d, S), dtype=torch.uint8,
                         device=q.device) for _ in range(wl.n_sparse)]
    stream = torch.cuda.current_stream()

    def step():
        hs2.full_attn_select_ragged(q, k, v, lens, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws)
        for i in range(wl.n_sparse):
            hs2.sparse_attn(qs[i], k, v, idx, scale=wl.scale, out=outs[i], workspace=ws_sp[i])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(steps):
            hs2.profile_enable("dec_fused" if i % 8 == 0 else None)
            step()
        hs2.profile_enable(None)
    graph.replay()            # upload and warm (the timing events of the replay below overwrite its own)
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    e1.synchronize()
    _barrier(world)
    ms = _max_over_ranks(e0.elapsed_time(e1), world)
    dec_ms, dec_n = hs2.profile_read("dec_fused")
    status = hs2.read_device_status(ws)
    del graph

    # the same tokens in 128-token pages scattered over shared pools (a page table per sequence)
    rng = np.random.default_rng(1)
    tiles = [(n + 127) // 128 for n in lens]
    n_pages, max_pages = sum(tiles), max(tiles)
    perm = rng.permutation(n_pages)
    kp = torch.empty((n_pages, 128, wl.d), dtype=torch.bfloat16, device=q.device)
    vp = torch.empty_like(kp)
    table = np.zeros((wl.B, max_pages), np.int32)
    nxt = 0
    for b, n in enumerate(lens):
        for i in range(tiles[b]):
            pg = int(perm[nxt]); nxt += 1
            table[b, i] = pg
            r = min(128, n - 128 * i)
            kp[pg, :r] = k[b, 128 * i:128 * i + r]
            vp[pg, :r] = v[b, 128 * i:128 * i + r]
    table = torch.from_numpy(table).to(q.device)
    ws_p = torch.zeros(hs2.full_attn_select_paged_workspace_bytes(lens, max_pages, wl.H, wl.d), dtype=torch.uint8,
                       device=q.device)

    def step_paged():
        hs2.full_attn_select_paged(q, kp, vp, table, lens, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws_p)
        for i in range(wl.n_sparse):
            hs2.sparse_attn_paged(qs[i], kp, vp, table, idx, scale=wl.scale, out=outs[i], workspace=ws_sp[i])

    for _ in range(warmup):
        step_paged()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for _ in range(steps):
            step_paged()
    graph.replay()
    torch.cuda.synchronize()
    _barrier(world)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    e1.synchronize()
    _barrier(world)
    ms_p = _max_over_ranks(e0.elapsed_time(e1), world)
    status_p = hs2.read_device_status(ws_p)
    del graph, kp, vp

    dec_bytes = sum(n * wl.d * 2 * 2 + max(n - wl.window, 0) * 4 for n in lens)
    dec_s = dec_ms / max(dec_n, 1) / 1e3
    return {"workload": f"decode_ragged: B={wl.B} sequences of {lens} tokens in the {wl.Lk}-row cache buffers, "
                        f"H={wl.H}, d={wl.d}, window {wl.window} + top-{wl.topk}, {wl.n_sparse} sparse layers",
            "value": _throughput(world, steps, ms), "unit": "steps/s", "ms_per_step": ms / steps,
            "tokens_per_step": sum(lens),
            "roofline": {"kernel": "dec_fused", "bound": "hbm", "achieved": dec_bytes / dec_s / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dec_bytes / dec_s / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_ms": dec_s * 1e3,
                         "launches_timed": dec_n},
            "paged": {"value": _throughput(world, steps, ms_p), "unit": "steps/s", "ms_per_step": ms_p / steps,
                      "layout": f"the same tokens in {n_pages} pages of 128 tokens, randomly placed in shared pools, "
                                f"one page-table row per sequence", "device_status": status_p},
            "device_status": status}


def bench_fp8(args, world, wl, hs2, q, k, v, qs, peaks, steps=200, warmup=5):
    """The decode step over the bench's cache stored as e4m3 codes (one power-of-two scale per
    tensor: the bf16 cache divided by 2^ceil(log2(max|x| / 448)) and rounded by torch's float8
    conversion on the device), one hs2_full_attn_select_fp8kv plus the sparse layers over the same
    codes per step, as one CUDA graph; device-timed like the main line."""
    import torch

    def quant(x):
        amax = float(x.abs().max())
        sc = 2.0 ** math.ceil(math.log2(amax / 448.0)) if amax > 0 else 1.0
        return (x.float() / sc).to(torch.float8_e4m3fn).view(torch.uint8).contiguous(), sc

    k8, ks = quant(k)
    v8, vs = quant(v)
    S = wl.window + wl.topk
    out = torch.empty_like(q)
    lse = torch.empty((wl.B, 1, wl.H), dtype=torch.float32, device=q.device)
    idx = torch.empty((wl.B, 1, S), dtype=torch.int32, device=q.device)
    outs = [torch.empty_like(q) for _ in range(wl.n_sparse)]
    ws = torch.zeros(hs2.full_attn_select_fp8kv_workspace_bytes(wl.B, None, wl.Lk, wl.H, wl.d), dtype=torch.uint8,
                     device=q.device)
    ws_sp = [torch.zeros(hs2.sparse_attn_workspace_bytes(wl.B, 1, wl.Lk, wl.H, wl.d, S), dtype=torch.uint8,
                         device=q.device) for _ in range(wl.n_sparse)]
    stream = torch.cuda.current_stream()

    def step():
        hs2.full_attn_select_fp8kv(q, k8, v8, ks, vs, scale=wl.scale, out=out, lse=lse, idx=idx, workspace=ws)
        for i in range(wl.n_sparse):
            hs2.sparse_attn_fp8kv(qs[i], k8, v8, ks, vs, idx, scale=wl.scale, out=outs[i], workspace=ws_sp[i])

    for _ in range(warmup):
        step()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        for i in range(steps):
            hs2.profile_enable("dec_fused" if i % 8 == 0 else None)
            step()
        hs2.profile_enable(None)
    graph.replay()
    torch.cuda.synchronize()
    _barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(stream)
    graph.replay()
    e1.record(stream)
    e1.synchronize()
    _barrier(world)
    ms = _max_over_ranks(e0.elapsed_time(e1), world)
    dec_ms, dec_n = hs2.profile_read("dec_fused")
    status = hs2.read_device_status(ws)
    del graph, k8, v8
    # one byte per cached K and V element, plus the 4-byte score of each older token
    dec_bytes = wl.B * (wl.Lk * wl.d * 2 + max(wl.Lk - wl.window, 0) * 4)
    dec_s = dec_ms / max(dec_n, 1) / 1e3
    return {"workload": f"{wl.name} with the K/V cache as e4m3 codes ({wl.B * wl.Lk * wl.d * 2 / 1e6:.0f} MB, half "
                        f"the bf16 bytes), per-tensor power-of-two scales",
            "value": _throughput(world, steps, ms), "unit": "steps/s", "ms_per_step": ms / steps,
            "roofline": {"kernel": "dec_fused (e4m3)", "bound": "hbm", "achieved": dec_bytes / dec_s / 1e9,
                         "peak": peaks["hbm_gbs"], "unit": "GB/s", "frac": dec_bytes / dec_s / 1e9 / peaks["hbm_gbs"],
                         "algorithmic_bytes_per_launch": dec_bytes, "avg_launch_ms": dec_s * 1e3,
                         "launches_timed": dec_n, "traffic": _traffic("dec_fused_e4m3")},
            "device_status": status}


def prefill_cpu_baseline(g, idx_gpu, n_strata=16, per_stratum=32):
    """The oracle's full layer (attention, scores, selection) on 512 sampled query rows of the
    prefill workload: 16 evenly spaced strata of 32 consecutive rows, so the sampled rows' mean
    position is L/2 and their time x L/512 estimates the whole prompt (labelled extrapolated).
    The same rows give the selection's swap count against the GPU's idx."""
    import oracle
    wl = g.wl
    L, S = wl.Lq, wl.window + wl.topk
    rows = np.concatenate([np.arange(per_stratum) + int((i + 0.5) * L / n_strata) - per_stratum // 2
                           for i in range(n_strata)])
    t0 = time.perf_counter()
    r = oracle.full_attn_select(g.q, g.k, g.v, wl.scale, wl.window, wl.topk, rows=rows, want_score=True)
    dt = time.perf_counter() - t0
    est = dt * L / rows.size
    base = {"value": L / est, "unit": "tok/s", "cores": oracle.default_threads(), "kind": "oracle",
            "sample": f"{rows.size} query rows ({n_strata} evenly spaced strata of {per_stratum} consecutive rows, "
                      f"mean position {rows.mean():.0f} of {L}), full layer with scores and selection, {dt:.1f} s; "
                      f"x{L // rows.size} (extrapolated)"}
    sys.path.insert(0, os.path.join(ROOT, "tests"))
    from parity import check_selection
    gi = idx_gpu.reshape(L, S).cpu().numpy()[rows]
    st = check_selection(gi, r["idx"], r["score"], rows, wl.window, wl.topk)
    sel = {"rows": st.rows, "swaps": st.swaps, "max_swap_rel": st.max_swap_rel, "ok": st.ok()}
    return base, sel


def bench_prefill(args, world, dev, peaks, reps=5, warmup=2):
    """Full-attention + top-k prefill on the 32k workload: tok/s and tensor roofline."""
    import torch
    import long_context_mqa_b200 as hs2
    wl = synth.WORKLOADS[PREFILL_WORKLOAD]
    if args.prefill_len:   # reduced case for profiler captures
        wl = wl.with_(name=f"{PREFILL_WORKLOAD}_L{args.prefill_len}", Lq=args.prefill_len, Lk=args.prefill_len)
    g = synth.SyntheticInputs(wl, seed=args.seed)
    try:
        q, k, v = _bf16(g.q, dev), _bf16(g.k, dev), _bf16(g.v, dev)
        out = torch.empty_like(q)
        lse = torch.empty((1, wl.Lq, wl.H), dtype=torch.float32, device=dev)
        idx = torch.empty((1, wl.Lq, wl.window + wl.topk), dtype=torch.int32, device=dev)
        hs2.full_attn_select(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx)
    except Exception as e:  # the prefill path reports its own absence
        return {"status": f"unavailable: {e}"}
    n_sparse = wl.n_sparse if args.sparse_layers < 0 else args.sparse_layers
    qs = [_bf16(g.q_sparse(i), dev) for i in range(n_sparse)]
    outs = torch.empty_like(q)
    for _ in range(warmup):
        hs2.full_attn_select(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx)
        for i in range(n_sparse):
            hs2.sparse_attn(qs[i], k, v, idx, scale=wl.scale, out=outs)
    _barrier(world)
    hs2.profile_enable("*")
    s = torch.cuda.current_stream()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s)
    for _ in range(reps):
        hs2.full_attn_select(q, k, v, scale=wl.scale, out=out, lse=lse, idx=idx)
    e1.record(s)
    e1.synchronize()
    hs2.profile_enable(None)
    kern = {}
    for name in ("fa_fwd", "score_select"):
        kms, kn = hs2.profile_read(name)
        kern[name] = kms / max(kn, 1)
    if n_sparse:
        t0 = torch.cuda.Event(enable_timing=True)
        t1 = torch.cuda.Event(enable_timing=True)
        t0.record(s)
        for _ in range(reps):
            for i in range(n_sparse):
                hs2.sparse_attn(qs[i], k, v, idx, scale=wl.scale, out=outs)
        t1.record(s)
        t1.synchronize()
        kern["sparse_attn_per_layer"] = t0.elapsed_time(t1) / (reps * n_sparse)
    hs2.profile_read("sparse_attn")
    ms = _max_over_ranks(e0.elapsed_time(e1), world) / reps
    P = wl.Lq * (wl.Lq + 1) / 2
    exec_flops = 6 * wl.H * wl.d * P
    alg_flops = 4 * wl.H * wl.d * P
    tf = exec_flops / (ms / 1e3) / 1e12
    res = {"workload": f"{wl.name}: L={wl.Lq}, H={wl.H}, d={wl.d}", "tok_per_s": world * wl.Lq / (ms / 1e3),
           "ms": ms, "kernel_ms": kern,
           "roofline": {"bound": "tensor", "achieved": tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                        "frac": tf / peaks["bf16_tflops"], "peak_source": peaks["source"] + " burst (the call is timed "
                        "alone, a few reps)", "frac_of_sustained": tf / peaks["bf16_tflops_sustained"],
                        "flops": "executed 6*H*d*L(L+1)/2 (QK^T twice, PV once)",
                        "algorithmic_tflops": alg_flops / (ms / 1e3) / 1e12}}
    if not args.prefill_len and world == 1 and not args.no_cpu_baseline and int(os.environ.get("RANK", "0")) == 0:
        res["cpu_baseline"], res["selection_check"] = prefill_cpu_baseline(g, idx)
    if n_sparse and "sparse_attn_per_layer" in kern:
        sp_flops = 4 * wl.H * wl.d * (wl.window + wl.topk) * wl.Lq   # QK^T and PV over the selected rows
        sp_tf = sp_flops / (kern["sparse_attn_per_layer"] / 1e3) / 1e12
        res["sparse_roofline"] = {"bound": "tensor", "achieved": sp_tf, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                                  "frac": sp_tf / peaks["bf16_tflops"], "flops": "4*H*d*S*L per layer"}
        # the gather side of the same layer: every query row gathers its S selected K and V rows
        # (2*d bf16 each) once for all heads; the cache is L2-resident, so this is the rate at which
        # the kernel moves gathered rows, set against the HBM copy bandwidth
        g_bytes = wl.Lq * (wl.window + wl.topk) * wl.d * 2 * 2
        g_gbs = g_bytes / (kern["sparse_attn_per_layer"] / 1e3) / 1e9
        res["sparse_gather"] = {"achieved": g_gbs, "unit": "GB/s", "peak": peaks["hbm_gbs"],
                                "frac": g_gbs / peaks["hbm_gbs"], "bytes_per_layer": g_bytes,
                                "note": "gathered K+V rows per layer (L2-resident cache) against the HBM copy peak"}
    if not args.prefill_len:
        # chunked prefill: the last CHUNK queries of the same prompt appended to the cache of the
        # first L - CHUNK tokens (query i at position L - CHUNK + i), same K/V buffers
        CHUNK = 4096
        qc = q[:, -CHUNK:]
        oc = torch.empty_like(qc)
        lc = torch.empty((1, CHUNK, wl.H), dtype=torch.float32, device=dev)
        ic = torch.empty((1, CHUNK, wl.window + wl.topk), dtype=torch.int32, device=dev)
        for _ in range(warmup):
            hs2.full_attn_select(qc, k, v, scale=wl.scale, out=oc, lse=lc, idx=ic)
        c0, c1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        c0.record(s)
        for _ in range(reps):
            hs2.full_attn_select(qc, k, v, scale=wl.scale, out=oc, lse=lc, idx=ic)
        c1.record(s)
        c1.synchronize()
        cms = _max_over_ranks(c0.elapsed_time(c1), world) / reps
        off = wl.Lk - CHUNK
        cP = CHUNK * off + CHUNK * (CHUNK + 1) / 2   # (query, key) pairs of the chunk
        ctf = 6 * wl.H * wl.d * cP / (cms / 1e3) / 1e12
        res["chunk"] = {"workload": f"{CHUNK} queries appended to a {off}-token cache (H={wl.H}, d={wl.d})",
                        "tok_per_s": world * CHUNK / (cms / 1e3), "ms": cms,
                        "roofline": {"bound": "tensor", "achieved": ctf, "peak": peaks["bf16_tflops"],
                                     "unit": "TFLOP/s", "frac": ctf / peaks["bf16_tflops"],
                                     "frac_of_sustained": ctf / peaks["bf16_tflops_sustained"],
                                     "flops": "executed 6*H*d*(pairs of the chunk's causal rows)"}}
    if wl.bridge_T and not args.prefill_len:
        # KV Bridging: one batched GEMM H[T x hidden] . [W_k^l | W_v^l ...]
        hb = _bf16(g.bridge_h, dev)
        wb = _bf16(g.bridge_w, dev)
        kvb = torch.empty((wl.bridge_layers, 2, wl.bridge_T, wl.d), dtype=torch.bfloat16, device=dev)
        for _ in range(3):
            hs2.bridge_kv_proj(hb, wb, out=kvb)
        b0, b1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        b0.record(s)
        for _ in range(20):
            hs2.bridge_kv_proj(hb, wb, out=kvb)
        b1.record(s)
        b1.synchronize()
        bms = b0.elapsed_time(b1) / 20
        bflops = 2.0 * wl.bridge_T * wl.bridge_hidden * 2 * wl.bridge_layers * wl.d
        btf = bflops / (bms / 1e3) / 1e12
        res["bridge"] = {"workload": f"H[{wl.bridge_T}x{wl.bridge_hidden}] x W[{wl.bridge_layers},2,{wl.bridge_hidden},{wl.d}]",
                         "ms": bms, "roofline": {"bound": "tensor", "achieved": btf, "peak": peaks["bf16_tflops"],
                                                 "unit": "TFLOP/s", "frac": btf / peaks["bf16_tflops"],
                                                 "flops": "2*T*hidden*(2*n_layers*d)"}}
    return res


if __name__ == "__main__":
    sys.exit(main())
