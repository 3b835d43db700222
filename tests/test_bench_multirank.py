"""The benchmark's multi-rank host logic on CPU: two gloo ranks (world size 2).

On GPUs `bench.py --gpus N` runs one process per GPU (torchrun, NCCL). Decode batches are
independent, so the ranks are replicas with no data-path collective: each times its own seeded
batch, the job's time is the slowest rank's, and the reported value is the whole job's steps/s.
These tests run that logic -- rank setup from the torchrun environment, barrier, max and sum over
ranks, the throughput formula, per-rank seeding, and the reference arm's rank-0-only rule -- in two
CPU processes.
"""
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

_CHILD = r"""
import os, sys, json
sys.path.insert(0, os.environ["REPO_ROOT"])
import bench, synth
world, rank, local = bench._dist_init()
assert world == 2 and local == rank
bench._barrier(world)
# each rank measured its own time; the job time is the slowest
ms = [40.0, 55.0][rank]
ms_max = bench._max_over_ranks(ms, world)
launches = bench._sum_over_ranks([7.0, 9.0][rank], world)
value = bench._throughput(world, 100, ms_max)
# weak scaling: each rank draws its own batch (seed + rank)
g = synth.SyntheticInputs(synth.small("decode_32k", B=1, Lk=256), seed=rank)
print(json.dumps({"rank": rank, "ms_max": ms_max, "launches": launches, "value": value,
                  "q0": float(g.q.reshape(-1)[0])}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run_ranks(code, world=2, extra_env=None, timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, REPO_ROOT=ROOT, MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), WORLD_SIZE=str(world),
                   RANK=str(r), LOCAL_RANK=str(r), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        try:
            o, e = p.communicate(timeout=timeout)
        except subprocess.TimeoutExpired:
            for q in procs:
                q.kill()
            raise
        assert p.returncode == 0, e[-2000:]
        outs.append(o)
    return outs


def test_two_gloo_ranks_max_time_and_whole_job_throughput():
    import json
    outs = [json.loads(o.strip().splitlines()[-1]) for o in _run_ranks(_CHILD)]
    for d in outs:
        assert d["ms_max"] == 55.0                      # the slowest rank's time
        assert d["launches"] == 16.0                    # summed launch counts
        assert abs(d["value"] - 2 * 100 / 0.055) < 1e-6  # whole job: 2 ranks x 100 steps / slowest time
    assert outs[0]["q0"] != outs[1]["q0"]               # each rank has its own batch


def test_reference_arm_runs_on_rank_zero_only():
    # a non-zero rank returns at once without touching the oracle
    code = r"""
import os, sys
sys.path.insert(0, os.environ["REPO_ROOT"])
import bench
sys.exit(bench.main())
"""
    env = dict(os.environ, REPO_ROOT=ROOT, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1", CUDA_VISIBLE_DEVICES="")
    r = subprocess.run([sys.executable, "-c", code, "--impl", "reference", "--gpus", "2", "--steps", "1",
                        "--warmup", "0"], env=env, capture_output=True, text=True, timeout=120)
    assert r.returncode == 0, r.stderr[-2000:]
    assert r.stdout.strip() == ""
