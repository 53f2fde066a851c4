"""Multi-rank host logic of bench.py on CPU (gloo, world size 2).

The path shards by batch (every (b, h) head is independent), so ranks share no
data-path collective; what runs across ranks is the timing plumbing: process
group set-up, per-rank seeds, barrier, the max-over-ranks reduction of the
timed region, and the reference arm running on rank 0 only.
"""
import json
import os
import socket
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import os, sys, json
sys.path.insert(0, os.environ["ROOT"])
import bench
rank, world, local = bench.dist_env()
bench.dist_init(world, "gloo")
bench.barrier(world)
mx = bench.max_over_ranks(10.0 * (rank + 1), world)
seed = bench.rank_seed(rank)
print(json.dumps({"rank": rank, "max": mx, "seed": seed}), flush=True)
import torch.distributed as dist
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _launch(code, world, extra_env=None, timeout=120):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="")
        env.update(extra_env or {})
        procs.append(subprocess.Popen([sys.executable, "-c", code], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    outs = []
    for p in procs:
        out, err = p.communicate(timeout=timeout)
        assert p.returncode == 0, err
        outs.append(out)
    return outs


def test_max_over_ranks_and_seeds_gloo():
    outs = _launch(WORKER, 2)
    recs = [json.loads(o.strip().splitlines()[-1]) for o in outs]
    assert sorted(r["rank"] for r in recs) == [0, 1]
    assert all(r["max"] == 20.0 for r in recs)  # every rank sees the slowest rank's time
    assert len({r["seed"] for r in recs}) == 2   # each rank draws its own batch


REFERENCE = r"""
import os, sys
sys.path.insert(0, os.environ["ROOT"])
import bench
bench.main(["--impl", "reference", "--workload", "decode", "--steps", "1", "--warmup", "3"])
"""


def test_reference_arm_runs_on_rank0_only():
    outs = _launch(REFERENCE, 2, extra_env={"OMP_NUM_THREADS": "2"}, timeout=300)
    lines = [o for o in outs if o.strip()]
    assert len(lines) == 1
    rec = json.loads(lines[0].strip().splitlines()[-1])
    assert rec["impl"] == "reference" and rec["unit"] == "steps/s" and rec["value"] > 0
    assert rec["cpu_baseline"]["kind"] == "oracle"
    assert rec["e2e"]["h2d_bytes_per_step"] == 0


def test_workload_arithmetic():
    sys.path.insert(0, ROOT)
    import bench
    w = bench.workload("retnet_1p3b")
    assert w["bytes"] == 4 * 8 * 2048 * (2 * 256 + 2 * 512) * 2   # read Q, K, V and write O once, bf16
    assert w["flops"] == 4 * 8 * 2048 * (2 * 64 * (256 + 512) + 4 * 256 * 512)
    d = bench.workload("decode")
    assert d["bytes"] == 2 * 64 * 16 * 256 * 512 * 4 + 64 * 16 * (2 * 256 + 2 * 512) * 2
    gt = bench.workload("gated")
    assert gt["bytes"] == 2 * 8 * 16384 * (4 * 128) * 2 + 2 * 8 * 16384 * 4
