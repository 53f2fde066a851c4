#!/usr/bin/env python
"""Throughput benchmark of the B200 retention library.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME] [--also A,B] [--impl ours|reference]

With no --workload the line's top-level figures are retnet_1p3b's and the line
carries a "workloads" object with one sub-record each for decode,
retnet_6p7b_long and gated, measured the same way (own timed region, roofline,
e2e, clocks and CPU baseline). One step is one call of the hot path on one
batch of seeded synthetic input already resident in HBM:
  retnet_1p3b       (default) ret_chunkwise, B=4 H=8 N=2048 dk=256 dv=512 chunk 64, bf16
  retnet_6p7b_long  ret_chunkwise, B=1 H=16 N=8192 dk=256 dv=512 chunk 128, bf16
  gated             gated_ret_chunkwise, B=2 H=8 N=16384 dk=dv=128 chunk 64, bf16
  decode            ret_recurrent_step, B=64 H=16 dk=256 dv=512, fp32 state
  gated_decode      gated_ret_recurrent_step, same shapes, a fresh log-decay g [B, H] per step
  seqpar_6p7b       the retnet_6p7b_long sequence split across the ranks (strong scaling):
                    segment end states, one all-gather, start states, ret_chunkwise per segment
  backward_1p3b     ret_chunkwise_backward on the retnet_1p3b shapes: dq, dk, dv and dgamma
                    from q, k, v, gamma and an output gradient dO
  backward_gated    gated_ret_chunkwise_backward on the gated workload's shapes: dq, dk, dv and
                    dg from q, k, v, g and dO
  msr_norm_1p3b     ret_msr_norm_gate on the retnet_1p3b output: per-head RMSNorm and swish gate
  retention_msr_1p3b  ret_chunkwise then ret_msr_norm_gate on its output (retnet_1p3b shapes)
For N > 1 (torchrun, one rank per GPU) every rank runs its own batch of the
same shape (batch sharding, no collective on the data path): weak scaling.
Rank 0 prints one JSON line. `--impl reference` times the fp64 CPU oracle on a
bounded sample of the same workload instead (rank 0 only).
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
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

FALLBACK_HBM_GBS = 6650.0
FALLBACK_BF16_TFLOPS = 1590.0
L2_BYTES = 126 * 1024 * 1024
NORM_EPS = 1e-5  # the norm epsilon the pages give as the module default
GATED_BWD_SAMPLE_TOKENS = 2048  # tokens per head in the gated backward's CPU sample


# ----------------------------------------------------------------------------- workload arithmetic

def workload(name: str):
    """Shapes plus the algorithmic work of one step (one call)."""
    from linear_attention_ret_b200 import inputs as I
    if name == "seqpar_6p7b":
        # the 6.7B-shaped sequence split across the ranks (strong scaling): per step the
        # whole sequence once, each rank its segment; work counted as for ret_chunkwise
        spec = workload("retnet_6p7b_long")
        spec.update(kind="seqpar", metric="retention tokens/s (sequence-parallel chunkwise fwd)")
        return spec
    if name in ("backward_1p3b", "backward_gated"):
        gated = name == "backward_gated"
        cfg = I.CONFIGS["gated" if gated else "retnet_1p3b"]
        B, H, N, dk, dv, C = cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk
        elt = 2
        # reads q, k, v, dO; writes dq, dk, dv (dgamma is H floats; gated: g read, dg written, fp32)
        gb = 4 * B * H * N if gated else 0
        io = B * H * N * (4 * dk + 3 * dv) * elt + 2 * gb
        # three contractions of the forward's shape: dQ (scores dO.v), dK (dO.v), dV (q.k)
        flops = 3 * B * H * N * (2 * C * (dk + dv) + 4 * dk * dv)
        return dict(cfg=cfg, kind="backward", gated=gated, units=B * N, unit="tokens/s",
                    metric="retention tokens/s (gated chunkwise backward)" if gated
                    else "retention tokens/s (chunkwise backward)", tokens=B * N, bytes=io, flops=flops,
                    h2d=B * H * N * (2 * dk + 2 * dv) * elt + gb,
                    d2h=B * H * N * (2 * dk + dv) * elt + (gb if gated else H * 4))
    if name in ("msr_norm_1p3b", "retention_msr_1p3b"):
        cfg = I.CONFIGS["retnet_1p3b"]
        B, H, N, dk, dv, C = cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk
        elt = 2
        gy = 2 * B * H * N * dv * elt  # gate read, y written
        if name == "msr_norm_1p3b":
            return dict(cfg=cfg, kind="norm", units=B * N, unit="tokens/s",
                        metric="tokens/s (multi-scale retention output epilogue)", tokens=B * N,
                        bytes=B * H * N * dv * elt + gy, flops=0,
                        h2d=2 * B * H * N * dv * elt, d2h=B * H * N * dv * elt)
        # o stays an intermediate: the algorithmic bytes are q, k, v and the gate in, y out
        return dict(cfg=cfg, kind="ret_norm", units=B * N, unit="tokens/s",
                    metric="retention tokens/s (chunkwise fwd + output epilogue)", tokens=B * N,
                    bytes=B * H * N * 2 * dk * elt + B * H * N * dv * elt + gy,
                    flops=B * H * N * (2 * C * (dk + dv) + 4 * dk * dv),
                    h2d=B * H * N * (2 * dk + 2 * dv) * elt, d2h=B * H * N * dv * elt)
    cfg = I.CONFIGS[name]
    B, H, N, dk, dv, C = cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk
    if name in ("decode", "gated_decode"):
        gated = name == "gated_decode"
        state = B * H * dk * dv * 4
        io = B * H * (2 * dk + 2 * dv) * 2 + (B * H * 4 if gated else 0)  # + the step's g [B, H] fp32
        return dict(cfg=cfg, kind="decode", gated=gated, units=1, unit="steps/s",
                    metric="gated decode steps/s" if gated else "decode steps/s",
                    tokens=B, bytes=2 * state + io, flops=4 * B * H * dk * dv,
                    h2d=B * H * (2 * dk + dv) * 2 + (B * H * 4 if gated else 0), d2h=B * H * dv * 2)
    elt = 2
    qkvo = B * H * N * (2 * dk + 2 * dv) * elt
    gbytes = B * H * N * 4 if cfg.gamma_schedule == "gated" else 0
    flops = B * H * N * (2 * C * (dk + dv) + 4 * dk * dv)
    return dict(cfg=cfg, kind="gated" if gbytes else "chunkwise", units=B * N, unit="tokens/s",
                metric="retention tokens/s (chunkwise fwd)", tokens=B * N, bytes=qkvo + gbytes, flops=flops,
                h2d=B * H * N * (2 * dk + dv) * elt + gbytes, d2h=B * H * N * dv * elt)


def measured_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            p = json.load(f)
        return float(p["hbm_gbs"]), float(p["bf16_tflops"]), float(p.get("bf16_tflops_sustained", p["bf16_tflops"])), "measured"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, FALLBACK_BF16_TFLOPS, 1400.0, "fallback"


# The sources each workload's measured kernels are compiled and launched from; a
# traffic figure counts only while these files still hash to the value it was taken at.
KERNEL_SOURCES = {
    "chunk": ("common.cuh", "tc_chunk.cuh", "tc_wide.cuh", "tc_state.cuh"),
    "decode": ("common.cuh", "decode.cuh"),
    "norm": ("common.cuh", "norm.cuh"),
    "backward": ("common.cuh", "tc_chunk.cuh", "tc_wide.cuh", "tc_state.cuh", "backward.cuh", "ret_api.cu"),
}
WORKLOAD_KERNELS = {"retnet_1p3b": "chunk", "retnet_6p7b_long": "chunk", "gated": "chunk", "seqpar_6p7b": "chunk",
                    "decode": "decode", "gated_decode": "decode", "backward_1p3b": "backward", "backward_gated": "backward",
                    "msr_norm_1p3b": "norm", "retention_msr_1p3b": "chunk"}


def kernel_source_sha(name: str) -> str:
    h = hashlib.sha256()
    csrc = os.path.join(ROOT, "linear_attention_ret_b200", "csrc")
    for fn in KERNEL_SOURCES[WORKLOAD_KERNELS[name]]:
        with open(os.path.join(csrc, fn), "rb") as f:
            h.update(fn.encode() + f.read())
    return h.hexdigest()[:16]


def ncu_traffic(name: str):
    """DRAM bytes per launch of the dominant kernel from the committed ncu summary,
    or None when no capture matches the current kernel sources."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            rec = json.load(f).get(name)
    except (OSError, ValueError):
        return None
    if not rec or rec.get("source_sha") != kernel_source_sha(name):
        return None
    return rec.get("traffic_bytes_per_launch")


# ----------------------------------------------------------------------------- distributed plumbing

def dist_env():
    return int(os.environ.get("RANK", 0)), int(os.environ.get("WORLD_SIZE", 1)), int(os.environ.get("LOCAL_RANK", 0))


def dist_init(world: int, backend: str):
    import datetime
    import torch.distributed as dist
    if world > 1 and not dist.is_initialized():
        os.environ.setdefault("MASTER_ADDR", "127.0.0.1")
        dist.init_process_group(backend, timeout=datetime.timedelta(seconds=120))
    return dist


def max_over_ranks(x: float, world: int, device=None) -> float:
    if world <= 1:
        return float(x)
    import torch
    import torch.distributed as dist
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(world: int, device=None):
    if world > 1:
        import torch.distributed as dist
        if device is not None and device.type == "cuda":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def rank_seed(rank: int) -> int:
    """Each rank draws its own batch (batch sharding across GPUs)."""
    return 1000 * rank


# ----------------------------------------------------------------------------- clocks

class ClockSampler:
    """nvidia-smi clock / throttle samples while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_id: str | None):
        self.gpu_id = gpu_id
        self.proc = None
        self.path = None

    def start(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        cmd = ["nvidia-smi", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits", "-lms", "100"]
        if self.gpu_id:
            cmd += ["-i", self.gpu_id]
        try:
            self.proc = subprocess.Popen(cmd, stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except OSError:
            self.proc = None
        time.sleep(0.3)

    def stop(self):
        if self.proc is None:
            return None
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        rows = []
        with open(self.path) as f:
            for line in f:
                parts = [p.strip() for p in line.split(",")]
                if len(parts) == 8:
                    rows.append(parts)
        os.unlink(self.path)
        if not rows:
            return None
        sm = [float(r[0]) for r in rows if r[0].replace(".", "").isdigit()]
        mx = max(float(r[1]) for r in rows if r[1].replace(".", "").isdigit())
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i in range(4) if r[4 + i].lower() == "active"})
        loaded = [s for s in sm if s > 0.5 * mx] or sm
        return {"sm_mhz": statistics.median(loaded), "sm_max_mhz": mx, "reasons": reasons,
                "samples": len(rows), "power_w_max": max(float(r[2]) for r in rows
                                                          if r[2].replace(".", "").isdigit())}


def gpu_uuid(dev_index: int):
    import torch
    try:
        return "GPU-" + str(torch.cuda.get_device_properties(dev_index).uuid)
    except Exception:
        return None


# ----------------------------------------------------------------------------- our arm

def make_step(spec, dev, seed):
    """Device-resident inputs and a closure that runs one step."""
    import torch
    from linear_attention_ret_b200 import inputs as I
    from linear_attention_ret_b200 import ret
    cfg = spec["cfg"]
    if spec["kind"] == "decode":
        gated = spec["gated"]
        gam = None if gated else I.gammas(cfg.H, cfg.gamma_schedule).to(dev)
        S = I.decode_state(cfg.B, cfg.H, cfg.dk, cfg.dv, seed=seed).to(dev)
        steps = [tuple(t.to(dev) for t in I.decode_step_inputs(cfg.B, cfg.H, cfg.dk, cfg.dv, s, seed=seed))
                 + ((I.decode_gate(cfg.B, cfg.H, s, seed=seed).to(dev),) if gated else ())
                 for s in range(8)]
        o = torch.empty(cfg.B, cfg.H, cfg.dv, dtype=cfg.dtype, device=dev)
        counter = [0]

        def step():
            x = steps[counter[0] % len(steps)]
            counter[0] += 1
            if gated:
                ret.gated_ret_recurrent_step(x[0], x[1], x[2], x[3], S, o=o)
            else:
                ret.ret_recurrent_step(x[0], x[1], x[2], gam, S, o=o)
        return step, {"q": steps[0][0], "k": steps[0][1], "v": steps[0][2]}, o, 1

    if spec["kind"] == "seqpar":
        from linear_attention_ret_b200 import seqpar
        rank, world, _ = dist_env()
        x = {key: val.to(dev) for key, val in seqpar_segment(cfg, rank, world).items()}

        def step():
            seqpar.sequence_parallel_chunkwise(x["q"], x["k"], x["v"], x["gamma"], cfg.chunk)
        return step, x, None, launches_per_call(spec)
    if spec["kind"] == "norm":
        x = {"o": I.retention_output(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed).to(dev),
             "gate": I.gate_projection(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed).to(dev)}
        y = torch.empty_like(x["gate"])

        def step():
            ret.msr_norm_gate(x["o"], x["gate"], NORM_EPS, y=y)
        return step, x, y, launches_per_call(spec)
    x = {key: val.to(dev) for key, val in I.config_inputs(cfg, seed=seed).items()}
    if spec["kind"] == "ret_norm":
        x["gate"] = I.gate_projection(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed).to(dev)
        o = torch.empty(cfg.B, cfg.H, cfg.N, cfg.dv, dtype=cfg.dtype, device=dev)
        y = torch.empty_like(x["gate"])

        def step():
            ret.ret_chunkwise(x["q"], x["k"], x["v"], x["gamma"], cfg.chunk, o=o)
            ret.msr_norm_gate(o, x["gate"], NORM_EPS, y=y)
        return step, x, y, launches_per_call(spec)
    if spec["kind"] == "backward":
        x["do"] = I.output_grad(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed).to(dev)

        gated = spec["gated"]

        def step():
            ret.chunkwise_backward(x["q"], x["k"], x["v"], x["g"] if gated else x["gamma"], x["do"], cfg.chunk,
                                   gated=gated)
        return step, x, None, launches_per_call(spec)
    o = torch.empty(cfg.B, cfg.H, cfg.N, cfg.dv, dtype=cfg.dtype, device=dev)
    if spec["kind"] == "gated":
        def step():
            ret.gated_ret_chunkwise(x["q"], x["k"], x["v"], x["g"], cfg.chunk, o=o)
    else:
        def step():
            ret.ret_chunkwise(x["q"], x["k"], x["v"], x["gamma"], cfg.chunk, o=o)
    return step, x, o, launches_per_call(spec)


def seqpar_segment(cfg, rank, world):
    """Rank `rank`'s consecutive slice of one seeded sequence (the same seed on every rank)."""
    from linear_attention_ret_b200 import inputs as I
    x = I.config_inputs(cfg, seed=0)
    t0, t1 = cfg.N * rank // world, cfg.N * (rank + 1) // world
    return {k: (t[:, :, t0:t1].contiguous() if t.dim() == 4 else t) for k, t in x.items()}


def launches_per_call(spec) -> int:
    """Kernels one call of the step launches (the library's own kernels only)."""
    from linear_attention_ret_b200 import ret
    cfg = spec["cfg"]
    if spec["kind"] == "decode":
        return 1
    if spec["kind"] == "norm":
        return 1
    if spec["kind"] == "ret_norm":
        return ret.chunkwise_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, cfg.dtype) + 1
    if spec["kind"] == "backward":
        return ret.chunkwise_backward_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, cfg.dtype,
                                               gated=spec["gated"])
    if spec["kind"] == "seqpar":
        _, world, _ = dist_env()
        n = cfg.N // world + (1 if cfg.N % world else 0)
        return (ret.chunkwise_state_launches(cfg.B, cfg.H, n, cfg.dk, cfg.dv, cfg.chunk, cfg.dtype) + 1
                + ret.chunkwise_launches(cfg.B, cfg.H, n, cfg.dk, cfg.dv, cfg.chunk, cfg.dtype))
    return ret.chunkwise_launches(cfg.B, cfg.H, cfg.N, cfg.dk, cfg.dv, cfg.chunk, cfg.dtype)


DTYPE_NAMES = {"torch.bfloat16": "bf16", "torch.float32": "f32"}

# Workloads measured beside the headline one in the default line (each as a sub-record
# with its own roofline, e2e, clocks and CPU baseline): the recurrent decode step, the
# 6.7B-shaped long sequence and the gated form.
DEFAULT_ALSO = ("decode", "retnet_6p7b_long", "gated")


def dtype_name(cfg) -> str:
    """The arithmetic type of the inputs and outputs (accumulation and state are fp32)."""
    return DTYPE_NAMES[str(cfg.dtype)]


def measure(args, name, spec, dev, stream, world, steps, cpu_budget):
    """One workload on this rank: warm-up, clock-sampled burn-in, K timed steps (CUDA
    events on the launch stream, max over ranks), then the end-to-end figure. Returns
    the record rank 0 prints (every rank takes the same collective steps)."""
    import torch
    from linear_attention_ret_b200 import ret
    rank = dist_env()[0]
    step, x, o, launches = make_step(spec, dev, rank_seed(rank))
    # nvidia-smi samples every 100 ms while a timed region lasts milliseconds, so sampling
    # starts before the warm-up and an untimed burn-in keeps the same load for about a
    # second; the samples then describe the clocks the timed region runs at.
    clocks = ClockSampler(gpu_uuid(dev.index))
    clocks.start()
    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    err = ret.last_device_error()
    if err != 0:
        raise SystemExit(f"{name}: device error word set after warm-up: {err}")
    t_burn = time.perf_counter()
    while time.perf_counter() - t_burn < args.burn_in:
        for _ in range(10):
            step()
        torch.cuda.synchronize()

    # timed region: K steps, barrier + synchronize on both sides, events per step on the launch stream
    ev = [torch.cuda.Event(enable_timing=True) for _ in range(steps + 1)]
    barrier(world, dev)
    torch.cuda.synchronize()
    ev[0].record(stream)
    for i in range(steps):
        step()
        ev[i + 1].record(stream)
    torch.cuda.synchronize()
    barrier(world, dev)
    clk = clocks.stop()
    per_step = [ev[i].elapsed_time(ev[i + 1]) for i in range(steps)]
    total_ms = ev[0].elapsed_time(ev[-1])
    max_ms = max_over_ranks(total_ms, world, dev)
    if ret.last_device_error() != 0:
        raise SystemExit(f"{name}: device error word set in the timed region")
    del x, o
    e2e = run_e2e(args, spec, dev, stream, world)

    ms_per_step = max_ms / steps
    strong = spec["kind"] == "seqpar"  # one sequence split across the ranks
    if spec["kind"] == "decode":
        value = world * 1e3 / ms_per_step
    else:
        value = spec["units"] * (1 if strong else world) / (ms_per_step / 1e3)
    hbm, tf_burst, tf_sust, peak_src = measured_peaks()
    # the step's mean duration on this rank: a step is one launch of the dominant kernel
    # (plus, for split sequences, two short launches whose share the ncu launch list records)
    kern_ms = statistics.mean(per_step)
    achieved = spec["bytes"] / (kern_ms / 1e3) / 1e9
    roofline = {"bound": "hbm", "achieved": round(achieved, 1), "peak": hbm, "unit": "GB/s",
                "frac": round(achieved / hbm, 4), "traffic": ncu_traffic(name),
                "traffic_note": "dram__bytes_read.sum + dram__bytes_write.sum per step from one ncu capture "
                                "(null unless the kernel sources are unchanged since); the write count misses "
                                "output rows still in L2 when the kernel ends",
                "algorithmic_bytes": spec["bytes"],
                "peak_source": "measured (MEASURED_PEAKS.json hbm_gbs, copy)" if peak_src == "measured"
                else "fallback 6.65 TB/s",
                "kernel_ms": round(kern_ms, 5),
                "scope": ("the whole step: " + str(launches) + " launches (the dQ and dK passes, dV, the decay "
                          "gradient)") if spec["kind"] == "backward"
                else "the step's launches",
                "tensor_tflops": round(spec["flops"] / (kern_ms / 1e3) / 1e12, 2),
                "tensor_frac_of_bf16_burst": round(spec["flops"] / (kern_ms / 1e3) / 1e12 / tf_burst, 4),
                "tensor_frac_of_bf16_sustained": round(spec["flops"] / (kern_ms / 1e3) / 1e12 / tf_sust, 4)}
    cfg = spec["cfg"]
    rec = {
        "metric": spec["metric"], "value": round(value, 2), "unit": spec["unit"], "n_gpus": world,
        "steps": steps, "warmup": args.warmup, "ms_per_step": round(ms_per_step, 5),
        "ms_per_step_median": round(statistics.median(per_step), 5),  # this rank's CUDA-event times per step
        "higher_is_better": True, "scaling": "strong" if strong else "weak", "vs_baseline": None,
        "dtype": dtype_name(cfg),
        "data": "synthetic (seeded N(0,1)/sqrt(dk); " + ("one sequence split across ranks)" if strong
                                                        else "per-rank seeds)"),
        "config": {"workload": name, "B": cfg.B, "H": cfg.H, "N": cfg.N, "dk": cfg.dk, "dv": cfg.dv,
                   "chunk": cfg.chunk, "state": "fp32", "accumulate": "fp32",
                   "l2": f"working set {spec['bytes'] / 1e6:.0f} MB per step > 126 MB L2 (no flush)",
                   "parallelism": (f"sequence-parallel x{world} (one all-gather of segment states)" if strong
                                   else f"batch-sharded x{world}") if world > 1 else "single GPU"},
        "roofline": roofline,
        "clocks": dict(clk, window="warm-up, ~1 s untimed burn-in and the timed region") if clk else None,
        "e2e": e2e,
        "gpu_launches": steps * launches,
        "launches_per_step": launches,
    }
    if spec["kind"] == "decode":
        rec["ms_per_1024_steps"] = round(1024 * ms_per_step, 3)  # a 1024-token generation
        rec["tokens_per_s"] = round(world * cfg.B * 1e3 / ms_per_step, 1)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        rec["cpu_baseline"] = cpu_baseline(spec, budget_s=cpu_budget, single_budget_s=max(1.0, cpu_budget / 3))
    return rec


def run_ours(args, spec):
    import torch
    rank, world, local = dist_env()
    if not torch.cuda.is_available():
        raise SystemExit("bench.py needs a CUDA device (the library has no CPU path)")
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    dist_init(world, "nccl")
    from linear_attention_ret_b200 import ret
    ret.load()
    stream = torch.cuda.current_stream(dev)

    line = measure(args, args.workload, spec, dev, stream, world, args.steps, args.cpu_seconds)
    also = [w for w in args.also if w != args.workload]
    if also:
        # the other headline workloads, each measured the same way, as sub-records of this line
        line["workloads"] = {}
        for name in also:
            sub = measure(args, name, workload(name), dev, stream, world, args.steps, args.cpu_seconds / 2)
            line["workloads"][name] = sub
            torch.cuda.empty_cache()
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()


def run_e2e(args, spec, dev, stream, world):
    """Same metric through the public API with host buffers: every step copies its
    inputs host->device from pinned memory and the result device->host."""
    import torch
    from linear_attention_ret_b200 import inputs as I
    from linear_attention_ret_b200 import ret
    cfg = spec["cfg"]
    rank = dist_env()[0]
    if spec["kind"] == "decode":
        gated = spec["gated"]
        host = [t.pin_memory() for t in I.decode_step_inputs(cfg.B, cfg.H, cfg.dk, cfg.dv, 0, seed=rank_seed(rank))]
        if gated:
            host.append(I.decode_gate(cfg.B, cfg.H, 0, seed=rank_seed(rank)).pin_memory())
        dev_in = [torch.empty_like(t, device=dev) for t in host]
        gam = None if gated else I.gammas(cfg.H, cfg.gamma_schedule).to(dev)
        S = I.decode_state(cfg.B, cfg.H, cfg.dk, cfg.dv).to(dev)
        o = torch.empty(cfg.B, cfg.H, cfg.dv, dtype=cfg.dtype, device=dev)
        o_host = torch.empty(o.shape, dtype=o.dtype).pin_memory()

        def step():
            for d, h in zip(dev_in, host):
                d.copy_(h, non_blocking=True)
            if gated:
                ret.gated_ret_recurrent_step(dev_in[0], dev_in[1], dev_in[2], dev_in[3], S, o=o)
            else:
                ret.ret_recurrent_step(dev_in[0], dev_in[1], dev_in[2], gam, S, o=o)
            o_host.copy_(o, non_blocking=True)
    elif spec["kind"] == "seqpar":
        from linear_attention_ret_b200 import seqpar
        xh = {k: t.pin_memory() for k, t in seqpar_segment(cfg, rank, world).items()}
        xd = {k: torch.empty_like(t, device=dev) for k, t in xh.items()}
        o_host = torch.empty(xh["v"].shape, dtype=cfg.dtype).pin_memory()

        def step():
            for key in xh:
                xd[key].copy_(xh[key], non_blocking=True)
            o, _ = seqpar.sequence_parallel_chunkwise(xd["q"], xd["k"], xd["v"], xd["gamma"], cfg.chunk)
            o_host.copy_(o, non_blocking=True)
    elif spec["kind"] in ("norm", "ret_norm"):
        seed = rank_seed(rank)
        xh = ({"o": I.retention_output(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed)} if spec["kind"] == "norm"
              else I.config_inputs(cfg, seed=seed))
        xh["gate"] = I.gate_projection(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed)
        xh = {k: t.pin_memory() for k, t in xh.items()}
        xd = {k: torch.empty_like(t, device=dev) for k, t in xh.items()}
        o = torch.empty(cfg.B, cfg.H, cfg.N, cfg.dv, dtype=cfg.dtype, device=dev)
        y = torch.empty_like(xd["gate"])
        y_host = torch.empty(y.shape, dtype=y.dtype).pin_memory()

        def step():
            for key in xh:
                xd[key].copy_(xh[key], non_blocking=True)
            if spec["kind"] == "norm":
                ret.msr_norm_gate(xd["o"], xd["gate"], NORM_EPS, y=y)
            else:
                ret.ret_chunkwise(xd["q"], xd["k"], xd["v"], xd["gamma"], cfg.chunk, o=o)
                ret.msr_norm_gate(o, xd["gate"], NORM_EPS, y=y)
            y_host.copy_(y, non_blocking=True)
    elif spec["kind"] == "backward":
        # the host-buffer backward: inputs in and gradients out, pipelined over groups of heads
        xh = {k: t.pin_memory() for k, t in I.config_inputs(cfg, seed=rank_seed(rank)).items()}
        xh["do"] = I.output_grad(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=rank_seed(rank)).pin_memory()
        gated = spec["gated"]
        outs_h = tuple(torch.empty(xh[n].shape, dtype=cfg.dtype).pin_memory() for n in ("q", "k", "v")) + (
            torch.empty(xh["g"].shape if gated else (cfg.H,), dtype=torch.float32).pin_memory(),)

        def step():
            ret.chunkwise_backward_host(xh["q"], xh["k"], xh["v"], xh["g"] if gated else xh["gamma"], xh["do"],
                                        cfg.chunk, gated=gated, out=outs_h, stream=stream)
    else:
        # the host-buffer entry point: the library copies the inputs in and o out itself,
        # pipelined with the forward over groups of heads; each call returns with o on the host
        xh = {k: t.pin_memory() for k, t in I.config_inputs(cfg, seed=rank_seed(rank)).items()}
        o_host = torch.empty(cfg.B, cfg.H, cfg.N, cfg.dv, dtype=cfg.dtype).pin_memory()
        gated = spec["kind"] == "gated"

        def step():
            if gated:
                ret.gated_ret_chunkwise_host(xh["q"], xh["k"], xh["v"], xh["g"], cfg.chunk, o=o_host, stream=stream)
            else:
                ret.ret_chunkwise_host(xh["q"], xh["k"], xh["v"], xh["gamma"], cfg.chunk, o=o_host, stream=stream)
    steps = max(3, min(args.steps, 20))
    for _ in range(2):
        step()
    torch.cuda.synchronize()
    t0, t1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier(world, dev)
    t0.record(stream)
    for _ in range(steps):
        step()
    t1.record(stream)
    torch.cuda.synchronize()
    ms = max_over_ranks(t0.elapsed_time(t1), world, dev) / steps
    value = (spec["units"] if spec["kind"] != "decode" else 1) * (1 if spec["kind"] == "seqpar" else world) / (ms / 1e3)
    return {"value": round(value, 2), "unit": spec["unit"], "ms_per_step": round(ms, 4),
            "h2d_bytes_per_step": spec["h2d"], "d2h_bytes_per_step": spec["d2h"]}


# ----------------------------------------------------------------------------- oracle timing

def _oracle_sample_step(spec, heads, seed=0):
    """Inputs for a bounded sample (the first `heads` (b, h) pairs) and a closure
    that runs the oracle on it once. Returns (closure, units the sample covers)."""
    import torch
    from linear_attention_ret_b200 import inputs as I
    from oracle import oracle as O
    cfg = spec["cfg"]
    if spec["kind"] == "decode":
        q, k, v = I.decode_step_inputs(cfg.B, cfg.H, cfg.dk, cfg.dv, 0, seed=seed)
        S = I.decode_state(cfg.B, cfg.H, cfg.dk, cfg.dv, seed=seed)
        b_needed = max(1, -(-heads // cfg.H))
        qs, ks, vs, Ss = (t[:b_needed] for t in (q, k, v, S))
        state = [Ss.double().numpy()]
        if spec["gated"]:
            gs = I.decode_gate(cfg.B, cfg.H, 0, seed=seed)[:b_needed]

            def run():
                _, state[0] = O.gated_recurrent_step(qs, ks, vs, gs, state[0])
            return run, b_needed * cfg.H / (cfg.B * cfg.H)
        gam = I.gammas(cfg.H, cfg.gamma_schedule)

        def run():
            _, state[0] = O.ret_recurrent_step(qs, ks, vs, gam, state[0])
        return run, b_needed * cfg.H / (cfg.B * cfg.H)  # fraction of one decode step
    if spec["kind"] == "norm":
        o = I.retention_output(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed)
        gate = I.gate_projection(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed)

        def run():
            O.msr_norm_gate(o, gate, NORM_EPS)
        return run, cfg.B * cfg.N  # the whole workload: the epilogue is linear in its size
    x = I.config_inputs(cfg, seed=seed, B=max(1, -(-heads // cfg.H)))
    if spec["kind"] == "ret_norm":
        bh_idx = torch.arange(heads) % cfg.H
        sl = {k: t.reshape(-1, *t.shape[2:])[:heads].unsqueeze(0) for k, t in x.items() if k != "gamma"}
        gate = I.gate_projection(1, heads, cfg.N, cfg.dv, cfg.dtype, seed=seed)

        def run():
            o, _ = O.ret_chunkwise(sl["q"], sl["k"], sl["v"], x["gamma"][bh_idx], cfg.chunk)
            O.msr_norm_gate(o, gate, NORM_EPS)
        return run, heads * cfg.N / cfg.H
    if spec["kind"] == "backward":
        x["do"] = I.output_grad(x["q"].shape[0], cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=seed)
    sl = {k: t.reshape(-1, *t.shape[2:])[:heads].unsqueeze(0) for k, t in x.items() if k != "gamma"}
    if spec["kind"] == "backward":
        if spec["gated"]:
            # the oracle's cost grows faster than N^2, so the sample is the first
            # GATED_BWD_SAMPLE_TOKENS tokens of each head (a full head of 16384 takes ~17 min)
            n = min(cfg.N, GATED_BWD_SAMPLE_TOKENS)
            gs = {key: (t[:, :, :n] if key == "g" else t[:, :, :n, :]) for key, t in sl.items()}

            def run():
                O.gated_backward(gs["q"], gs["k"], gs["v"], gs["g"], gs["do"])
            return run, heads * n / cfg.H
        gam = x["gamma"][torch.arange(heads) % cfg.H]

        def run():
            O.ret_backward(sl["q"], sl["k"], sl["v"], gam, sl["do"])
        return run, heads * cfg.N / cfg.H
    if spec["kind"] == "gated":
        def run():
            O.gated_chunkwise(sl["q"], sl["k"], sl["v"], sl["g"], cfg.chunk)
    else:
        bh_idx = torch.arange(heads) % cfg.H
        gam = x["gamma"][bh_idx]
        # heads of the sample become the H axis of one batch element, each with its own gamma

        def run():
            O.ret_chunkwise(sl["q"], sl["k"], sl["v"], gam, cfg.chunk)
    return run, heads * cfg.N / cfg.H  # tokens (all heads of a token count once)


def _time_oracle(run, budget_s):
    """Runs `run` at least once and until about budget_s seconds; returns (reps, seconds)."""
    t0 = time.perf_counter()
    run()
    t = time.perf_counter() - t0
    reps = 1
    while time.perf_counter() - t0 + t <= budget_s and reps < 64:
        run()
        reps += 1
    return reps, time.perf_counter() - t0


def cpu_baseline(spec, budget_s: float = 12.0, single_budget_s: float = 4.0):
    """The fp64 oracle on the host cores (OpenMP over heads) on a bounded sample, plus the
    same oracle on one thread and one head for the per-core figure."""
    from oracle import oracle as O
    threads = O.max_threads()
    cfg = spec["cfg"]
    total_heads = cfg.B * cfg.H
    heads = min(total_heads, threads)
    run, units = _oracle_sample_step(spec, heads)
    reps, el = _time_oracle(run, budget_s)
    value = units * reps / el
    what = ("decode steps" if spec["kind"] == "decode"
            else f"the first {min(cfg.N, GATED_BWD_SAMPLE_TOKENS)} of {cfg.N} tokens"
            if spec["kind"] == "backward" and spec.get("gated") else f"{cfg.N} tokens")
    covered = lambda n: (total_heads if spec["kind"] == "norm"  # the epilogue sample is the whole workload
                         else max(1, -(-n // cfg.H)) * cfg.H if spec["kind"] == "decode"  # whole batch rows
                         else n)
    heads = covered(heads)
    O.set_threads(1)
    try:
        run1, units1 = _oracle_sample_step(spec, 1)
        reps1, el1 = _time_oracle(run1, single_budget_s)
    finally:
        O.set_threads(threads)
    heads1 = covered(1)
    return {"value": round(value, 3), "unit": spec["unit"], "cores": threads, "kind": "oracle",
            "sample": f"{reps} run(s) of the fp64 oracle on {heads} of {total_heads} (b,h) heads x {what} "
                      f"({el:.1f} s wall, OpenMP over heads)",
            "single_thread": {"value": round(units1 * reps1 / el1, 3), "unit": spec["unit"], "cores": 1,
                              "sample": f"{reps1} run(s) on {heads1} of {total_heads} (b,h) heads x {what} "
                                        f"({el1:.1f} s wall, one thread)"},
            "cpu": _cpu_model()}


def _cpu_model():
    try:
        with open("/proc/cpuinfo") as f:
            for line in f:
                if line.startswith("model name"):
                    return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, spec):
    rank, world, _ = dist_env()
    if rank != 0:
        return  # the oracle runs on rank 0's host cores only
    from oracle import oracle as O
    threads = O.max_threads()
    cfg = spec["cfg"]
    heads = min(cfg.B * cfg.H, threads)
    run, units = _oracle_sample_step(spec, heads)
    for _ in range(args.warmup):
        run()
    t0 = time.perf_counter()
    for _ in range(args.steps):
        run()
    el = time.perf_counter() - t0
    value = units * args.steps / el
    what = ("decode steps" if spec["kind"] == "decode"
            else f"the first {min(cfg.N, GATED_BWD_SAMPLE_TOKENS)} of {cfg.N} tokens"
            if spec["kind"] == "backward" and spec.get("gated") else f"{cfg.N} tokens")
    if spec["kind"] == "norm":
        heads = cfg.B * cfg.H  # the epilogue sample is the whole workload
    sample = (f"each step: fp64 oracle on {heads} of {cfg.B * cfg.H} (b,h) heads x {what}, "
              f"OpenMP over heads")
    line = {"impl": "reference", "metric": spec["metric"], "value": round(value, 4), "unit": spec["unit"],
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
            "ms_per_step": round(el / args.steps * 1e3, 3), "higher_is_better": True, "scaling": "weak",
            "vs_baseline": None, "dtype": "f64", "data": "synthetic",
            "config": {"workload": args.workload, "B": cfg.B, "H": cfg.H, "N": cfg.N, "dk": cfg.dk,
                       "dv": cfg.dv, "chunk": cfg.chunk},
            "cpu_baseline": {"value": round(value, 4), "unit": spec["unit"], "cores": threads, "kind": "oracle",
                             "sample": sample, "cpu": _cpu_model()},
            "e2e": {"value": round(value, 4), "unit": spec["unit"], "h2d_bytes_per_step": 0,
                    "d2h_bytes_per_step": 0},
            "gpu_launches": 0}
    print(json.dumps(line), flush=True)


def main(argv=None):
    ap = argparse.ArgumentParser(description=__doc__, formatter_class=argparse.RawDescriptionHelpFormatter)
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--workload", default=None, choices=list(WORKLOAD_KERNELS),
                    help="one workload (default: retnet_1p3b, with decode, retnet_6p7b_long and gated "
                         "as sub-records of the same line)")
    ap.add_argument("--also", default=None,
                    help="comma-separated workloads measured as sub-records of the line "
                         "(default: none with --workload, else " + ",".join(DEFAULT_ALSO) + ")")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--cpu-seconds", type=float, default=12.0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--burn-in", type=float, default=1.0,
                    help="seconds of untimed steps after warm-up while clocks are sampled")
    args = ap.parse_args(argv)
    if args.warmup < 3:
        ap.error("--warmup must be >= 3")
    if args.also is None:
        args.also = [] if args.workload else list(DEFAULT_ALSO)
    else:
        args.also = [w for w in args.also.split(",") if w]
        for w in args.also:
            if w not in WORKLOAD_KERNELS:
                ap.error(f"--also: unknown workload {w!r}")
    if args.workload is None:
        args.workload = "retnet_1p3b"
    spec = workload(args.workload)
    if args.impl == "reference":
        run_reference(args, spec)
    else:
        run_ours(args, spec)


if __name__ == "__main__":
    main()
