"""Seeded synthetic inputs for the retention operator.

This module holds only random-number draws and casts: no retention arithmetic.
Tests, the bench and the smoke check use it to feed the CUDA library and the
fp64 oracle the same host arrays, so parity measures kernel error only.

Recipe (all draws on the CPU torch generator, in this order):
  q, k, v  ~ N(0, 1) / sqrt(dk), then cast to the config dtype
  x        ~ N(0, 1) and g = logsigmoid(x) / 16 for the gated form (the gate
             transform of the gated-RetNet module, upstream of the operator)
  S_0      ~ N(0, 0.01^2) (decode state, fp32)
  dO       ~ N(0, 1) / sqrt(dv) (output gradient of the backward, own generator)
  epilogue inputs (own generators): a retention output o [B, H, N, dv] ~ N(0, 1) times a
             per-row scale e^z, z ~ N(0, 1) (rows of very different size, as the decays
             make them), and a gate projection [B, N, H, dv] ~ N(0, 1)
Per-head decays are the multi-scale schedules gamma_h = 1 - 2^(-5-h) and
gamma_h = 1 - 2^(-5-h/3), h = 0..H-1, rounded to fp32.
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class RetConfig:
    name: str
    B: int
    H: int
    N: int
    dk: int
    dv: int
    chunk: int
    dtype: torch.dtype
    gamma_schedule: str  # "h" -> 1-2^(-5-h); "h/3" -> 1-2^(-5-h/3); "gated" -> per-token g
    seed: int = 0

    @property
    def tokens(self) -> int:
        return self.B * self.N


# The five workloads: a tiny fp32 check, two RetNet-layer-shaped chunkwise
# forwards (1.3B- and 6.7B-shaped heads), the decode step and the gated form.
CONFIGS = {
    "tiny": RetConfig("tiny", 1, 2, 128, 32, 32, 32, torch.float32, "h"),
    "retnet_1p3b": RetConfig("retnet_1p3b", 4, 8, 2048, 256, 512, 64, torch.bfloat16, "h"),
    "retnet_6p7b_long": RetConfig("retnet_6p7b_long", 1, 16, 8192, 256, 512, 128, torch.bfloat16, "h/3"),
    "decode": RetConfig("decode", 64, 16, 1, 256, 512, 1, torch.bfloat16, "h/3"),
    "gated": RetConfig("gated", 2, 8, 16384, 128, 128, 64, torch.bfloat16, "gated"),
    "gated_decode": RetConfig("gated_decode", 64, 16, 1, 256, 512, 1, torch.bfloat16, "gated"),
}
DECODE_STEPS = 1024


def gammas(H: int, schedule: str = "h") -> torch.Tensor:
    """Per-head decay gamma_h (fp32, shape [H])."""
    if schedule == "h":
        vals = [1.0 - 2.0 ** (-5 - h) for h in range(H)]
    elif schedule == "h/3":
        vals = [1.0 - 2.0 ** (-5 - h / 3.0) for h in range(H)]
    else:
        raise ValueError(f"unknown gamma schedule {schedule!r}")
    return torch.tensor(vals, dtype=torch.float32)


def _gen(seed: int) -> torch.Generator:
    g = torch.Generator(device="cpu")
    g.manual_seed(int(seed))
    return g


def qkv(B: int, H: int, N: int, dk: int, dv: int, dtype=torch.bfloat16, seed: int = 0,
        gen: torch.Generator | None = None):
    """q, k [B, H, N, dk] and v [B, H, N, dv], N(0,1)/sqrt(dk), cast to dtype (CPU)."""
    g = gen if gen is not None else _gen(seed)
    s = 1.0 / math.sqrt(dk)
    q = (torch.randn(B, H, N, dk, generator=g) * s).to(dtype)
    k = (torch.randn(B, H, N, dk, generator=g) * s).to(dtype)
    v = (torch.randn(B, H, N, dv, generator=g) * s).to(dtype)
    return q, k, v


def gate(B: int, H: int, N: int, gen: torch.Generator) -> torch.Tensor:
    """Per-token log-decay g = logsigmoid(x)/16, x ~ N(0,1); fp32 [B, H, N], all < 0."""
    x = torch.randn(B, H, N, generator=gen)
    return torch.nn.functional.logsigmoid(x) / 16.0


def config_inputs(cfg: RetConfig, seed: int | None = None, N: int | None = None, B: int | None = None):
    """Inputs for one config: dict with q, k, v and gamma (or g). Sizes may be overridden."""
    seed = cfg.seed if seed is None else seed
    N = cfg.N if N is None else N
    B = cfg.B if B is None else B
    gen = _gen(seed)
    q, k, v = qkv(B, cfg.H, N, cfg.dk, cfg.dv, cfg.dtype, gen=gen)
    out = {"q": q, "k": k, "v": v}
    if cfg.gamma_schedule == "gated":
        out["g"] = gate(B, cfg.H, N, gen)
    else:
        out["gamma"] = gammas(cfg.H, cfg.gamma_schedule)
    return out


def output_grad(B: int, H: int, N: int, dv: int, dtype=torch.bfloat16, seed: int = 0) -> torch.Tensor:
    """Output gradient dO [B, H, N, dv] ~ N(0, 1) / sqrt(dv) (seed + 104729), cast to dtype."""
    g = _gen(seed + 104729)
    return (torch.randn(B, H, N, dv, generator=g) / math.sqrt(dv)).to(dtype)


def retention_output(B: int, H: int, N: int, dv: int, dtype=torch.bfloat16, seed: int = 0) -> torch.Tensor:
    """Stand-in retention output o [B, H, N, dv]: N(0, 1) times e^z per row, z ~ N(0, 1) (seed + 7211)."""
    g = _gen(seed + 7211)
    x = torch.randn(B, H, N, dv, generator=g)
    return (x * torch.exp(torch.randn(B, H, N, 1, generator=g))).to(dtype)


def gate_projection(B: int, H: int, N: int, dv: int, dtype=torch.bfloat16, seed: int = 0) -> torch.Tensor:
    """Gate projection output [B, N, H, dv] ~ N(0, 1) (seed + 9049), token-major."""
    g = _gen(seed + 9049)
    return torch.randn(B, N, H, dv, generator=g).to(dtype)


def decode_state(B: int, H: int, dk: int, dv: int, seed: int = 0) -> torch.Tensor:
    """Initial decode state S_0 ~ N(0, 0.01^2), fp32 [B, H, dk, dv]."""
    g = _gen(seed + 7919)
    return torch.randn(B, H, dk, dv, generator=g) * 0.01


def decode_gate(B: int, H: int, step: int, seed: int = 0) -> torch.Tensor:
    """Log-decay g [B, H] of gated decode step `step`: logsigmoid(x)/16, x ~ N(0,1) (seed + 50021 + step)."""
    g = _gen(seed + 50021 + step)
    return torch.nn.functional.logsigmoid(torch.randn(B, H, generator=g)) / 16.0


def decode_step_inputs(B: int, H: int, dk: int, dv: int, step: int, seed: int = 0,
                       dtype=torch.bfloat16):
    """Single-token q, k [B, H, dk] and v [B, H, dv] for decode step `step` (seed + step)."""
    q, k, v = qkv(B, H, 1, dk, dv, dtype, seed=seed + 1 + step)
    return q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous()
