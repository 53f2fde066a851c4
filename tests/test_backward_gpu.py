"""GPU parity of the backward pass (gradients of sum(dO * O) from a zero initial
state) against the fp64 oracle's gradients by definition, which are pinned to
finite differences of the brute-force forward."""
import numpy as np
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from oracle import oracle as O
from tests.parity import TOL_BF16, TOL_F32, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

BWD_CASES = [
    # B, H, N, dk, dv, dtype
    (1, 2, 77, 32, 40, torch.float32),       # CUDA-core path, ragged
    (2, 2, 130, 64, 96, torch.float32),
    (1, 2, 200, 128, 128, torch.bfloat16),   # tensor-core path
    (1, 2, 257, 256, 512, torch.bfloat16),   # dv = 512: the dq/dk contraction in two pieces
    (2, 1, 64, 64, 128, torch.bfloat16),
    (1, 2, 130, 64, 512, torch.bfloat16),   # dv pieces copied out (value width 64 is off the tensor-core path)
    (1, 1, 70, 32, 300, torch.float32),     # fp32 pieces of 256 and a ragged 44
]


def _case(B, H, N, dk, dv, dtype, seed):
    gen = torch.Generator().manual_seed(seed)
    q, k, v = I.qkv(B, H, N, dk, dv, dtype, gen=gen)
    do = (torch.randn(B, H, N, dv, generator=gen) / np.sqrt(dv)).to(dtype)
    return q, k, v, do, gen


def _check(got, want, dtype, what, tol=None):
    tol = tol if tol is not None else (TOL_F32 if dtype == torch.float32 else TOL_BF16)
    err = rel_l2(got, want)
    assert err <= tol, f"{what}: rel-L2 {err:.3e} > {tol:.0e}"


@pytest.mark.parametrize("B,H,N,dk,dv,dtype", BWD_CASES)
def test_backward_matches_oracle(cuda_lib, B, H, N, dk, dv, dtype):
    q, k, v, do, _ = _case(B, H, N, dk, dv, dtype, seed=N + dv)
    gam = torch.tensor([0.96875, 0.999, 0.9, 0.75][:H], dtype=torch.float32)
    dq, dkk, dvv, dgam = cuda_lib.chunkwise_backward(*(t.to(DEV) for t in (q, k, v, gam, do)), 64)
    assert cuda_lib.last_device_error() == 0
    want = O.ret_backward(q, k, v, gam, do)
    _check(dq, want[0], dtype, "dq")
    _check(dkk, want[1], dtype, "dk")
    _check(dvv, want[2], dtype, "dv")
    # dgamma is a sum over the sequence of differences q.dq - k.dk: allow for the cancellation
    _check(dgam, want[3], dtype, "dgamma", tol=1e-3 if dtype == torch.float32 else 5e-2)


@pytest.mark.parametrize("B,H,N,dk,dv,dtype", BWD_CASES)
def test_gated_backward_matches_oracle(cuda_lib, B, H, N, dk, dv, dtype):
    q, k, v, do, gen = _case(B, H, N, dk, dv, dtype, seed=3 * N + dv)
    g = I.gate(B, H, N, gen) * 4.0
    dq, dkk, dvv, dg = cuda_lib.chunkwise_backward(*(t.to(DEV) for t in (q, k, v, g, do)), 64, gated=True)
    assert cuda_lib.last_device_error() == 0
    want = O.gated_backward(q, k, v, g, do)
    _check(dq, want[0], dtype, "dq")
    _check(dkk, want[1], dtype, "dk")
    _check(dvv, want[2], dtype, "dv")
    _check(dg, want[3], dtype, "dg", tol=1e-3 if dtype == torch.float32 else 5e-2)


def test_backward_gradient_of_forward_by_directional_derivative(cuda_lib):
    """Independent of the oracle's backward: for a random direction (Q', K', V') the
    directional derivative of sum(dO * O) computed from the GPU forward by central
    differences equals <dq, Q'> + <dk, K'> + <dv, V'> from the GPU backward."""
    B, H, N, dk, dv = 1, 2, 150, 32, 40
    q, k, v, do, gen = _case(B, H, N, dk, dv, torch.float32, seed=11)
    gam = torch.tensor([0.9, 0.97])
    dirs = [torch.randn(t.shape, generator=gen) for t in (q, k, v)]
    d = [t.to(DEV) for t in (q, k, v, gam, do)]
    dq, dkk, dvv, _ = cuda_lib.chunkwise_backward(*d, 64)
    eps = 1e-3

    def loss(s):
        qq, kk, vv = (t + s * e for t, e in zip((q, k, v), dirs))
        o = cuda_lib.ret_chunkwise(qq.to(DEV), kk.to(DEV), vv.to(DEV), gam.to(DEV), 64)
        return float((o.double() * do.to(DEV).double()).sum())
    fd = (loss(eps) - loss(-eps)) / (2 * eps)
    an = sum(float((g.double().cpu() * e.double()).sum()) for g, e in zip((dq, dkk, dvv), dirs))
    assert abs(fd - an) <= 1e-3 * abs(an), (fd, an)


def test_backward_full_size_sampled_heads(cuda_lib):
    """The 1.3B-shaped workload (B4 H8 N2048 dk256 dv512) as bench.py times it; the oracle
    computes head 7 of every batch element (its dgamma sums over the batch) and head 0
    of batch element 0, each by definition."""
    cfg = I.CONFIGS["retnet_1p3b"]
    x = I.config_inputs(cfg, seed=0)
    do = I.output_grad(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=0)
    dq, dkk, dvv, dgam = cuda_lib.chunkwise_backward(*(x[n].to(DEV) for n in ("q", "k", "v", "gamma")),
                                                     do.to(DEV), cfg.chunk)
    assert cuda_lib.last_device_error() == 0
    for h, bs in ((7, range(cfg.B)), (0, range(1))):
        sel = lambda t: t[list(bs), h:h + 1]
        want = O.ret_backward(sel(x["q"]), sel(x["k"]), sel(x["v"]), x["gamma"][h:h + 1], sel(do))
        for got, ref, what in zip((dq, dkk, dvv), want[:3], ("dq", "dk", "dv")):
            _check(sel(got.cpu()), ref, cfg.dtype, f"{what} head {h}")
        if h == 7:
            _check(dgam[h:h + 1], want[3], cfg.dtype, "dgamma head 7", tol=5e-2)


@pytest.mark.parametrize("gated", [False, True])
def test_backward_without_decay_gradient(cuda_lib, gated):
    """ddecay=False: the same dq, dk, dv (the tensor-core path with dv in pieces)."""
    q, k, v, do, gen = _case(1, 2, 190, 256, 512, torch.bfloat16, seed=21)
    decay = I.gate(1, 2, 190, gen) * 4.0 if gated else torch.tensor([0.97, 0.9])
    d = [t.to(DEV) for t in (q, k, v, decay, do)]
    full = cuda_lib.chunkwise_backward(*d, 64, gated=gated)
    part = cuda_lib.chunkwise_backward(*d, 64, gated=gated, ddecay=False)
    assert part[3] is None
    for a, b in zip(full[:3], part[:3]):
        assert torch.equal(a, b)
