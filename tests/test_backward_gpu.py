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
    (1, 2, 90, 48, 40, torch.float32),      # rows of 12 16-byte chunks: the decay gradient's per-warp form
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


def _f64(t):
    return t.detach().to("cpu", torch.float64).numpy() if hasattr(t, "detach") else np.asarray(t, np.float64)


def _check_decay_grad(got, q, k, decay, dq, dk, want, want_dq, want_dk, dtype, gated, what):
    """dgamma (fixed) or dg (gated), which the library forms from a_t = q_t . dQ_t - k_t . dK_t:
    dgamma_h = (1 / gamma_h) sum_{b,t} t a_t, dg_t = sum_{u>=t} a_u.

    (1) The decay-gradient step itself: the result equals that formula evaluated in fp64 on
        the library's own dq and dk, to fp32 summation error (1e-4 of the summed magnitudes).
    (2) Against the oracle: the formula is exact, so the error is what the errors of dq and dk
        propagate to. Their check allows ||dQ - dQ_ref|| <= tol ||dQ_ref||; by Cauchy-Schwarz
        |sum_t w_t q_t . (dQ - dQ_ref)_t| <= ||w_t |q_t| || tol ||dQ_ref|| (w_t = t / gamma for
        dgamma, the suffix indicator for dg), and the same for k and dK. That sum cancels
        (sum_t a_t = 0): the bound grows with N (1 - gamma^2) while dgamma does not, so the
        check allows the larger of the bound and tol_decay ||ref||.
    """
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    tol_decay = 1e-3 if dtype == torch.float32 else 5e-2
    q, k, dq, dk = (_f64(t) for t in (q, k, dq, dk))
    a = (q * dq).sum(-1) - (k * dk).sum(-1)                    # [B, H, N]
    mag = np.abs(q * dq).sum(-1) + np.abs(k * dk).sum(-1)
    qn, kn = np.linalg.norm(q, axis=-1), np.linalg.norm(k, axis=-1)
    eq, ek = tol * np.linalg.norm(_f64(want_dq)), tol * np.linalg.norm(_f64(want_dk))
    got, want = _f64(got), _f64(want)
    N = q.shape[2]
    if gated:
        formula = np.flip(np.cumsum(np.flip(a, -1), -1), -1)
        scale = np.flip(np.cumsum(np.flip(mag, -1), -1), -1)
        # every suffix sum is bounded through the whole sequence's norms
        per_row = np.linalg.norm(qn, axis=-1) * eq + np.linalg.norm(kn, axis=-1) * ek   # [B, H]
        bound = np.sqrt(N * (per_row ** 2).sum())
    else:
        t = np.arange(N, dtype=np.float64)
        gam = _f64(decay)
        formula = (t * a).sum((0, 2)) / gam
        scale = (t * mag).sum((0, 2)) / gam
        per_head = (np.sqrt(((t * qn) ** 2).sum((0, 2))) * eq + np.sqrt(((t * kn) ** 2).sum((0, 2))) * ek) / gam
        bound = np.linalg.norm(per_head)
    assert np.all(np.abs(got - formula) <= 1e-4 * scale + 1e-30), f"{what}: differs from its formula on dq, dk"
    err = np.linalg.norm(got - want)
    allowed = max(bound, tol_decay * np.linalg.norm(want))
    assert err <= allowed, f"{what}: error {err:.3e} > {allowed:.3e} (rel-L2 {err / np.linalg.norm(want):.3e})"


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
    _check_decay_grad(dgam, q, k, gam, dq, dkk, want[3], want[0], want[1], dtype, False, "dgamma")


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
    _check_decay_grad(dg, q, k, g, dq, dkk, want[3], want[0], want[1], dtype, True, "dg")


def test_gated_backward_steep_and_mild_gates(cuda_lib):
    """The reversed gated kernels form their mask weights from a row and a column factor when
    the chunk's cumulative log2-decay stays within +-100, else element by element; dq, dk and
    dv must match the oracle with both kinds of chunk in one call."""
    q, k, v, do, gen = _case(1, 4, 300, 64, 128, torch.bfloat16, seed=78)
    g = I.gate(1, 4, 300, gen)
    g[:, 1] *= 200.0
    g[:, 2, 150:] *= 200.0
    dq, dkk, dvv, _ = cuda_lib.chunkwise_backward(*(t.to(DEV) for t in (q, k, v, g, do)), 64, gated=True)
    assert cuda_lib.last_device_error() == 0
    want = O.gated_backward(q, k, v, g, do)
    _check(dq, want[0], torch.bfloat16, "dq")
    _check(dkk, want[1], torch.bfloat16, "dk")
    _check(dvv, want[2], torch.bfloat16, "dv")


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
    """ddecay=False: the same dq, dk, dv, bit for bit (the tensor-core path with dv in two
    pieces whose tiles add onto dq and dk in either order: each element is round(a + b))."""
    q, k, v, do, gen = _case(1, 2, 190, 256, 512, torch.bfloat16, seed=21)
    decay = I.gate(1, 2, 190, gen) * 4.0 if gated else torch.tensor([0.97, 0.9])
    d = [t.to(DEV) for t in (q, k, v, decay, do)]
    full = cuda_lib.chunkwise_backward(*d, 64, gated=gated)
    part = cuda_lib.chunkwise_backward(*d, 64, gated=gated, ddecay=False)
    assert part[3] is None
    for a, b in zip(full[:3], part[:3]):
        assert torch.equal(a, b)


# The dK and dV sums run over later tokens; on the tensor-core path they are computed by the
# time-reversed forward kernels (chunks visited from the last back, upper-triangular mask,
# mirrored decay factors). These cases reach each body of that kernel: the 128-token body
# (gamma >= 0.595, or gates in [-0.52, 0], with widths 128 or 256), the 64-token body with the
# merged output accumulator (gamma in [0.5, 0.595)) and with split accumulators (gamma < 0.5,
# steeper gates), on sequences long enough for few heads to be cut into segments chained from
# the end, with ragged last chunks.
REV_CASES = [
    # B, H, N, dk, dv, gammas (None: gated, gates x4; "mild": gated, gates as drawn)
    (1, 4, 450, 128, 128, [0.3, 0.55, 0.9, 0.999]),
    (1, 2, 300, 256, 256, [0.2, 0.45]),
    (2, 2, 700, 256, 512, [0.5, 0.7]),
    (1, 2, 1333, 128, 128, None),
    (1, 1, 2049, 256, 256, None),
    # gates in [-0.52, 0] ("mild"): the gated passes take the 128-token body too
    (1, 2, 700, 128, 128, "mild"),
    (1, 1, 2049, 256, 256, "mild"),
    (1, 2, 300, 256, 512, "mild"),
]


@pytest.mark.parametrize("B,H,N,dk,dv,gams", REV_CASES)
def test_backward_reversed_kernels_match_oracle(cuda_lib, B, H, N, dk, dv, gams):
    dtype = torch.bfloat16
    q, k, v, do, gen = _case(B, H, N, dk, dv, dtype, seed=5 * N + dk)
    gated = gams is None or gams == "mild"
    if gated:
        decay = I.gate(B, H, N, gen) * (1.0 if gams == "mild" else 4.0)
        want = O.gated_backward(q, k, v, decay, do)
    else:
        decay = torch.tensor(gams, dtype=torch.float32)
        want = O.ret_backward(q, k, v, decay, do)
    got = cuda_lib.chunkwise_backward(*(t.to(DEV) for t in (q, k, v, decay, do)), 64, gated=gated)
    assert cuda_lib.last_device_error() == 0
    for g, w, what in zip(got[:3], want[:3], ("dq", "dk", "dv")):
        _check(g, w, dtype, what)
    _check_decay_grad(got[3], q, k, decay, got[0], got[1], want[3], want[0], want[1], dtype, gated,
                      "dg" if gated else "dgamma")


def test_backward_launches_on_tensor_cores(cuda_lib):
    """The 1.3B-shaped backward launches two dQ pieces, two reversed dK pieces (each adding its
    tiles onto the zeroed dq or dk), the reversed dV call and the decay gradient: no copies
    of reversed operands and no separate sums of the pieces."""
    assert cuda_lib.chunkwise_backward_launches(4, 8, 2048, 256, 512, 64, torch.bfloat16) == 6
    assert cuda_lib.chunkwise_backward_launches(4, 8, 2048, 256, 512, 64, torch.bfloat16, ddecay=False) == 5
    # one piece (dv <= 256): dQ and dK store dq and dk directly
    assert cuda_lib.chunkwise_backward_launches(4, 8, 2048, 128, 256, 64, torch.bfloat16) == 4
