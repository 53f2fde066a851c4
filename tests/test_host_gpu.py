"""The host-buffer forward (ret_chunkwise_host, gated_ret_chunkwise_host): inputs and output in
host memory, copies pipelined with the forward over groups of heads. Each group is computed as
a problem of its own, whose plan (sequence segments to fill the SMs) may differ from the whole
batch's, so the result is checked against the fp64 oracle, like every forward, and against the
device-buffer call to the same tolerance; repeated calls agree bit for bit."""
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from linear_attention_ret_b200 import ret
from oracle import oracle as O
from tests.parity import TOL_BF16, TOL_F32, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

CASES = [
    # B, H, N, dk, dv, chunk, dtype
    (4, 8, 512, 256, 512, 64, torch.bfloat16),   # 8 groups of 4 heads inside one batch each
    (1, 3, 300, 64, 128, 64, torch.bfloat16),    # 3 heads, one group each, ragged tail
    (3, 5, 200, 128, 256, 64, torch.bfloat16),   # 2 groups per batch, of 3 and 2 heads
    (9, 2, 130, 64, 128, 64, torch.bfloat16),    # B >= 8: groups of whole batches (2, 2, 2, 2, 1)
    (2, 2, 100, 32, 48, 32, torch.float32),      # CUDA-core path
]


def _device_reference(q, k, v, decay, chunk, gated):
    qd, kd, vd, dd = (t.to(DEV) for t in (q, k, v, decay))
    o = ret.gated_ret_chunkwise(qd, kd, vd, dd, chunk) if gated else ret.ret_chunkwise(qd, kd, vd, dd, chunk)
    return o.cpu()


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("B,H,N,dk,dv,chunk,dtype", CASES)
def test_host_call_matches_oracle(cuda_lib, B, H, N, dk, dv, chunk, dtype, gated):
    gen = torch.Generator().manual_seed(B * 100 + H * 10 + N)
    q, k, v = (t.pin_memory() for t in I.qkv(B, H, N, dk, dv, dtype, gen=gen))
    decay = (I.gate(B, H, N, gen) if gated else I.gammas(H)).pin_memory()
    f = ret.gated_ret_chunkwise_host if gated else ret.ret_chunkwise_host
    o = f(q, k, v, decay, chunk)
    assert ret.last_device_error() == 0
    assert not o.is_cuda and o.shape == (B, H, N, dv)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    want = (O.gated_chunkwise if gated else O.ret_chunkwise)(q, k, v, decay, chunk)[0]
    err = rel_l2(o, want)
    assert err <= tol, f"against the oracle: rel-L2 {err:.3e} > {tol:.0e}"
    err = rel_l2(o, _device_reference(q, k, v, decay, chunk, gated).double())
    assert err <= tol, f"against the device-buffer call: rel-L2 {err:.3e} > {tol:.0e}"
    assert torch.equal(f(q, k, v, decay, chunk), o)   # the same plan every call


def test_host_call_with_pageable_buffers_and_preallocated_output(cuda_lib):
    B, H, N, dk, dv = 2, 8, 640, 128, 128
    gen = torch.Generator().manual_seed(12)
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen)     # not page-locked
    g = I.gate(B, H, N, gen)
    o = torch.full((B, H, N, dv), float("nan"), dtype=torch.bfloat16)
    out = ret.gated_ret_chunkwise_host(q, k, v, g, 64, o=o)
    assert out is o
    assert torch.equal(o, ret.gated_ret_chunkwise_host(q.pin_memory(), k.pin_memory(), v.pin_memory(),
                                                       g.pin_memory(), 64))
    err = rel_l2(o, O.gated_chunkwise(q, k, v, g, 64)[0])
    assert err <= TOL_BF16, f"rel-L2 {err:.3e}"


def test_host_call_back_to_back_on_a_side_stream(cuda_lib):
    """Calls enqueued without waiting, on a stream other than the default: each result is
    complete once the stream is."""
    B, H, N, dk, dv = 4, 8, 512, 256, 512
    gam = I.gammas(H)
    ins = [tuple(t.pin_memory() for t in I.qkv(B, H, N, dk, dv, torch.bfloat16, seed=20 + i)) for i in range(3)]
    outs = [torch.empty(B, H, N, dv, dtype=torch.bfloat16).pin_memory() for _ in ins]
    s = torch.cuda.Stream()
    for (q, k, v), o in zip(ins, outs):
        ret.ret_chunkwise_host(q, k, v, gam, 64, o=o, stream=s, sync=False)
    s.synchronize()
    for (q, k, v), o in zip(ins, outs):
        assert torch.equal(o, ret.ret_chunkwise_host(q, k, v, gam, 64))


BWD_CASES = [
    # B, H, N, dk, dv, dtype
    (4, 8, 256, 256, 512, torch.bfloat16),   # 8 groups; two dv pieces per group
    (2, 3, 200, 128, 128, torch.bfloat16),   # groups of 2 and 1 heads
    (9, 2, 100, 64, 128, torch.bfloat16),    # groups of whole batches
    (1, 2, 90, 48, 40, torch.float32),       # CUDA-core path, rows of 12 chunks
]


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("B,H,N,dk,dv,dtype", BWD_CASES)
def test_host_backward_matches_oracle(cuda_lib, B, H, N, dk, dv, dtype, gated):
    gen = torch.Generator().manual_seed(7 * B + 3 * H + N)
    q, k, v = I.qkv(B, H, N, dk, dv, dtype, gen=gen)
    do = (torch.randn(B, H, N, dv, generator=gen) / dv ** 0.5).to(dtype)
    decay = I.gate(B, H, N, gen) * 4.0 if gated else torch.tensor([0.96875, 0.999, 0.9, 0.75, 0.5][:H] + [0.99] * max(0, H - 5))
    host = [t.pin_memory() for t in (q, k, v, decay, do)]
    got = ret.chunkwise_backward_host(*host, 64, gated=gated)
    assert ret.last_device_error() == 0
    assert all(not t.is_cuda for t in got)
    dev = ret.chunkwise_backward(*(t.to(DEV) for t in (q, k, v, decay, do)), 64, gated=gated)
    want = (O.gated_backward if gated else O.ret_backward)(q, k, v, decay, do)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    for name, g, d, w in zip(("dq", "dk", "dv"), got[:3], dev[:3], want[:3]):
        assert rel_l2(g, w) <= tol, f"{name} against the oracle"
        assert rel_l2(g, d.double().cpu()) <= tol, f"{name} against the device-buffer call"
    # the decay gradient against the device-buffer call (which is checked against the oracle and
    # its formula elsewhere): it sums a_t = q_t.dQ_t - k_t.dK_t with cancellation, and a group's
    # dq, dk may round differently from the whole batch's, so the bound scales with the summed
    # magnitudes |q_t.dQ_t| + |k_t.dK_t| (suffix sums for dg; sum_t t(..)/gamma for dgamma)
    qd, kd, dqd, dkd = (t.double().cpu() for t in (q, k, dev[0], dev[1]))
    mag = (qd * dqd).abs().sum(-1) + (kd * dkd).abs().sum(-1)
    if gated:
        scale = mag.flip(-1).cumsum(-1).flip(-1)
    else:
        scale = (torch.arange(N, dtype=torch.float64) * mag).sum((0, 2)) / decay.double()
    rel = 1e-5 if dtype == torch.float32 else 1e-2
    assert torch.all((got[3].double() - dev[3].double().cpu()).abs() <= rel * scale + 1e-12)


def test_host_backward_without_decay_gradient(cuda_lib):
    B, H, N, dk, dv = 2, 4, 300, 128, 256
    q, k, v = (t.pin_memory() for t in I.qkv(B, H, N, dk, dv, torch.bfloat16, seed=9))
    do = I.output_grad(B, H, N, dv, torch.bfloat16, seed=9).pin_memory()
    gam = I.gammas(H).pin_memory()
    with_dd = ret.chunkwise_backward_host(q, k, v, gam, do, 64)
    without = ret.chunkwise_backward_host(q, k, v, gam, do, 64, ddecay=False)
    assert without[3] is None
    for a, b in zip(with_dd[:3], without[:3]):
        assert torch.equal(a, b)


def _head(t, b, h):
    return t[b:b + 1, h:h + 1].contiguous()


@pytest.mark.parametrize("name", ["retnet_1p3b", "retnet_6p7b_long", "gated"])
def test_full_size_host_call_sampled_heads(cuda_lib, name):
    """The host-buffer forward at the workloads' full sizes, as the bench's e2e part calls it,
    against the oracle on sampled heads (one of them in the last head group)."""
    cfg = I.CONFIGS[name]
    x = {key: t.pin_memory() for key, t in I.config_inputs(cfg).items()}
    gated = "g" in x
    if gated:
        o = ret.gated_ret_chunkwise_host(x["q"], x["k"], x["v"], x["g"], cfg.chunk)
    else:
        o = ret.ret_chunkwise_host(x["q"], x["k"], x["v"], x["gamma"], cfg.chunk)
    assert ret.last_device_error() == 0
    for b, h in [(0, 0), (cfg.B - 1, cfg.H - 1)]:
        q, k, v = (_head(x[n], b, h) for n in ("q", "k", "v"))
        if gated:
            want = O.gated_chunkwise(q, k, v, _head(x["g"], b, h), cfg.chunk)[0]
        else:
            want = O.ret_chunkwise(q, k, v, x["gamma"][h:h + 1], cfg.chunk)[0]
        err = rel_l2(o[b:b + 1, h:h + 1], want)
        assert err <= TOL_BF16, f"{name} head ({b},{h}): rel-L2 {err:.3e}"


@pytest.mark.parametrize("gated", [False, True])
def test_full_size_host_backward_matches_device_call(cuda_lib, gated):
    """The host-buffer backward at the backward workloads' full sizes against the device-buffer
    call (itself checked against the oracle on sampled heads at full size)."""
    cfg = I.CONFIGS["gated" if gated else "retnet_1p3b"]
    x = I.config_inputs(cfg)
    do = I.output_grad(cfg.B, cfg.H, cfg.N, cfg.dv, cfg.dtype, seed=0)
    decay = x["g"] if gated else x["gamma"]
    got = ret.chunkwise_backward_host(*(t.pin_memory() for t in (x["q"], x["k"], x["v"], decay, do)), cfg.chunk,
                                      gated=gated)
    dev = ret.chunkwise_backward(*(t.to(DEV) for t in (x["q"], x["k"], x["v"], decay, do)), cfg.chunk, gated=gated)
    assert ret.last_device_error() == 0
    for name, g, d in zip(("dq", "dk", "dv"), got[:3], dev[:3]):
        err = rel_l2(g, d.double().cpu())
        assert err <= TOL_BF16, f"{name}: rel-L2 {err:.3e}"
