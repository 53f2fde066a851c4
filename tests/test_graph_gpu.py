"""The C ABI under CUDA graph capture: each call only enqueues work on the caller's stream
(and, for the backward, on library streams forked from it and joined back), so a captured
call replays to the same result as the eager call. Covered: the chunkwise forward with a
split sequence (its segment states live in scratch taken from the stream-ordered pool), the
gated forward, the fixed-buffer entry point and both backward forms with their fork/join of
library streams."""
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from linear_attention_ret_b200 import ret

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _capture_and_replay(fn, replays=3):
    """Warm fn up on a side stream, capture it in a graph, replay it and return its outputs
    from the last replay together with the eager outputs taken before the capture."""
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        eager = [t.clone() if t is not None else None for t in fn()]
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        outs = fn()
    for _ in range(replays):
        graph.replay()
    torch.cuda.synchronize()
    assert ret.last_device_error() == 0
    got = [t.clone() if t is not None else None for t in outs]
    del graph
    return eager, got


@pytest.mark.parametrize("B,H,N,dk,dv,chunk", [
    (1, 2, 4096, 256, 512, 64),    # few CTAs: the sequence is cut into segments (scratch, three launches)
    (2, 4, 1000, 128, 128, 64),    # ragged tail
])
def test_chunkwise_forward_replays_like_eager(cuda_lib, B, H, N, dk, dv, chunk):
    q, k, v = (t.to(DEV) for t in I.qkv(B, H, N, dk, dv, torch.bfloat16, seed=3))
    gam = I.gammas(H).to(DEV)
    o = torch.empty(B, H, N, dv, dtype=torch.bfloat16, device=DEV)
    st = torch.empty(B, H, dk, dv, dtype=torch.float32, device=DEV)
    eager, got = _capture_and_replay(lambda: (ret.ret_chunkwise(q, k, v, gam, chunk, state_out=st, o=o), st))
    for e, g in zip(eager, got):
        assert torch.equal(e, g)


def test_noalloc_forward_replays_like_eager(cuda_lib):
    B, H, N, dk, dv = 1, 2, 2048, 256, 256
    q, k, v = (t.to(DEV) for t in I.qkv(B, H, N, dk, dv, torch.bfloat16, seed=4))
    gam = I.gammas(H).to(DEV)
    o = torch.empty(B, H, N, dv, dtype=torch.bfloat16, device=DEV)
    eager, got = _capture_and_replay(lambda: (ret.ret_chunkwise_noalloc(q, k, v, gam, 64, o=o),))
    assert torch.equal(eager[0], got[0])


def test_gated_forward_replays_like_eager(cuda_lib):
    B, H, N, dk, dv = 1, 2, 8192, 128, 128
    gen = torch.Generator().manual_seed(5)
    q, k, v = (t.to(DEV) for t in I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen))
    g = I.gate(B, H, N, gen).to(DEV)
    o = torch.empty(B, H, N, dv, dtype=torch.bfloat16, device=DEV)
    eager, got = _capture_and_replay(lambda: (ret.gated_ret_chunkwise(q, k, v, g, 64, o=o),))
    assert torch.equal(eager[0], got[0])


@pytest.mark.parametrize("gated,B,H,N,dk,dv", [
    (False, 1, 2, 1024, 256, 512),   # two pieces of the dv contraction adding onto zeroed dq, dk
    (True, 1, 2, 4096, 128, 128),    # one piece; the gate gradient's suffix sum
])
def test_backward_replays_like_eager(cuda_lib, gated, B, H, N, dk, dv):
    gen = torch.Generator().manual_seed(6)
    q, k, v = (t.to(DEV) for t in I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen))
    do = (torch.randn(B, H, N, dv, generator=gen) / dv ** 0.5).to(torch.bfloat16).to(DEV)
    decay = (I.gate(B, H, N, gen) if gated else I.gammas(H)).to(DEV)
    eager, got = _capture_and_replay(lambda: ret.chunkwise_backward(q, k, v, decay, do, 64, gated=gated))
    for name, e, g in zip(("dq", "dk", "dv"), eager[:3], got[:3]):
        assert torch.equal(e, g), name   # two pieces: round(a + b) in either order
    # the decay gradient: dgamma sums with fp32 atomics in any order, so two calls agree to
    # rounding of the summed magnitudes (the sum itself cancels: sum_t a_t = 0); dg in one order
    if gated:
        assert torch.equal(got[3], eager[3])
    else:
        qd, kd, dqd, dkd = (t.double() for t in (q, k, eager[0], eager[1]))
        mag = (qd * dqd).abs().sum(-1) + (kd * dkd).abs().sum(-1)        # [B, H, N]
        t = torch.arange(N, dtype=torch.float64, device=DEV)
        scale = (t * mag).sum((0, 2)) / decay.double()
        assert torch.all((got[3].double() - eager[3].double()).abs() <= 1e-5 * scale)
