"""The autograd wrapper's routing on the CPU: the library calls are replaced, inside this
test only, by the fp64 oracle, so that what is checked is which tensors reach which call and
which gradients come back (the kernels themselves are covered by the GPU parity tests)."""
import numpy as np
import pytest
import torch

from linear_attention_ret_b200 import autograd as A
from linear_attention_ret_b200 import ret
from oracle import oracle as O


@pytest.fixture
def oracle_library(monkeypatch):
    calls = []

    def fwd(q, k, v, decay, chunk, **_):
        calls.append(("fwd", chunk))
        return torch.from_numpy(O.ret_chunkwise(q, k, v, decay, chunk)[0])

    def gfwd(q, k, v, g, chunk, **_):
        calls.append(("gfwd", chunk))
        return torch.from_numpy(O.gated_chunkwise(q, k, v, g, chunk)[0])

    def bwd(q, k, v, decay, do, chunk, gated=False, ddecay=True, **_):
        calls.append(("bwd", chunk, gated, ddecay))
        grads = (O.gated_backward if gated else O.ret_backward)(q, k, v, decay, do)
        out = [torch.from_numpy(np.ascontiguousarray(g)) for g in grads]
        return out[0], out[1], out[2], (out[3] if ddecay else None)

    monkeypatch.setattr(ret, "ret_chunkwise", fwd)
    monkeypatch.setattr(ret, "gated_ret_chunkwise", gfwd)
    monkeypatch.setattr(ret, "chunkwise_backward", bwd)
    return calls


def _leaves(gated, decay_grad, seed=0):
    g = torch.Generator().manual_seed(seed)
    q, k = torch.randn(1, 2, 13, 4, generator=g, dtype=torch.float64), torch.randn(1, 2, 13, 4, generator=g,
                                                                                    dtype=torch.float64)
    v = torch.randn(1, 2, 13, 3, generator=g, dtype=torch.float64)
    decay = (-torch.rand(1, 2, 13, generator=g, dtype=torch.float64) / 4) if gated else \
        torch.tensor([0.9, 0.7], dtype=torch.float64)
    for t in (q, k, v):
        t.requires_grad_(True)
    decay.requires_grad_(decay_grad)
    return q, k, v, decay


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("decay_grad", [False, True])
def test_gradients_route_to_the_inputs(oracle_library, gated, decay_grad):
    q, k, v, decay = _leaves(gated, decay_grad)
    o = A.chunkwise_retention(q, k, v, decay, chunk=8, gated=gated)
    do = torch.randn(o.shape, dtype=torch.float64, generator=torch.Generator().manual_seed(5))
    (o * do).sum().backward()
    want = (O.gated_backward if gated else O.ret_backward)(q.detach(), k.detach(), v.detach(), decay.detach(), do)
    np.testing.assert_allclose(q.grad.numpy(), want[0], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(k.grad.numpy(), want[1], rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(v.grad.numpy(), want[2], rtol=1e-12, atol=1e-12)
    if decay_grad:
        np.testing.assert_allclose(decay.grad.numpy(), want[3], rtol=1e-12, atol=1e-12)
    else:
        assert decay.grad is None
    # one forward call, one backward call that asks for the decay gradient only when it is wanted
    assert oracle_library[0] == ("gfwd" if gated else "fwd", 8)
    assert oracle_library[1] == ("bwd", 8, gated, decay_grad)


def test_forward_matches_the_operator(oracle_library):
    q, k, v, decay = _leaves(False, False, seed=3)
    o = A.chunkwise_retention(q, k, v, decay, chunk=4)
    want = O.ret_brute(q.detach(), k.detach(), v.detach(), decay.detach())
    np.testing.assert_allclose(o.detach().numpy(), want, rtol=1e-12, atol=1e-12)
