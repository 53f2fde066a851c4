"""ret_chunkwise_noalloc: the chunkwise call for callers that cannot let the
library allocate device memory (their own allocator owns the memory, or
allocation is forbidden once they are running). It must give what
ret_chunkwise gives, call after call, while taking its scratch from the fixed
buffer compiled into libret.so.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it; it also passes on its own in a
fresh process.
"""
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from tests.parity import TOL_BF16, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _inputs(B, H, N, dk, dv, seed):
    gen = torch.Generator().manual_seed(seed)
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    return [t.to(DEV) for t in (q, k, v, I.gammas(H), S0)]


@pytest.mark.parametrize("B,H,N,dk,dv", [(1, 2, 2048, 128, 128), (1, 4, 1500, 256, 256)])
def test_noalloc_matches_allocating_call_twice(cuda_lib, B, H, N, dk, dv):
    # a long sequence of few heads: the tensor-core path splits it and needs scratch
    assert cuda_lib.chunkwise_launches(B, H, N, dk, dv, 64, torch.bfloat16) == 3  # state-only pass, segment prefix, full pass
    q, k, v, gam, S0 = _inputs(B, H, N, dk, dv, seed=N + dk)
    s_ref = torch.empty_like(S0)
    o_ref = cuda_lib.ret_chunkwise(q, k, v, gam, 64, state_in=S0, state_out=s_ref)
    for call in range(2):  # the buffer keeps the previous call's contents; results must not depend on it
        s_out = torch.full_like(S0, float("nan"))
        o = cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S0, state_out=s_out)
        torch.cuda.synchronize()
        assert cuda_lib.last_device_error() == 0
        assert rel_l2(o, o_ref.float().cpu().double().numpy()) <= TOL_BF16, f"o, call {call}"
        assert rel_l2(s_out, s_ref.cpu().double().numpy()) <= TOL_BF16, f"state, call {call}"


def test_noalloc_in_place_state_twice(cuda_lib):
    B, H, N, dk, dv = 1, 2, 1200, 64, 128
    q, k, v, gam, S0 = _inputs(B, H, N, dk, dv, seed=5)
    s_ref = torch.empty_like(S0)
    o_ref = cuda_lib.ret_chunkwise(q, k, v, gam, 64, state_in=S0, state_out=s_ref)
    for call in range(2):
        S = S0.clone()
        o = cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S, state_out=S)
        torch.cuda.synchronize()
        assert rel_l2(o, o_ref.float().cpu().double().numpy()) <= TOL_BF16, f"o, call {call}"
        assert rel_l2(S, s_ref.cpu().double().numpy()) <= TOL_BF16, f"state, call {call}"


def test_noalloc_rejects_problem_larger_than_buffer(cuda_lib):
    # 8 heads x 256 x 1024 fp32 end states (8 MiB) plus the copy an in-place state needs (8 MiB)
    # exceed the 16 MiB buffer: rejected on the host, nothing launched
    B, H, N, dk, dv = 1, 8, 640, 256, 1024
    q, k, v, gam, S0 = _inputs(B, H, N, dk, dv, seed=7)
    with pytest.raises(cuda_lib.RetError) as err:
        cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S0, state_out=S0)
    assert err.value.code == 8  # RET_ERR_SCRATCH
    # separate state buffers fit
    s_out = torch.empty_like(S0)
    o = cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S0, state_out=s_out)
    o_ref = cuda_lib.ret_chunkwise(q, k, v, gam, 64, state_in=S0)
    torch.cuda.synchronize()
    assert rel_l2(o, o_ref.float().cpu().double().numpy()) <= TOL_BF16
