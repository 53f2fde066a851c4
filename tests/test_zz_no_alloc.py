"""ret_chunkwise_noalloc: the chunkwise call for callers that cannot let the
library allocate device memory (their own allocator owns the memory, or
allocation is forbidden once they are running). Each call is checked against
the fp64 oracle's chunkwise form on the same inputs and initial state, call
after call, while the scratch comes from the fixed buffer compiled into
libret.so; the allocating call is run beside it only as a second witness.

Whether a shape needs scratch depends on the device's SM count (long
sequences of few heads are split into segments to fill the SMs), so every
expectation about the buffer comes from the library's own host-side query of
the scratch a call would use.

This file is named to be collected last, so a run that stops at the first
failure has run every other test before it; it also passes on its own in a
fresh process.
"""
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from oracle import oracle as O
from tests.parity import TOL_BF16, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _inputs(B, H, N, dk, dv, seed):
    gen = torch.Generator().manual_seed(seed)
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    gam = I.gammas(H)
    want_o, want_s = O.ret_chunkwise(q, k, v, gam, 64, state_in=S0.double().numpy())
    return [t.to(DEV) for t in (q, k, v, gam, S0)], want_o, want_s


@pytest.mark.parametrize("B,H,N,dk,dv", [(1, 2, 2048, 128, 128), (1, 4, 1500, 256, 256)])
def test_noalloc_matches_oracle_twice(cuda_lib, B, H, N, dk, dv):
    # a long sequence of few heads: the tensor-core path splits it and takes scratch
    need = cuda_lib.noalloc_scratch_bytes(B, H, N, dk, dv, 64, torch.bfloat16)
    if need == 0:
        pytest.skip("this device's SM count does not split the sequence, so no scratch is used")
    assert 0 < need <= cuda_lib.NOALLOC_SCRATCH_BYTES
    (q, k, v, gam, S0), want_o, want_s = _inputs(B, H, N, dk, dv, seed=N + dk)
    o_alloc = cuda_lib.ret_chunkwise(q, k, v, gam, 64, state_in=S0)
    for call in range(2):  # the buffer keeps the previous call's contents; results must not depend on it
        s_out = torch.full_like(S0, float("nan"))
        o = cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S0, state_out=s_out)
        torch.cuda.synchronize()
        assert cuda_lib.last_device_error() == 0
        assert rel_l2(o, want_o) <= TOL_BF16, f"o vs oracle, call {call}"
        assert rel_l2(s_out, want_s) <= TOL_BF16, f"state vs oracle, call {call}"
        assert rel_l2(o, o_alloc.float().cpu().double().numpy()) <= TOL_BF16, f"o vs ret_chunkwise, call {call}"


def test_noalloc_in_place_state_twice(cuda_lib):
    B, H, N, dk, dv = 1, 2, 1200, 64, 128
    (q, k, v, gam, S0), want_o, want_s = _inputs(B, H, N, dk, dv, seed=5)
    assert cuda_lib.noalloc_scratch_bytes(B, H, N, dk, dv, 64, torch.bfloat16, in_place=True) \
        <= cuda_lib.NOALLOC_SCRATCH_BYTES
    for call in range(2):
        S = S0.clone()
        o = cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S, state_out=S)
        torch.cuda.synchronize()
        assert rel_l2(o, want_o) <= TOL_BF16, f"o, call {call}"
        assert rel_l2(S, want_s) <= TOL_BF16, f"state, call {call}"


def test_noalloc_rejects_problem_larger_than_buffer(cuda_lib):
    # 8 heads x 256 x 1024 fp32 end states plus the copy an in-place state needs: on a
    # device that splits this sequence they exceed the buffer and the call is rejected on
    # the host, nothing launched; with separate state buffers the same problem fits
    B, H, N, dk, dv = 1, 8, 640, 256, 1024
    (q, k, v, gam, S0), want_o, want_s = _inputs(B, H, N, dk, dv, seed=7)
    need_in_place = cuda_lib.noalloc_scratch_bytes(B, H, N, dk, dv, 64, torch.bfloat16, in_place=True)
    if need_in_place > cuda_lib.NOALLOC_SCRATCH_BYTES:
        S = S0.clone()
        with pytest.raises(cuda_lib.RetError) as err:
            cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S, state_out=S)
        assert err.value.code == 8  # RET_ERR_SCRATCH
        torch.cuda.synchronize()
        assert torch.equal(S, S0), "a rejected call must not touch the state"
    assert cuda_lib.noalloc_scratch_bytes(B, H, N, dk, dv, 64, torch.bfloat16) <= cuda_lib.NOALLOC_SCRATCH_BYTES
    s_out = torch.empty_like(S0)
    o = cuda_lib.ret_chunkwise_noalloc(q, k, v, gam, 64, state_in=S0, state_out=s_out)
    torch.cuda.synchronize()
    assert rel_l2(o, want_o) <= TOL_BF16
    assert rel_l2(s_out, want_s) <= TOL_BF16


def test_noalloc_scratch_query_on_the_host(cuda_lib):
    # the query launches nothing; invalid sizes give -1, the CUDA-core path and N = 0 need nothing
    assert cuda_lib.noalloc_scratch_bytes(0, 1, 64, 64, 128, 64, torch.bfloat16) == -1
    assert cuda_lib.noalloc_scratch_bytes(1, 1, 0, 64, 128, 64, torch.bfloat16) == 0
    assert cuda_lib.noalloc_scratch_bytes(1, 1, 4096, 32, 32, 32, torch.float32) == 0
    # many heads fill the SMs without a split: no scratch
    assert cuda_lib.noalloc_scratch_bytes(4, 64, 2048, 128, 128, 64, torch.bfloat16) == 0
