"""Failure detection on the GPU without a fault: the kernels' bounded wait, made to
run out by the library's self-test, must set the device error word, report it once
through ret_last_device_error, release the tensor memory it took and leave the
device usable for the tensor-core path."""
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from oracle import oracle as O
from tests.parity import TOL_BF16, assert_close

pytestmark = pytest.mark.gpu

DEV = "cuda:0"
RET_OK, RET_ERR_SHAPE, RET_ERR_TIMEOUT = 0, 2, 6


def _small_tensor_core_call(cuda_lib):
    B, H, N, dk, dv = 1, 2, 200, 128, 128
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, seed=77)
    gam = I.gammas(H)
    assert cuda_lib.chunkwise_path(dk, dv, 64, torch.bfloat16) == 1
    o = cuda_lib.ret_chunkwise(q.to(DEV), k.to(DEV), v.to(DEV), gam.to(DEV), 64)
    assert_close(o, O.ret_chunkwise(q, k, v, gam, 64)[0], torch.bfloat16, "o after self-test")


def test_selftest_rejects_limits_out_of_range(cuda_lib):
    assert cuda_lib.selftest_wait_timeout(0) == RET_ERR_SHAPE
    assert cuda_lib.selftest_wait_timeout(1_000_001) == RET_ERR_SHAPE


def test_bounded_wait_runs_out_reports_once_and_recovers(cuda_lib):
    assert cuda_lib.last_device_error() == RET_OK
    for _ in range(3):  # repeated: tensor memory is released each time
        assert cuda_lib.selftest_wait_timeout(2000) == RET_OK
        assert cuda_lib.last_device_error() == RET_ERR_TIMEOUT
        assert cuda_lib.last_device_error() == RET_OK  # reading clears the word
    _small_tensor_core_call(cuda_lib)
    assert cuda_lib.last_device_error() == RET_OK
