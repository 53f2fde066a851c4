"""GPU parity of the multi-scale retention output epilogue (per-head RMSNorm without
affine weights times the swish of the gate) against the fp64 oracle."""
import numpy as np
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from oracle import oracle as O
from tests.parity import TOL_BF16, TOL_F32, rel_l2

pytestmark = pytest.mark.gpu

DEV = "cuda:0"

NORM_CASES = [
    # B, H, N, dv, dtype: vector kernel with 1..8 chunks per lane and 1..32 lanes per row, and the scalar kernel
    (4, 8, 2048, 512, torch.bfloat16),   # the 1.3B-shaped retention output
    (2, 3, 77, 128, torch.bfloat16),
    (1, 2, 33, 64, torch.bfloat16),
    (1, 1, 5, 8, torch.bfloat16),        # one chunk per row
    (1, 2, 9, 2048, torch.bfloat16),     # eight chunks per lane
    (1, 3, 19, 40, torch.bfloat16),      # 80-byte rows: scalar kernel
    (2, 2, 31, 32, torch.float32),
    (1, 2, 17, 1024, torch.float32),
    (1, 2, 13, 100, torch.float32),      # scalar kernel
    (1, 1, 3, 3, torch.float32),
]


def _inputs(B, H, N, dv, dtype, seed):
    o = I.retention_output(B, H, N, dv, dtype, seed=seed)
    gate = I.gate_projection(B, H, N, dv, dtype, seed=seed)
    return o, gate


@pytest.mark.parametrize("B,H,N,dv,dtype", NORM_CASES)
def test_norm_gate_matches_oracle(cuda_lib, B, H, N, dv, dtype):
    o, gate = _inputs(B, H, N, dv, dtype, seed=N + dv)
    y = cuda_lib.msr_norm_gate(o.to(DEV), gate.to(DEV), 1e-5)
    want = O.msr_norm_gate(o, gate, 1e-5)
    tol = TOL_F32 if dtype == torch.float32 else TOL_BF16
    assert rel_l2(y, want) <= tol
    # every row, not only the whole tensor: worst row's relative error
    got = y.double().cpu().numpy().reshape(-1, dv)
    ref = want.reshape(-1, dv)
    row_err = np.linalg.norm(got - ref, axis=1) / np.maximum(np.linalg.norm(ref, axis=1), 1e-30)
    assert row_err.max() <= (1e-5 if dtype == torch.float32 else 1e-2), row_err.max()


def test_norm_gate_in_place_on_gate(cuda_lib):
    o, gate = _inputs(2, 4, 50, 256, torch.bfloat16, seed=5)
    g = gate.to(DEV)
    y = cuda_lib.msr_norm_gate(o.to(DEV), g, 1e-5, y=g)
    assert y.data_ptr() == g.data_ptr()
    assert rel_l2(y, O.msr_norm_gate(o, gate, 1e-5)) <= TOL_BF16


def test_norm_gate_edge_cases(cuda_lib):
    # zero rows stay zero; a large eps scales down; N = 0 launches nothing
    o = torch.zeros(1, 2, 4, 64, dtype=torch.float32)
    gate = torch.randn(1, 4, 2, 64)
    y = cuda_lib.msr_norm_gate(o.to(DEV), gate.to(DEV), 1e-5)
    assert torch.count_nonzero(y).item() == 0
    o2, gate2 = _inputs(1, 2, 8, 64, torch.float32, seed=3)
    for eps in (0.0, 10.0):
        y2 = cuda_lib.msr_norm_gate(o2.to(DEV), gate2.to(DEV), eps)
        assert rel_l2(y2, O.msr_norm_gate(o2, gate2, eps)) <= TOL_F32
    empty = torch.empty(1, 2, 0, 64, device=DEV)
    assert cuda_lib.msr_norm_gate(empty, torch.empty(1, 0, 2, 64, device=DEV)).numel() == 0
    assert cuda_lib.last_device_error() == 0


def test_norm_gate_rejects_overlap_and_bad_eps(cuda_lib):
    import ctypes
    from linear_attention_ret_b200 import ret
    lib = ret.load()
    o = torch.randn(1, 2, 8, 64, device=DEV)
    g = torch.randn(1, 8, 2, 64, device=DEV)
    p = lambda t: ctypes.c_void_p(t.data_ptr())
    # y overlapping o, y overlapping gate without being gate, negative eps
    assert lib.ret_msr_norm_gate(p(o), p(g), p(o), 1, 2, 8, 64, 1e-5, ret.RET_F32, None) == 4
    assert lib.ret_msr_norm_gate(p(o), p(g), ctypes.c_void_p(g.data_ptr() + 256), 1, 2, 8, 64, 1e-5, ret.RET_F32,
                                 None) == 4
    assert lib.ret_msr_norm_gate(p(o), p(g), p(g), 1, 2, 8, 64, -1.0, ret.RET_F32, None) == 2


def test_chunkwise_then_norm_gate_matches_oracle(cuda_lib):
    """The module's retention output path: chunkwise retention, then the epilogue on its output."""
    cfg = I.CONFIGS["retnet_1p3b"]
    x = I.config_inputs(cfg, seed=9, B=1, N=300)
    gate = I.gate_projection(1, cfg.H, 300, cfg.dv, cfg.dtype, seed=9)
    o = cuda_lib.ret_chunkwise(*(x[n].to(DEV) for n in ("q", "k", "v", "gamma")), cfg.chunk)
    y = cuda_lib.msr_norm_gate(o, gate.to(DEV), 1e-5)
    o_ref, _ = O.ret_chunkwise(x["q"], x["k"], x["v"], x["gamma"], cfg.chunk)
    want = O.msr_norm_gate(o_ref, gate, 1e-5)
    assert rel_l2(y, want) <= TOL_BF16
