"""The C ABI library builds, loads without a GPU, exports every declared symbol,
and rejects bad arguments on the host before anything is launched."""
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ret.h")


def _declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"RET_API\s+[\w\s\*]+?\b(\w+)\s*\(", text)))


@pytest.fixture(scope="module")
def lib():
    from linear_attention_ret_b200 import build, ret
    build.build()
    return ret.load()


def test_header_declares_the_four_entry_points():
    syms = _declared_symbols()
    for name in ("ret_parallel", "ret_chunkwise", "ret_recurrent_step", "gated_ret_chunkwise"):
        assert name in syms


def test_library_exports_every_declared_symbol(lib):
    from linear_attention_ret_b200 import ret
    syms = _declared_symbols()
    assert set(syms) == set(ret.SYMBOLS)
    for name in syms:
        assert hasattr(lib, name), name


def test_status_strings(lib):
    for code in range(9):
        assert lib.ret_status_str(code)
    assert lib.ret_status_str(99) == b"unknown status"
    assert lib.ret_version() == b"0.1.0"


def test_path_selection(lib):
    from linear_attention_ret_b200.ret import RET_BF16, RET_F32
    assert lib.ret_chunkwise_path(32, 32, 32, RET_F32) == 0
    assert lib.ret_chunkwise_path(512, 64, 64, RET_BF16) == -1   # dk above 256
    assert lib.ret_chunkwise_path(64, 64, 0, RET_BF16) == -1
    assert lib.ret_chunkwise_path(64, 64, 64, 7) == -1


def _call_chunkwise(lib, fn="ret_chunkwise", B=1, H=1, N=8, dk=64, dv=64, chunk=64, dt=1, ptr=None):
    p = ptr
    return getattr(lib, fn)(p, p, p, p, p, None, None, B, H, N, dk, dv, chunk, dt, None)


@pytest.mark.parametrize("fn", ["ret_chunkwise", "gated_ret_chunkwise"])
def test_chunkwise_validation(lib, fn):
    # shape errors come first, then unsupported sizes, then null pointers: no launch in any case
    assert _call_chunkwise(lib, fn, B=0) == 2
    assert _call_chunkwise(lib, fn, N=-1) == 2
    assert _call_chunkwise(lib, fn, chunk=0) == 2
    assert _call_chunkwise(lib, fn, dt=5) == 3
    assert _call_chunkwise(lib, fn, dk=300) == 4
    assert _call_chunkwise(lib, fn, B=70000) == 4
    assert _call_chunkwise(lib, fn) == 1  # NULL q, k, v


@pytest.mark.parametrize("fn", ["ret_chunkwise_host", "gated_ret_chunkwise_host"])
def test_host_chunkwise_validation(lib, fn):
    def call(B=1, H=1, N=8, dk=64, dv=64, chunk=64, dt=1):
        return getattr(lib, fn)(*([None] * 5), B, H, N, dk, dv, chunk, dt, None)
    assert call(B=0) == 2
    assert call(N=-1) == 2
    assert call(chunk=0) == 2
    assert call(dt=5) == 3
    assert call(dk=300) == 4
    assert call(N=0) == 0   # empty: nothing copied, nothing launched
    assert call() == 1      # NULL tensors


def test_parallel_and_step_validation(lib):
    assert lib.ret_parallel(None, None, None, None, None, 1, 1, 4, 2000, 8, 0, None) == 4
    assert lib.ret_parallel(None, None, None, None, None, 1, 1, 4, 8, 8, 0, None) == 1
    assert lib.ret_parallel(None, None, None, None, None, 1, 0, 4, 8, 8, 0, None) == 2
    assert lib.ret_recurrent_step(None, None, None, None, None, None, 1, 1, 8, 8, 0, None) == 1
    assert lib.ret_recurrent_step(None, None, None, None, None, None, 1, 1, 5000, 8, 0, None) == 4
    assert lib.ret_recurrent_step(None, None, None, None, None, None, 1, 1, 8, 8, 2, None) == 3


@pytest.mark.parametrize("fn", ["ret_chunkwise_backward", "gated_ret_chunkwise_backward",
                                "ret_chunkwise_backward_host", "gated_ret_chunkwise_backward_host"])
def test_backward_validation(lib, fn):
    def call(B=1, H=1, N=8, dk=64, dv=64, chunk=64, dt=1):
        return getattr(lib, fn)(*([None] * 9), B, H, N, dk, dv, chunk, dt, None)
    assert call(B=0) == 2
    assert call(N=-3) == 2
    assert call(chunk=0) == 2
    assert call(dt=9) == 3
    assert call(dk=512) == 4
    assert call() == 1  # NULL tensors


def test_backward_launch_count_validation(lib):
    f = lib.ret_chunkwise_backward_launches
    assert f(0, 1, 8, 64, 64, 64, 1, 0, 1) == -1
    assert f(1, 1, 8, 300, 64, 64, 1, 0, 1) == -1
    assert f(1, 1, 0, 64, 64, 64, 1, 0, 1) == 0
    n_fixed, n_gated = f(1, 2, 100, 32, 40, 64, 0, 0, 1), f(1, 2, 100, 32, 40, 64, 0, 1, 1)
    assert n_fixed > 0 and n_gated == n_fixed + 2  # the reversed gates and the gate-gradient suffix sum
    assert f(1, 2, 100, 32, 40, 64, 0, 0, 0) == n_fixed - 1  # no decay gradient


def test_norm_gate_validation(lib):
    import ctypes
    f = lib.ret_msr_norm_gate
    p = lambda x: ctypes.c_void_p(x)
    args = lambda o, g, y, B=1, H=2, N=8, dv=64, eps=1e-5, dt=1: (o, g, y, B, H, N, dv, eps, dt, None)
    assert f(*args(None, None, None, dt=4)) == 3
    assert f(*args(None, None, None, B=0)) == 2
    assert f(*args(None, None, None, dv=0)) == 2
    assert f(*args(None, None, None, eps=-1.0)) == 2
    assert f(*args(None, None, None, eps=float("nan"))) == 2
    assert f(*args(None, None, None, N=0)) == 0  # empty: nothing to do, nothing launched
    assert f(*args(None, None, None)) == 1
    # overlaps are rejected before any launch (the addresses are never dereferenced)
    base = 1 << 40
    nbytes = 1 * 2 * 8 * 64 * 2
    assert f(*args(p(base), p(base + 4 * nbytes), p(base + 64))) == 4           # y inside o
    assert f(*args(p(base), p(base + 4 * nbytes), p(base + 4 * nbytes + 32))) == 4  # y inside gate, not gate


def test_bindings_refuse_host_tensors(lib):
    """The product path has no CPU fallback: host tensors are refused before the library is called."""
    import torch
    from linear_attention_ret_b200 import ret
    q = torch.zeros(1, 1, 4, 8)
    with pytest.raises(ValueError):
        ret.chunkwise_backward(q, q, q, torch.ones(1), q, 64)
    with pytest.raises(ValueError):
        ret.msr_norm_gate(q, torch.zeros(1, 4, 1, 8))
    with pytest.raises(ValueError):
        ret.ret_chunkwise(q, q, q, torch.ones(1), 64)


def test_host_bindings_check_shapes_before_the_library(lib):
    """The host-buffer calls check shapes and dtypes before any pointer reaches the library."""
    import torch
    from linear_attention_ret_b200 import ret
    q = torch.zeros(1, 2, 4, 8, dtype=torch.bfloat16)
    with pytest.raises(ValueError):
        ret.ret_chunkwise_host(q, q, q, torch.ones(3), 64)               # gamma [H] with H = 2
    with pytest.raises(ValueError):
        ret.gated_ret_chunkwise_host(q, q, q, torch.ones(1, 2, 5), 64)   # g [B, H, N]
    with pytest.raises(ValueError):
        ret.ret_chunkwise_host(q, q.float(), q, torch.ones(2), 64)       # k's dtype


def test_missing_library_fails_loudly(monkeypatch, tmp_path):
    """No fallback: without libret.so every call raises instead of computing anything on the host."""
    import torch
    from linear_attention_ret_b200 import ret
    monkeypatch.setattr(ret, "_lib", None)
    monkeypatch.setattr(ret, "LIB_PATH", str(tmp_path / "absent" / "libret.so"))
    with pytest.raises(RuntimeError, match="libret.so not found"):
        ret.load()
    with pytest.raises(RuntimeError, match="libret.so not found"):
        ret.chunkwise_launches(1, 1, 8, 64, 64, 64, torch.bfloat16)
