"""Thin Python binding of libret.so, the C ABI declared in include/ret.h.

Argument marshalling only: shape and dtype checks, output allocation with
torch (device memory is plumbing), and the call through ctypes. Every step of
retention runs in the library's CUDA kernels; there is no fallback. If the
library is missing, load() raises.

Names match the C ABI: ret_parallel, ret_chunkwise, ret_recurrent_step,
gated_ret_chunkwise. Tensors are CUDA, contiguous, heads leading:
q, k [B, H, N, dk]; v [B, H, N, dv]; gamma [H] fp32; g [B, H, N] fp32;
state [B, H, dk, dv] fp32. q, k, v share one dtype (float32 or bfloat16).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_PKG = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_PKG, "libret.so")

RET_F32, RET_BF16 = 0, 1
STATUS = {0: "RET_OK", 1: "RET_ERR_NULL", 2: "RET_ERR_SHAPE", 3: "RET_ERR_DTYPE", 4: "RET_ERR_UNSUPPORTED",
          5: "RET_ERR_CUDA", 6: "RET_ERR_TIMEOUT", 7: "RET_ERR_ALIGN", 8: "RET_ERR_SCRATCH"}
# every symbol include/ret.h declares
SYMBOLS = ("ret_parallel", "ret_chunkwise", "ret_recurrent_step", "gated_ret_chunkwise", "ret_status_str",
           "ret_last_device_error", "ret_chunkwise_path", "ret_chunkwise_launches", "ret_version",
           "ret_chunkwise_noalloc", "ret_selftest_wait_timeout", "gated_ret_recurrent_step",
           "ret_chunkwise_state", "gated_ret_chunkwise_state", "ret_state_prefix", "ret_chunkwise_state_launches",
           "ret_chunkwise_backward", "gated_ret_chunkwise_backward", "ret_chunkwise_backward_launches",
           "ret_msr_norm_gate", "ret_chunkwise_noalloc_scratch_bytes", "ret_chunkwise_host",
           "gated_ret_chunkwise_host", "ret_chunkwise_backward_host", "gated_ret_chunkwise_backward_host")

_lock = threading.Lock()
_lib = None

_vp = ctypes.c_void_p
_i = ctypes.c_int


class RetError(RuntimeError):
    def __init__(self, fn: str, code: int, msg: str):
        super().__init__(f"{fn}: {STATUS.get(code, code)} ({msg})")
        self.code = code


def load(path: str | None = None) -> ctypes.CDLL:
    """Load libret.so (built in-tree by linear_attention_ret_b200.build)."""
    global _lib
    with _lock:
        if _lib is not None:
            return _lib
        p = path or LIB_PATH
        if not os.path.exists(p):
            raise RuntimeError(f"libret.so not found at {p}: build it with "
                               "`python -m linear_attention_ret_b200.build`")
        lib = ctypes.CDLL(p)
        lib.ret_parallel.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _vp]
        lib.ret_chunkwise.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
        lib.gated_ret_chunkwise.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
        lib.ret_chunkwise_noalloc.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
        lib.ret_recurrent_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
        lib.gated_ret_recurrent_step.argtypes = [_vp, _vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
        lib.ret_chunkwise_state.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
        lib.gated_ret_chunkwise_state.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _i, _i, _vp]
        lib.ret_state_prefix.argtypes = [_vp, _vp, _vp, _vp, _vp, _i, _i, _i, _i, _i, _vp]
        lib.ret_chunkwise_state_launches.argtypes = [_i, _i, _i, _i, _i, _i, _i]
        lib.ret_chunkwise_backward_launches.argtypes = [_i, _i, _i, _i, _i, _i, _i, _i, _i]
        for fn in ("ret_chunkwise_host", "gated_ret_chunkwise_host"):
            getattr(lib, fn).argtypes = [_vp] * 5 + [_i] * 7 + [_vp]
            getattr(lib, fn).restype = _i
        lib.ret_msr_norm_gate.argtypes = [_vp, _vp, _vp, _i, _i, _i, _i, ctypes.c_float, _i, _vp]
        lib.ret_msr_norm_gate.restype = _i
        for fn in ("ret_chunkwise_backward", "gated_ret_chunkwise_backward", "ret_chunkwise_backward_host",
                   "gated_ret_chunkwise_backward_host"):
            getattr(lib, fn).argtypes = [_vp] * 9 + [_i] * 7 + [_vp]
            getattr(lib, fn).restype = _i
        lib.ret_chunkwise_state_launches.restype = _i
        for fn in ("ret_parallel", "ret_chunkwise", "gated_ret_chunkwise", "ret_recurrent_step",
                   "ret_chunkwise_noalloc", "gated_ret_recurrent_step", "ret_chunkwise_state",
                   "gated_ret_chunkwise_state", "ret_state_prefix"):
            getattr(lib, fn).restype = _i
        lib.ret_status_str.argtypes = [_i]
        lib.ret_status_str.restype = ctypes.c_char_p
        lib.ret_last_device_error.argtypes = [_vp]
        lib.ret_last_device_error.restype = _i
        lib.ret_selftest_wait_timeout.argtypes = [ctypes.c_uint, _vp]
        lib.ret_selftest_wait_timeout.restype = _i
        lib.ret_chunkwise_path.argtypes = [_i, _i, _i, _i]
        lib.ret_chunkwise_path.restype = _i
        lib.ret_chunkwise_launches.argtypes = [_i, _i, _i, _i, _i, _i, _i]
        lib.ret_chunkwise_launches.restype = _i
        lib.ret_chunkwise_noalloc_scratch_bytes.argtypes = [_i] * 8
        lib.ret_chunkwise_noalloc_scratch_bytes.restype = ctypes.c_longlong
        lib.ret_version.argtypes = []
        lib.ret_version.restype = ctypes.c_char_p
        _lib = lib
        return lib


def _check(fn: str, code: int):
    if code != 0:
        raise RetError(fn, code, load().ret_status_str(code).decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return RET_F32
    if t.dtype == torch.bfloat16:
        return RET_BF16
    raise TypeError(f"unsupported dtype {t.dtype}; use float32 or bfloat16")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _cuda(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous CUDA tensors")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise ValueError(f"tensors must be on one device, got {dev} and {t.device}")


def _host(*ts):
    for t in ts:
        if t.is_cuda or not t.is_contiguous():
            raise ValueError("tensors must be contiguous host (CPU) tensors")


def _expect(name, t, shape, dtype=None):
    """Shape (and dtype) every tensor must have given the leading one, checked before any
    pointer reaches the library: a wrong size there would read past an allocation."""
    if t is None:
        return
    if tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name} must have shape {tuple(shape)}, got {tuple(t.shape)}")
    if dtype is not None and t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")


def _rank(name, t, n):
    if t.dim() != n:
        raise ValueError(f"{name} must have {n} dimensions, got shape {tuple(t.shape)}")


def _seq_args(q, k, v, decay, gated, o=None, state_in=None, state_out=None):
    """q, k [B, H, N, dk]; v, o [B, H, N, dv] (q's dtype); gamma [H] or g [B, H, N] fp32;
    states [B, H, dk, dv] fp32. Returns (B, H, N, dk, dv)."""
    _rank("q", q, 4)
    _rank("v", v, 4)
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (B, H, N, dk), q.dtype)
    _expect("v", v, (B, H, N, dv), q.dtype)
    _expect("g" if gated else "gamma", decay, (B, H, N) if gated else (H,), torch.float32)
    _expect("o", o, (B, H, N, dv), q.dtype)
    _expect("state_in", state_in, (B, H, dk, dv), torch.float32)
    _expect("state_out", state_out, (B, H, dk, dv), torch.float32)
    return B, H, N, dk, dv


def _step_args(q, k, v, decay, state, o, gated):
    """q, k [B, H, dk]; v, o [B, H, dv]; gamma [H] or g [B, H] fp32; state [B, H, dk, dv] fp32."""
    _rank("q", q, 3)
    _rank("v", v, 3)
    B, H, dk = q.shape
    dv = v.shape[-1]
    _expect("k", k, (B, H, dk), q.dtype)
    _expect("v", v, (B, H, dv), q.dtype)
    _expect("g" if gated else "gamma", decay, (B, H) if gated else (H,), torch.float32)
    _expect("state", state, (B, H, dk, dv), torch.float32)
    _expect("o", o, (B, H, dv), q.dtype)
    return B, H, dk, dv


def ret_parallel(q, k, v, gamma, o=None, stream=None):
    """O = (Q K^T (.) D) V. Returns o [B, H, N, dv] (dtype of q)."""
    B, H, N, dk, dv = _seq_args(q, k, v, gamma, False, o)
    o = torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device) if o is None else o
    _cuda(q, k, v, gamma, o)
    _check("ret_parallel", load().ret_parallel(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(o),
                                               B, H, N, dk, dv, _dt(q), _stream(stream)))
    return o


def ret_chunkwise(q, k, v, gamma, chunk, state_in=None, state_out=None, o=None, stream=None):
    """Chunkwise retention. Returns o; writes the final state into state_out if given."""
    B, H, N, dk, dv = _seq_args(q, k, v, gamma, False, o, state_in, state_out)
    o = torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device) if o is None else o
    _cuda(q, k, v, gamma, o, state_in, state_out)
    _check("ret_chunkwise", load().ret_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(o),
                                                 _ptr(state_in), _ptr(state_out), B, H, N, dk, dv, int(chunk),
                                                 _dt(q), _stream(stream)))
    return o


def ret_chunkwise_noalloc(q, k, v, gamma, chunk, state_in=None, state_out=None, o=None, stream=None):
    """ret_chunkwise without device allocation by the library: scratch comes from a
    fixed 16 MiB buffer inside libret.so (see include/ret.h). Returns o."""
    B, H, N, dk, dv = _seq_args(q, k, v, gamma, False, o, state_in, state_out)
    o = torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device) if o is None else o
    _cuda(q, k, v, gamma, o, state_in, state_out)
    _check("ret_chunkwise_noalloc", load().ret_chunkwise_noalloc(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(o),
                                                                 _ptr(state_in), _ptr(state_out), B, H, N, dk, dv,
                                                                 int(chunk), _dt(q), _stream(stream)))
    return o


def gated_ret_chunkwise(q, k, v, g, chunk, state_in=None, state_out=None, o=None, stream=None):
    """Gated chunkwise retention (per-token log-decay g). Returns o."""
    B, H, N, dk, dv = _seq_args(q, k, v, g, True, o, state_in, state_out)
    o = torch.empty(B, H, N, dv, dtype=q.dtype, device=q.device) if o is None else o
    _cuda(q, k, v, g, o, state_in, state_out)
    _check("gated_ret_chunkwise", load().gated_ret_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o),
                                                             _ptr(state_in), _ptr(state_out), B, H, N, dk, dv,
                                                             int(chunk), _dt(q), _stream(stream)))
    return o


def _chunkwise_host(name, q, k, v, decay, chunk, o, gated, stream, sync):
    B, H, N, dk, dv = _seq_args(q, k, v, decay, gated, o)
    if o is None:
        o = torch.empty(B, H, N, dv, dtype=q.dtype, pin_memory=q.is_pinned())
    _host(q, k, v, decay, o)
    s = torch.cuda.current_stream() if stream is None else stream
    _check(name, getattr(load(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(o), B, H, N, dk, dv,
                                       int(chunk), _dt(q), ctypes.c_void_p(s.cuda_stream)))
    if sync:
        s.synchronize()
    return o


def ret_chunkwise_host(q, k, v, gamma, chunk, o=None, stream=None, sync=True):
    """ret_chunkwise on host (CPU) tensors, pinned for copy/compute overlap: the library copies
    the inputs in, computes and copies o back, pipelined over groups of heads, on the current
    CUDA device. Returns o once the stream has completed (sync=False: once enqueued)."""
    return _chunkwise_host("ret_chunkwise_host", q, k, v, gamma, chunk, o, False, stream, sync)


def gated_ret_chunkwise_host(q, k, v, g, chunk, o=None, stream=None, sync=True):
    """gated_ret_chunkwise on host (CPU) tensors; as ret_chunkwise_host."""
    return _chunkwise_host("gated_ret_chunkwise_host", q, k, v, g, chunk, o, True, stream, sync)


def ret_recurrent_step(q, k, v, gamma, state, o=None, stream=None):
    """One decode step; updates state [B, H, dk, dv] in place and returns o [B, H, dv]."""
    B, H, dk, dv = _step_args(q, k, v, gamma, state, o, False)
    o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device) if o is None else o
    _cuda(q, k, v, gamma, state, o)
    _check("ret_recurrent_step", load().ret_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(state),
                                                           _ptr(o), B, H, dk, dv, _dt(q), _stream(stream)))
    return o


def gated_ret_recurrent_step(q, k, v, g, state, o=None, stream=None):
    """One gated decode step with log-decay g [B, H] (fp32); updates state in place, returns o [B, H, dv]."""
    B, H, dk, dv = _step_args(q, k, v, g, state, o, True)
    o = torch.empty(B, H, dv, dtype=q.dtype, device=q.device) if o is None else o
    _cuda(q, k, v, g, state, o)
    _check("gated_ret_recurrent_step", load().gated_ret_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(g),
                                                                       _ptr(state), _ptr(o), B, H, dk, dv, _dt(q),
                                                                       _stream(stream)))
    return o


def chunkwise_state(k, v, decay, chunk, gated=False, state_out=None, log2_decay=None, stream=None):
    """End state U [B, H, dk, dv] of a segment from a zero start and log2 of its total decay
    [B, H] (decay: gamma [H], or g [B, H, N] with gated=True). Returns (U, log2_decay)."""
    B, H, N, dk, dv = _seq_args(k, k, v, decay, gated, None, None, state_out)
    _expect("log2_decay", log2_decay, (B, H), torch.float32)
    state_out = torch.empty(B, H, dk, dv, dtype=torch.float32, device=k.device) if state_out is None else state_out
    log2_decay = torch.empty(B, H, dtype=torch.float32, device=k.device) if log2_decay is None else log2_decay
    _cuda(k, v, decay, state_out, log2_decay)
    name = "gated_ret_chunkwise_state" if gated else "ret_chunkwise_state"
    _check(name, getattr(load(), name)(_ptr(k), _ptr(v), _ptr(decay), _ptr(state_out), _ptr(log2_decay),
                                       B, H, N, dk, dv, int(chunk), _dt(k), _stream(stream)))
    return state_out, log2_decay


def state_prefix(seg_states, seg_log2_decay, state_in=None, stream=None):
    """Start states [R, B, H, dk, dv] of R consecutive segments and the state after all of
    them, from their end states U [R, B, H, dk, dv] and log2 decays [R, B, H]."""
    _rank("seg_states", seg_states, 5)
    R, B, H, dk, dv = seg_states.shape
    _expect("seg_states", seg_states, (R, B, H, dk, dv), torch.float32)
    _expect("seg_log2_decay", seg_log2_decay, (R, B, H), torch.float32)
    _expect("state_in", state_in, (B, H, dk, dv), torch.float32)
    starts = torch.empty_like(seg_states)
    end = torch.empty(B, H, dk, dv, dtype=torch.float32, device=seg_states.device)
    _cuda(seg_states, seg_log2_decay, state_in, starts, end)
    _check("ret_state_prefix", load().ret_state_prefix(_ptr(seg_states), _ptr(seg_log2_decay), _ptr(state_in),
                                                       _ptr(starts), _ptr(end), R, B, H, dk, dv, _stream(stream)))
    return starts, end


def chunkwise_backward(q, k, v, decay, dout, chunk, gated=False, ddecay=True, stream=None):
    """Gradients of sum(dout * o) for o = ret_chunkwise(q, k, v, decay) (gated=True:
    gated_ret_chunkwise with g = decay) from a zero initial state. Returns
    (dq, dk, dv, ddecay) with ddecay = dgamma [H] or dg [B, H, N] (fp32), or None."""
    B, H, N, dk, dv = _seq_args(q, k, v, decay, gated)
    _expect("dout", dout, (B, H, N, dv), q.dtype)
    dq, dkk, dvv = torch.empty_like(q), torch.empty_like(k), torch.empty_like(v)
    dd = None
    if ddecay:
        dd = torch.empty(B, H, N, dtype=torch.float32, device=q.device) if gated else \
            torch.empty(H, dtype=torch.float32, device=q.device)
    _cuda(q, k, v, decay, dout, dq, dkk, dvv, dd)
    name = "gated_ret_chunkwise_backward" if gated else "ret_chunkwise_backward"
    _check(name, getattr(load(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq), _ptr(dkk),
                                       _ptr(dvv), _ptr(dd), B, H, N, dk, dv, int(chunk), _dt(q), _stream(stream)))
    return dq, dkk, dvv, dd


def chunkwise_backward_host(q, k, v, decay, dout, chunk, gated=False, ddecay=True, out=None, stream=None, sync=True):
    """chunkwise_backward on host (CPU) tensors, pinned for copy/compute overlap: the library
    copies the inputs in and the gradients out, pipelined over groups of heads, on the current
    CUDA device. out: optional (dq, dk, dv, ddecay) host tensors to write. Returns them once the
    stream has completed (sync=False: once enqueued)."""
    B, H, N, dk, dv = _seq_args(q, k, v, decay, gated)
    _expect("dout", dout, (B, H, N, dv), q.dtype)
    pin = q.is_pinned()
    if out is None:
        dd = None
        if ddecay:
            dd = torch.empty((B, H, N) if gated else (H,), dtype=torch.float32, pin_memory=pin)
        out = (torch.empty(B, H, N, dk, dtype=q.dtype, pin_memory=pin),
               torch.empty(B, H, N, dk, dtype=q.dtype, pin_memory=pin),
               torch.empty(B, H, N, dv, dtype=q.dtype, pin_memory=pin), dd)
    dq, dkk, dvv, dd = out
    _expect("dq", dq, (B, H, N, dk), q.dtype)
    _expect("dk", dkk, (B, H, N, dk), q.dtype)
    _expect("dv", dvv, (B, H, N, dv), q.dtype)
    _expect("ddecay", dd, (B, H, N) if gated else (H,), torch.float32)
    _host(*(t for t in (q, k, v, decay, dout, dq, dkk, dvv, dd) if t is not None))
    s = torch.cuda.current_stream() if stream is None else stream
    name = "gated_ret_chunkwise_backward_host" if gated else "ret_chunkwise_backward_host"
    _check(name, getattr(load(), name)(_ptr(q), _ptr(k), _ptr(v), _ptr(decay), _ptr(dout), _ptr(dq), _ptr(dkk),
                                       _ptr(dvv), _ptr(dd), B, H, N, dk, dv, int(chunk), _dt(q),
                                       ctypes.c_void_p(s.cuda_stream)))
    if sync:
        s.synchronize()
    return dq, dkk, dvv, dd


def msr_norm_gate(o, gate, eps: float = 1e-5, y=None, stream=None):
    """Multi-scale retention output epilogue: y[b, n, h] = swish(gate[b, n, h]) * RMSNorm(o[b, h, n])
    over dv (no affine weights). o [B, H, N, dv]; gate [B, N, H, dv] (same dtype);
    returns y [B, N, H, dv] (may be `gate` itself for an in-place update)."""
    _rank("o", o, 4)
    B, H, N, dv = o.shape
    if tuple(gate.shape) != (B, N, H, dv):
        raise ValueError(f"gate must be [B, N, H, dv] = {(B, N, H, dv)}, got {tuple(gate.shape)}")
    if y is None:
        y = torch.empty_like(gate)
    if gate.dtype != o.dtype or y.dtype != o.dtype or tuple(y.shape) != tuple(gate.shape):
        raise ValueError("o, gate and y must share one dtype; y has gate's shape")
    _cuda(o, gate, y)
    _check("ret_msr_norm_gate", load().ret_msr_norm_gate(_ptr(o), _ptr(gate), _ptr(y), B, H, N, dv, float(eps), _dt(o),
                                                         _stream(stream)))
    return y


def last_device_error(stream=None) -> int:
    return int(load().ret_last_device_error(_stream(stream)))


def selftest_wait_timeout(limit_us: int, stream=None) -> int:
    """Launch the failure-path self-test (a bounded wait that runs out); returns the launch status."""
    return int(load().ret_selftest_wait_timeout(limit_us, _stream(stream)))


def chunkwise_launches(B: int, H: int, N: int, dk: int, dv: int, chunk: int, dtype: torch.dtype) -> int:
    return int(load().ret_chunkwise_launches(B, H, N, dk, dv, chunk, RET_BF16 if dtype == torch.bfloat16 else RET_F32))


def chunkwise_state_launches(B: int, H: int, N: int, dk: int, dv: int, chunk: int, dtype: torch.dtype) -> int:
    return int(load().ret_chunkwise_state_launches(B, H, N, dk, dv, chunk,
                                                   RET_BF16 if dtype == torch.bfloat16 else RET_F32))


def chunkwise_backward_launches(B: int, H: int, N: int, dk: int, dv: int, chunk: int, dtype: torch.dtype,
                                gated: bool = False, ddecay: bool = True) -> int:
    return int(load().ret_chunkwise_backward_launches(B, H, N, dk, dv, chunk,
                                                      RET_BF16 if dtype == torch.bfloat16 else RET_F32,
                                                      int(gated), int(ddecay)))


def chunkwise_path(dk: int, dv: int, chunk: int, dtype: torch.dtype) -> int:
    return int(load().ret_chunkwise_path(dk, dv, chunk, RET_BF16 if dtype == torch.bfloat16 else RET_F32))


def noalloc_scratch_bytes(B: int, H: int, N: int, dk: int, dv: int, chunk: int, dtype: torch.dtype,
                          in_place: bool = False) -> int:
    """Bytes of the fixed buffer ret_chunkwise_noalloc would use on the current device (0: none,
    -1: invalid sizes); above NOALLOC_SCRATCH_BYTES the call is rejected with RET_ERR_SCRATCH."""
    return int(load().ret_chunkwise_noalloc_scratch_bytes(B, H, N, dk, dv, chunk,
                                                          RET_BF16 if dtype == torch.bfloat16 else RET_F32,
                                                          int(in_place)))


NOALLOC_SCRATCH_BYTES = 16 << 20  # RET_NOALLOC_SCRATCH_BYTES in include/ret.h
