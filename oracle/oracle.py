"""Python access to the fp64 retention oracle (oracle.c).

TEST INFRASTRUCTURE ONLY: only tests/, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this module. The product path (the
CUDA library in ``linear_attention_ret_b200``) never imports or calls it, and
this module imports nothing from the product package.

Every function takes numpy arrays (any float dtype; they are widened to fp64,
so the oracle sees exactly the values a GPU kernel reads) and returns fp64
numpy arrays. Shapes follow the pages' [..., N, d] convention with heads
leading: q, k [B, H, N, dk]; v [B, H, N, dv]; gamma [H]; g [B, H, N];
state [B, H, dk, dv].
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "oracle.c")
_BUILD_DIR = os.path.join(_HERE, "_build")
_LIB_PATH = os.path.join(_BUILD_DIR, "liboracle.so")
_lock = threading.Lock()
_lib = None

_P = ctypes.POINTER(ctypes.c_double)
_I = ctypes.c_int


def build(force: bool = False) -> str:
    """Compile oracle.c into oracle/_build/liboracle.so (gcc, -O2, OpenMP)."""
    os.makedirs(_BUILD_DIR, exist_ok=True)
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        cmd = ["gcc", "-O2", "-std=c11", "-fopenmp", "-fPIC", "-shared",
               "-Wall", "-Werror", _SRC, "-o", tmp, "-lm"]
        subprocess.run(cmd, check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            sig = {
                "oracle_decay_matrix": [ctypes.c_double, _I, _P],
                "oracle_ret_brute": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_ret_parallel": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_ret_recurrent": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_ret_recurrent_step": [_P, _P, _P, _P, _P, _P, _I, _I, _I, _I],
                "oracle_ret_chunkwise": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I],
                "oracle_gated_brute": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_gated_parallel": [_P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_gated_recurrent": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_gated_chunkwise": [_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I],
                "oracle_ret_backward": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_gated_backward": [_P, _P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I],
                "oracle_msr_norm_gate": [_P, _P, _P, _I, _I, _I, _I, ctypes.c_double],
            }
            for name, argtypes in sig.items():
                fn = getattr(lib, name)
                fn.argtypes = argtypes
                fn.restype = _I
            lib.oracle_max_threads.argtypes = []
            lib.oracle_max_threads.restype = _I
            lib.oracle_set_threads.argtypes = [_I]
            lib.oracle_set_threads.restype = None
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    """Widen to a C-contiguous fp64 array (accepts numpy or torch CPU tensors)."""
    if a is None:
        return None
    if hasattr(a, "detach"):  # torch tensor
        a = a.detach().to("cpu")
        import torch  # local: torch is only needed when a tensor is passed
        a = a.to(torch.float64).numpy()
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _ptr(a):
    return None if a is None else a.ctypes.data_as(_P)


def _check(rc: int, name: str):
    if rc != 0:
        raise ValueError(f"{name} failed with code {rc}")


def _dims(q, v):
    B, H, N, dk = q.shape
    dv = v.shape[-1]
    return B, H, N, dk, dv


def max_threads() -> int:
    return int(_load().oracle_max_threads())


def set_threads(n: int) -> None:
    _load().oracle_set_threads(int(n))


def decay_matrix(gamma: float, N: int) -> np.ndarray:
    D = np.empty((N, N), dtype=np.float64)
    _check(_load().oracle_decay_matrix(float(gamma), int(N), _ptr(D)), "decay_matrix")
    return D


def ret_brute(q, k, v, gamma):
    q, k, v, gamma = map(_f64, (q, k, v, gamma))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    _check(_load().oracle_ret_brute(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(o), B, H, N, dk, dv),
           "ret_brute")
    return o


def ret_parallel(q, k, v, gamma):
    q, k, v, gamma = map(_f64, (q, k, v, gamma))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    _check(_load().oracle_ret_parallel(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(o), B, H, N, dk, dv),
           "ret_parallel")
    return o


def ret_recurrent(q, k, v, gamma, state_in=None):
    """Returns (o, final_state)."""
    q, k, v, gamma, s_in = map(_f64, (q, k, v, gamma, state_in))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    s_out = np.empty((B, H, dk, dv))
    _check(_load().oracle_ret_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(s_in), _ptr(s_out),
                                        _ptr(o), B, H, N, dk, dv), "ret_recurrent")
    return o, s_out


def ret_recurrent_step(q, k, v, gamma, state):
    """One decode step. q, k [B, H, dk]; v [B, H, dv]; returns (o [B, H, dv], new_state)."""
    q, k, v, gamma = map(_f64, (q, k, v, gamma))
    S = _f64(state).copy()
    B, H, dk = q.shape
    dv = v.shape[-1]
    o = np.empty((B, H, dv))
    _check(_load().oracle_ret_recurrent_step(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(S), _ptr(o),
                                             B, H, dk, dv), "ret_recurrent_step")
    return o, S


def ret_chunkwise(q, k, v, gamma, chunk, state_in=None):
    """Returns (o, final_state)."""
    q, k, v, gamma, s_in = map(_f64, (q, k, v, gamma, state_in))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    s_out = np.empty((B, H, dk, dv))
    _check(_load().oracle_ret_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(s_in), _ptr(s_out),
                                        _ptr(o), B, H, N, dk, dv, int(chunk)), "ret_chunkwise")
    return o, s_out


def gated_brute(q, k, v, g):
    q, k, v, g = map(_f64, (q, k, v, g))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    _check(_load().oracle_gated_brute(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), B, H, N, dk, dv),
           "gated_brute")
    return o


def gated_parallel(q, k, v, g):
    q, k, v, g = map(_f64, (q, k, v, g))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    _check(_load().oracle_gated_parallel(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(o), B, H, N, dk, dv),
           "gated_parallel")
    return o


def gated_recurrent(q, k, v, g, state_in=None):
    q, k, v, g, s_in = map(_f64, (q, k, v, g, state_in))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    s_out = np.empty((B, H, dk, dv))
    _check(_load().oracle_gated_recurrent(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(s_in), _ptr(s_out),
                                          _ptr(o), B, H, N, dk, dv), "gated_recurrent")
    return o, s_out


def gated_recurrent_step(q, k, v, g, state):
    """One gated decode step (Gated RetNet page, recurrent_gate_retention): the gated
    recurrent form over a single token, S = exp(g) S + k^T v, o = q S (updated state).
    q, k [B, H, dk]; v [B, H, dv]; g [B, H]; returns (o [B, H, dv], new_state)."""
    o, s = gated_recurrent(_f64(q)[:, :, None], _f64(k)[:, :, None], _f64(v)[:, :, None], _f64(g)[:, :, None], state)
    return o[:, :, 0], s


def gated_chunkwise(q, k, v, g, chunk, state_in=None):
    q, k, v, g, s_in = map(_f64, (q, k, v, g, state_in))
    B, H, N, dk, dv = _dims(q, v)
    o = np.empty((B, H, N, dv))
    s_out = np.empty((B, H, dk, dv))
    _check(_load().oracle_gated_chunkwise(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(s_in), _ptr(s_out),
                                          _ptr(o), B, H, N, dk, dv, int(chunk)), "gated_chunkwise")
    return o, s_out


def ret_backward(q, k, v, gamma, do):
    """Gradients of L = sum dO . O (zero initial state) by definition: (dq, dk, dv, dgamma)."""
    q, k, v, gamma, do = map(_f64, (q, k, v, gamma, do))
    B, H, N, dk, dv = _dims(q, v)
    dq, dkk, dvv = np.empty_like(q), np.empty_like(k), np.empty_like(v)
    dgam = np.empty(H)
    _check(_load().oracle_ret_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(gamma), _ptr(do), _ptr(dq), _ptr(dkk),
                                       _ptr(dvv), _ptr(dgam), B, H, N, dk, dv), "ret_backward")
    return dq, dkk, dvv, dgam


def gated_backward(q, k, v, g, do):
    """Gated gradients of L = sum dO . O (zero initial state) by definition: (dq, dk, dv, dg)."""
    q, k, v, g, do = map(_f64, (q, k, v, g, do))
    B, H, N, dk, dv = _dims(q, v)
    dq, dkk, dvv, dg = np.empty_like(q), np.empty_like(k), np.empty_like(v), np.empty_like(g)
    _check(_load().oracle_gated_backward(_ptr(q), _ptr(k), _ptr(v), _ptr(g), _ptr(do), _ptr(dq), _ptr(dkk),
                                         _ptr(dvv), _ptr(dg), B, H, N, dk, dv), "gated_backward")
    return dq, dkk, dvv, dg


def msr_norm_gate(o, gate, eps=1e-5):
    """Multi-scale retention output epilogue (explainer page 3.2; Gated RetNet page,
    GateRetention's subln and swish gate): y[b, n, h] = swish(gate[b, n, h]) *
    RMSNorm(o[b, h, n]) over dv, no affine weights. o [B, H, N, dv]; gate [B, N, H, dv];
    returns y [B, N, H, dv]."""
    o, gate = _f64(o), _f64(gate)
    B, H, N, dv = o.shape
    if gate.shape != (B, N, H, dv):
        raise ValueError(f"gate shape {gate.shape} != {(B, N, H, dv)}")
    y = np.empty_like(gate)
    _check(_load().oracle_msr_norm_gate(_ptr(o), _ptr(gate), _ptr(y), B, H, N, dv, float(eps)), "msr_norm_gate")
    return y
