"""Sequence-parallel chunkwise (one sequence split across ranks, one exchange of states).

CPU (gloo, world sizes 2 and 3): the orchestration in seqpar.py -- segment order,
the all-gather of (U_r, log2 D_r), picking this rank's start state -- run with
the oracle standing in for the three kernels, against the oracle over the whole
sequence. GPU: the library's three kernels on one GPU, the ranks emulated one
after another (no kernel waits for another), against the oracle.
"""
import json
import os
import socket
import subprocess
import sys

import numpy as np
import pytest
import torch

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))

WORKER = r"""
import os, sys, json
sys.path.insert(0, os.environ["ROOT"])
import numpy as np, torch, torch.distributed as dist
from oracle import oracle as O
from linear_attention_ret_b200 import seqpar

class OracleOps:
    # the three steps computed by the fp64 oracle (test stand-in for the kernels)
    @staticmethod
    def state(k, v, decay, chunk, gated):
        B, H, N, dk = k.shape
        q0 = np.zeros((B, H, N, dk))
        if gated:
            _, U = O.gated_chunkwise(q0, k, v, decay, chunk)
            ld = decay.double().numpy().sum(axis=2) / np.log(2.0)
        else:
            _, U = O.ret_chunkwise(q0, k, v, decay, chunk)
            ld = np.broadcast_to(N * np.log2(decay.double().numpy()), (B, H)).copy()
        return torch.from_numpy(U), torch.from_numpy(ld)

    @staticmethod
    def prefix(seg_states, seg_log2_decay, state_in):
        x = torch.zeros_like(seg_states[0]) if state_in is None else state_in.clone()
        starts = []
        for r in range(seg_states.shape[0]):
            starts.append(x.clone())
            x = torch.exp2(seg_log2_decay[r])[..., None, None] * x + seg_states[r]
        return torch.stack(starts), x

    @staticmethod
    def chunkwise(q, k, v, decay, chunk, state_in, gated):
        f = O.gated_chunkwise if gated else O.ret_chunkwise
        return torch.from_numpy(f(q, k, v, decay, chunk, state_in=state_in)[0])

gated = os.environ["GATED"] == "1"
dist.init_process_group("gloo")
rank, world = dist.get_rank(), dist.get_world_size()
B, H, dk, dv, chunk = 1, 2, 6, 5, 4
lengths = [13, 9, 17][:world]
N = sum(lengths)
rng = np.random.default_rng(5)
q, k, v = rng.standard_normal((B, H, N, dk)), rng.standard_normal((B, H, N, dk)), rng.standard_normal((B, H, N, dv))
S0 = torch.from_numpy(rng.standard_normal((B, H, dk, dv)))
t0 = sum(lengths[:rank]); t1 = t0 + lengths[rank]
sl = lambda a: torch.from_numpy(np.ascontiguousarray(a[:, :, t0:t1]))
if gated:
    g = -np.abs(rng.standard_normal((B, H, N))) / 4.0
    decay = sl(g)
    want_o, want_s = O.gated_chunkwise(q, k, v, g, chunk, state_in=S0.numpy())
else:
    decay = torch.tensor([0.9, 0.97], dtype=torch.float64)
    want_o, want_s = O.ret_chunkwise(q, k, v, decay.numpy(), chunk, state_in=S0.numpy())
o, end = seqpar.sequence_parallel_chunkwise(sl(q), sl(k), sl(v), decay, chunk, gated=gated, state_in=S0,
                                            ops=OracleOps)
err_o = float(np.abs(o.numpy() - want_o[:, :, t0:t1]).max() / np.abs(want_o).max())
err_s = float(np.abs(end.numpy() - want_s).max() / np.abs(want_s).max())
print(json.dumps({"rank": rank, "err_o": err_o, "err_s": err_s}), flush=True)
dist.destroy_process_group()
"""


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("world", [2, 3])
def test_sequence_parallel_orchestration_gloo(world, gated):
    port = _free_port()
    procs = []
    for r in range(world):
        env = dict(os.environ, ROOT=ROOT, RANK=str(r), WORLD_SIZE=str(world), LOCAL_RANK=str(r),
                   MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), CUDA_VISIBLE_DEVICES="",
                   GATED="1" if gated else "0")
        procs.append(subprocess.Popen([sys.executable, "-c", WORKER], env=env, stdout=subprocess.PIPE,
                                      stderr=subprocess.PIPE, text=True))
    recs = []
    for p in procs:
        out, err = p.communicate(timeout=120)
        assert p.returncode == 0, err
        recs.append(json.loads(out.strip().splitlines()[-1]))
    assert sorted(r["rank"] for r in recs) == list(range(world))
    for r in recs:
        assert r["err_o"] < 1e-12 and r["err_s"] < 1e-12, r


# ------------------------------------------------------------------ GPU: the kernels, ranks emulated in turn

SEQPAR_CASES = [
    # B, H, segment lengths, dk, dv, dtype, gated
    (1, 4, [700, 500, 900], 256, 256, torch.bfloat16, False),   # tensor-core state pass (sub-segments)
    (2, 2, [300, 131], 128, 128, torch.bfloat16, False),
    (1, 2, [640, 700, 1], 128, 128, torch.bfloat16, True),      # gated, a one-token segment
    (1, 2, [50, 77], 32, 40, torch.float32, False),             # CUDA-core path
    (1, 2, [60, 45], 32, 40, torch.float32, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("B,H,lengths,dk,dv,dtype,gated", SEQPAR_CASES)
def test_segments_compose_on_gpu(cuda_lib, B, H, lengths, dk, dv, dtype, gated):
    from linear_attention_ret_b200 import inputs as I
    from oracle import oracle as O
    from tests.parity import assert_close, rel_l2, tol_for
    dev = "cuda:0"
    N = sum(lengths)
    gen = torch.Generator().manual_seed(N + dk)
    q, k, v = I.qkv(B, H, N, dk, dv, dtype, gen=gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    if gated:
        decay = I.gate(B, H, N, gen) * 4.0
        want_o, want_s = O.gated_chunkwise(q, k, v, decay, 64, state_in=S0)
    else:
        decay = torch.tensor([0.9, 0.96875, 0.999, 0.5][:H], dtype=torch.float32)
        want_o, want_s = O.ret_chunkwise(q, k, v, decay, 64, state_in=S0)
    bounds = np.cumsum([0] + lengths)
    seg = lambda t, r: t[:, :, bounds[r]:bounds[r + 1]].contiguous().to(dev)
    Us, lds = [], []
    for r in range(len(lengths)):
        d = seg(decay, r) if gated else decay.to(dev)
        U, ld = cuda_lib.chunkwise_state(seg(k, r), seg(v, r), d, 64, gated=gated)
        # each segment's own end state and decay against the oracle
        kk, vv = k[:, :, bounds[r]:bounds[r + 1]], v[:, :, bounds[r]:bounds[r + 1]]
        q0 = np.zeros(kk.shape)
        if gated:
            _, want_U = O.gated_chunkwise(q0, kk, vv, decay[:, :, bounds[r]:bounds[r + 1]], 64)
            want_ld = decay[:, :, bounds[r]:bounds[r + 1]].double().sum(2).numpy() / np.log(2.0)
        else:
            _, want_U = O.ret_chunkwise(q0, kk, vv, decay, 64)
            want_ld = np.broadcast_to(lengths[r] * np.log2(decay.double().numpy()), (B, H))
        assert_close(U, want_U, dtype, f"U segment {r}")
        np.testing.assert_allclose(ld.cpu().double().numpy(), want_ld, rtol=1e-5, atol=1e-5)
        Us.append(U)
        lds.append(ld)
    starts, end = cuda_lib.state_prefix(torch.stack(Us), torch.stack(lds), S0.to(dev))
    outs = []
    for r in range(len(lengths)):
        if gated:
            outs.append(cuda_lib.gated_ret_chunkwise(seg(q, r), seg(k, r), seg(v, r), seg(decay, r), 64,
                                                     state_in=starts[r].contiguous()))
        else:
            outs.append(cuda_lib.ret_chunkwise(seg(q, r), seg(k, r), seg(v, r), decay.to(dev), 64,
                                               state_in=starts[r].contiguous()))
    assert cuda_lib.last_device_error() == 0
    assert_close(torch.cat(outs, dim=2), want_o, dtype, "o over all segments")
    assert rel_l2(end, want_s) <= tol_for(dtype), "final state"


# ------------------------------------------------------------------ GPU: the product orchestration end to end

ORCH_CASES = [
    # B, H, N, dk, dv, dtype, gated
    (1, 4, 2100, 256, 256, torch.bfloat16, False),   # tensor-core path, split sequence inside the state pass
    (1, 2, 1333, 128, 128, torch.bfloat16, True),    # tensor-core gated path, ragged tail
    (1, 2, 111, 32, 40, torch.float32, False),       # CUDA-core path
    (1, 2, 97, 32, 40, torch.float32, True),
]


@pytest.mark.gpu
@pytest.mark.parametrize("with_group", [False, True])
@pytest.mark.parametrize("B,H,N,dk,dv,dtype,gated", ORCH_CASES)
def test_sequence_parallel_library_ops_on_gpu(cuda_lib, B, H, N, dk, dv, dtype, gated, with_group):
    """seqpar.sequence_parallel_chunkwise with the library's own kernels (LibraryOps) in one
    process: without a process group, and inside a one-rank NCCL group, where the
    all-gather of (U, log2 D) and the pick of this rank's start state run for real."""
    import torch.distributed as dist
    from linear_attention_ret_b200 import inputs as I
    from linear_attention_ret_b200 import seqpar
    from oracle import oracle as O
    from tests.parity import assert_close, rel_l2, tol_for
    dev = "cuda:0"
    gen = torch.Generator().manual_seed(N + dk + int(gated))
    q, k, v = I.qkv(B, H, N, dk, dv, dtype, gen=gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    if gated:
        decay = I.gate(B, H, N, gen) * 4.0
        want_o, want_s = O.gated_chunkwise(q, k, v, decay, 64, state_in=S0)
    else:
        decay = torch.tensor([0.9, 0.96875, 0.999, 0.5][:H], dtype=torch.float32)
        want_o, want_s = O.ret_chunkwise(q, k, v, decay, 64, state_in=S0)
    if with_group:
        dist.init_process_group("nccl", init_method=f"tcp://127.0.0.1:{_free_port()}", rank=0, world_size=1)
    try:
        o, end = seqpar.sequence_parallel_chunkwise(q.to(dev), k.to(dev), v.to(dev), decay.to(dev), 64,
                                                    gated=gated, state_in=S0.to(dev))
        torch.cuda.synchronize()
    finally:
        if with_group:
            dist.destroy_process_group()
    assert cuda_lib.last_device_error() == 0
    assert_close(o, want_o, dtype, "o")
    assert rel_l2(end, want_s) <= tol_for(dtype), "final state"
