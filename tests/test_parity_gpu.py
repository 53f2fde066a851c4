"""GPU parity: the CUDA library (through its C ABI) against the fp64 oracle.

Small cases compare every output element; the full-size workloads run in the
same launch configuration as bench.py and are compared on sampled heads, each
of which the oracle computes independently (heads do not interact).
"""
import numpy as np
import pytest
import torch

from linear_attention_ret_b200 import inputs as I
from oracle import oracle as O
from tests.parity import TOL_BF16, TOL_F32, assert_close, rel_l2, tol_for

pytestmark = pytest.mark.gpu

DEV = "cuda:0"


def _dev(*ts):
    return [None if t is None else t.to(DEV).contiguous() for t in ts]


def _rand_inputs(B, H, N, dk, dv, dtype, seed):
    return I.qkv(B, H, N, dk, dv, dtype, seed=seed)


# ------------------------------------------------------------------ tiny fp32 config, all forms

def test_tiny_config_all_forms(cuda_lib):
    cfg = I.CONFIGS["tiny"]
    x = I.config_inputs(cfg)
    q, k, v, gam = _dev(x["q"], x["k"], x["v"], x["gamma"])
    # parallel form
    o_par = cuda_lib.ret_parallel(q, k, v, gam)
    assert_close(o_par, O.ret_parallel(x["q"], x["k"], x["v"], x["gamma"]), torch.float32, "parallel")
    # chunkwise form, chunk 32, with the final state
    s_out = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, device=DEV)
    o_chk = cuda_lib.ret_chunkwise(q, k, v, gam, cfg.chunk, state_out=s_out)
    want_o, want_s = O.ret_chunkwise(x["q"], x["k"], x["v"], x["gamma"], cfg.chunk)
    assert_close(o_chk, want_o, torch.float32, "chunkwise")
    assert_close(s_out, want_s, torch.float32, "chunkwise state")
    # recurrent form: N single-token steps from a zero state
    S = torch.zeros(cfg.B, cfg.H, cfg.dk, cfg.dv, device=DEV)
    outs = [cuda_lib.ret_recurrent_step(q[:, :, t].contiguous(), k[:, :, t].contiguous(),
                                        v[:, :, t].contiguous(), gam, S) for t in range(cfg.N)]
    o_rec = torch.stack(outs, dim=2)
    want_rec, want_srec = O.ret_recurrent(x["q"], x["k"], x["v"], x["gamma"])
    assert_close(o_rec, want_rec, torch.float32, "recurrent")
    assert_close(S, want_srec, torch.float32, "recurrent state")
    assert cuda_lib.last_device_error() == 0


# ------------------------------------------------------------------ chunkwise, small shapes, all elements

CHUNK_CASES = [
    # B, H, N, dk, dv, chunk, dtype
    (1, 4, 77, 48, 40, 16, torch.float32),    # ragged tail, odd dims
    (2, 2, 130, 32, 96, 64, torch.float32),
    (1, 2, 150, 64, 96, 32, torch.bfloat16),  # CUDA-core bf16
    (2, 3, 200, 64, 128, 64, torch.bfloat16),
    (1, 2, 257, 128, 256, 64, torch.bfloat16),
    (1, 2, 320, 256, 128, 128, torch.bfloat16),
    (1, 1, 64, 256, 512, 64, torch.bfloat16),
    (1, 2, 1, 64, 128, 64, torch.bfloat16),    # single token
]


def _gammas_with_edges(H):
    base = [0.0, 0.5, 0.96875, 1.0, 0.9, 0.999]
    return torch.tensor([base[h % len(base)] for h in range(H)], dtype=torch.float32)


@pytest.mark.parametrize("B,H,N,dk,dv,chunk,dtype", CHUNK_CASES)
def test_chunkwise_matches_oracle(cuda_lib, B, H, N, dk, dv, chunk, dtype):
    q, k, v = _rand_inputs(B, H, N, dk, dv, dtype, seed=N + dk)
    gam = _gammas_with_edges(H)
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(3)) * 0.05
    qd, kd, vd, gd, S0d = _dev(q, k, v, gam, S0)
    s_out = torch.empty_like(S0d)
    o = cuda_lib.ret_chunkwise(qd, kd, vd, gd, chunk, state_in=S0d, state_out=s_out)
    want_o, want_s = O.ret_chunkwise(q, k, v, gam, chunk, state_in=S0)
    assert_close(o, want_o, dtype, "o")
    assert_close(s_out, want_s, dtype, "state")


@pytest.mark.parametrize("B,H,N,dk,dv,chunk,dtype", CHUNK_CASES)
def test_gated_chunkwise_matches_oracle(cuda_lib, B, H, N, dk, dv, chunk, dtype):
    gen = torch.Generator().manual_seed(N * 7 + dv)
    q, k, v = I.qkv(B, H, N, dk, dv, dtype, gen=gen)
    g = I.gate(B, H, N, gen) * 4.0  # stronger decay than the workload, to exercise the weights
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    qd, kd, vd, gdv, S0d = _dev(q, k, v, g, S0)
    s_out = torch.empty_like(S0d)
    o = cuda_lib.gated_ret_chunkwise(qd, kd, vd, gdv, chunk, state_in=S0d, state_out=s_out)
    want_o, want_s = O.gated_chunkwise(q, k, v, g, chunk, state_in=S0)
    assert_close(o, want_o, dtype, "o")
    assert_close(s_out, want_s, dtype, "state")


def _steep_and_mild_gates(B, H, N, gen):
    """Gates whose in-chunk cumulative log2-decay stays far inside +-100 on some heads and
    chunks and passes it on others (about -9 per token), with both kinds inside one head."""
    g = I.gate(B, H, N, gen)
    g[:, 1] *= 200.0
    g[:, 2, N // 2:] *= 200.0
    return g


def test_gated_steep_and_mild_gates(cuda_lib):
    """The gated mask weights exp(G_j - G_m) are formed from a row and a column factor when the
    chunk's cumulative log2-decay stays within +-100, else element by element; one call mixes
    both kinds of chunk (ragged tail, initial state) and must match the oracle."""
    B, H, N, dk, dv = 1, 4, 300, 64, 128
    gen = torch.Generator().manual_seed(77)
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen)
    g = _steep_and_mild_gates(B, H, N, gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    qd, kd, vd, gdv, S0d = _dev(q, k, v, g, S0)
    s_out = torch.empty_like(S0d)
    o = cuda_lib.gated_ret_chunkwise(qd, kd, vd, gdv, 64, state_in=S0d, state_out=s_out)
    assert cuda_lib.last_device_error() == 0
    want_o, want_s = O.gated_chunkwise(q, k, v, g, 64, state_in=S0)
    for h in range(H):
        assert rel_l2(o[0, h].cpu(), want_o[0, h]) <= TOL_BF16, ("o", h)
        assert rel_l2(s_out[0, h].cpu(), want_s[0, h]) <= TOL_BF16, ("state", h)


GATED_WIDE_CASES = [
    # B, H, N, dk, dv
    (1, 2, 300, 128, 128),   # ragged last tile
    (2, 3, 1000, 256, 256),  # two dv slices; the lazy scale renormalises along the sequence
    (1, 1, 2053, 128, 128),  # one head: the sequence is cut into segments
]


@pytest.mark.parametrize("B,H,N,dk,dv", GATED_WIDE_CASES)
def test_gated_128_token_body_matches_oracle(cuda_lib, B, H, N, dk, dv):
    """Gated segments whose every gate lies in [-0.52, 0] (log2-decay of at most 0.75 per
    token) run the 128-token body, with the tile decay exp2(c_last) and the key weights
    exp2(c_last - c_m) in place of gamma's powers. One gate of head 0 is set outside that
    range, so that head's segment takes the 64-token body in the same call."""
    gen = torch.Generator().manual_seed(N + dk)
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen)
    g = I.gate(B, H, N, gen)
    assert float(g.min()) > -0.5 and float(g.max()) <= 0.0
    g[0, 0, N // 3] = -1.0
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    qd, kd, vd, gdv, S0d = _dev(q, k, v, g, S0)
    s_out = torch.empty_like(S0d)
    o = cuda_lib.gated_ret_chunkwise(qd, kd, vd, gdv, 64, state_in=S0d, state_out=s_out)
    assert cuda_lib.last_device_error() == 0
    want_o, want_s = O.gated_chunkwise(q, k, v, g, 64, state_in=S0)
    for b in range(B):
        for h in range(H):
            assert rel_l2(o[b, h].cpu(), want_o[b, h]) <= TOL_BF16, ("o", b, h)
            assert rel_l2(s_out[b, h].cpu(), want_s[b, h]) <= TOL_BF16, ("state", b, h)


def test_chunkwise_no_state_and_in_place_state(cuda_lib):
    B, H, N, dk, dv = 2, 2, 96, 64, 128
    q, k, v = _rand_inputs(B, H, N, dk, dv, torch.bfloat16, seed=11)
    gam = I.gammas(H)
    qd, kd, vd, gd = _dev(q, k, v, gam)
    o = cuda_lib.ret_chunkwise(qd, kd, vd, gd, 64)
    assert_close(o, O.ret_chunkwise(q, k, v, gam, 64)[0], torch.bfloat16, "no state")
    # state_in == state_out (in place)
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(2)) * 0.05
    S = S0.to(DEV)
    o2 = cuda_lib.ret_chunkwise(qd, kd, vd, gd, 64, state_in=S, state_out=S)
    want_o, want_s = O.ret_chunkwise(q, k, v, gam, 64, state_in=S0)
    assert_close(o2, want_o, torch.bfloat16, "in-place o")
    assert_close(S, want_s, torch.bfloat16, "in-place state")


def test_chunkwise_split_sequence_matches_whole(cuda_lib):
    """Prefill in two calls, passing the state, equals one call over the whole sequence."""
    B, H, N, dk, dv, n1 = 1, 4, 300, 128, 128, 128
    q, k, v = _rand_inputs(B, H, N, dk, dv, torch.bfloat16, seed=21)
    gam = I.gammas(H)
    qd, kd, vd, gd = _dev(q, k, v, gam)
    S = torch.empty(B, H, dk, dv, device=DEV)
    o1 = cuda_lib.ret_chunkwise(qd[:, :, :n1].contiguous(), kd[:, :, :n1].contiguous(),
                                vd[:, :, :n1].contiguous(), gd, 64, state_out=S)
    o2 = cuda_lib.ret_chunkwise(qd[:, :, n1:].contiguous(), kd[:, :, n1:].contiguous(),
                                vd[:, :, n1:].contiguous(), gd, 64, state_in=S, state_out=S)
    want_o, want_s = O.ret_chunkwise(q, k, v, gam, 64)
    assert_close(torch.cat([o1, o2], dim=2), want_o, torch.bfloat16, "split o")
    assert_close(S, want_s, torch.bfloat16, "split state")


def test_empty_sequence_passes_state_through(cuda_lib):
    B, H, dk, dv = 1, 2, 64, 128
    q = torch.empty(B, H, 0, dk, dtype=torch.bfloat16, device=DEV)
    v = torch.empty(B, H, 0, dv, dtype=torch.bfloat16, device=DEV)
    gam = I.gammas(H).to(DEV)
    S0 = torch.randn(B, H, dk, dv, device=DEV)
    S1 = torch.full_like(S0, 7.0)
    cuda_lib.ret_chunkwise(q, q, v, gam, 64, state_in=S0, state_out=S1)
    torch.cuda.synchronize()
    assert torch.equal(S0, S1)
    cuda_lib.ret_chunkwise(q, q, v, gam, 64, state_out=S1)
    torch.cuda.synchronize()
    assert torch.count_nonzero(S1) == 0


@pytest.mark.parametrize("dtype", [torch.float32, torch.bfloat16])
def test_parallel_matches_oracle(cuda_lib, dtype):
    B, H, N, dk, dv = 2, 3, 100, 40, 72
    q, k, v = _rand_inputs(B, H, N, dk, dv, dtype, seed=5)
    gam = _gammas_with_edges(H)
    o = cuda_lib.ret_parallel(*_dev(q, k, v, gam))
    assert_close(o, O.ret_parallel(q, k, v, gam), dtype, "parallel")


def test_gamma_special_cases_on_gpu(cuda_lib):
    """gamma = 0 gives o_n = (q_n . k_n) v_n; gamma = 1 gives the undecayed prefix sum."""
    B, H, N, dk, dv = 1, 2, 70, 64, 128
    q, k, v = _rand_inputs(B, H, N, dk, dv, torch.float32, seed=9)
    qn, kn, vn = (t.double().numpy() for t in (q, k, v))
    gam = torch.tensor([0.0, 1.0])
    o = cuda_lib.ret_chunkwise(*_dev(q, k, v, gam), 16).cpu().double().numpy()
    want0 = np.einsum("nd,nd->n", qn[0, 0], kn[0, 0])[:, None] * vn[0, 0]
    kv = np.cumsum(np.einsum("nd,ne->nde", kn[0, 1], vn[0, 1]), axis=0)
    want1 = np.einsum("nd,nde->ne", qn[0, 1], kv)
    assert rel_l2(o[0, 0], want0) < TOL_F32
    assert rel_l2(o[0, 1], want1) < TOL_F32


MODE_GAMMAS = [0.0, 0.3, 0.49, 0.5, 0.75, 0.96875, 0.999, 1.0]


@pytest.mark.parametrize("dv", [128, 256])
@pytest.mark.parametrize("dk", [64, 128, 256])
def test_tensor_core_output_modes_per_head(cuda_lib, dk, dv):
    """The tensor-core path picks a kernel body per head from its gamma: the
    64-token body with split or merged output accumulators, or the 128-token
    body. One call mixes all of them, with a ragged last tile and an initial
    state, over one and two dv slices; every head must match the oracle."""
    B, H, N = 1, len(MODE_GAMMAS), 300
    assert cuda_lib.chunkwise_path(dk, dv, 64, torch.bfloat16) == 1
    gam = torch.tensor(MODE_GAMMAS, dtype=torch.float32)
    q, k, v = _rand_inputs(B, H, N, dk, dv, torch.bfloat16, seed=41 + dk)
    S0 = torch.randn(B, H, dk, dv, generator=torch.Generator().manual_seed(dk)) * 0.05
    qd, kd, vd, gd, S0d = _dev(q, k, v, gam, S0)
    s_out = torch.empty_like(S0d)
    o = cuda_lib.ret_chunkwise(qd, kd, vd, gd, 64, state_in=S0d, state_out=s_out).cpu()
    assert cuda_lib.last_device_error() == 0
    want_o, want_s = O.ret_chunkwise(q, k, v, gam, 64, state_in=S0)
    for h, g in enumerate(MODE_GAMMAS):
        assert rel_l2(o[0, h], want_o[0, h]) <= TOL_BF16, ("o", g)
        assert rel_l2(s_out[0, h].cpu(), want_s[0, h]) <= TOL_BF16, ("state", g)


# ------------------------------------------------------------------ decode step

@pytest.mark.parametrize("dtype,dv", [(torch.float32, 128), (torch.bfloat16, 512), (torch.float32, 30)])
def test_recurrent_step_matches_oracle(cuda_lib, dtype, dv):
    B, H, dk = 3, 4, 64
    gam = I.gammas(H, "h/3")
    S0 = I.decode_state(B, H, dk, dv, seed=1)
    Sd = S0.to(DEV)
    S_ref = S0.double().numpy()
    for step in range(5):
        q, k, v = I.decode_step_inputs(B, H, dk, dv, step, dtype=dtype)
        o = cuda_lib.ret_recurrent_step(*_dev(q, k, v, gam), Sd)
        want_o, S_ref = O.ret_recurrent_step(q, k, v, gam, S_ref)
        assert_close(o, want_o, dtype, f"o step {step}")
    assert_close(Sd, S_ref, dtype, "state")


@pytest.mark.parametrize("dtype,dv", [(torch.float32, 128), (torch.bfloat16, 512), (torch.float32, 30)])
def test_gated_recurrent_step_matches_oracle(cuda_lib, dtype, dv):
    """Gated decode step (vector path, and the scalar path for dv = 30), five steps
    with a fresh log-decay per step and (b, h), from a nonzero state."""
    B, H, dk = 3, 4, 64
    S0 = I.decode_state(B, H, dk, dv, seed=2)
    Sd = S0.to(DEV)
    S_ref = S0.double().numpy()
    for step in range(5):
        q, k, v = I.decode_step_inputs(B, H, dk, dv, step, dtype=dtype)
        g = I.decode_gate(B, H, step) * 8.0  # stronger decay than the workload
        o = cuda_lib.gated_ret_recurrent_step(*_dev(q, k, v, g), Sd)
        want_o, S_ref = O.gated_recurrent_step(q, k, v, g, S_ref)
        assert_close(o, want_o, dtype, f"o step {step}")
    assert_close(Sd, S_ref, dtype, "state")


# ------------------------------------------------------------------ full-size workloads, sampled heads

def _head(x, b, h):
    return x[b:b + 1, h:h + 1].contiguous()


@pytest.mark.parametrize("name", ["retnet_1p3b", "retnet_6p7b_long", "gated"])
def test_full_size_workload_sampled_heads(cuda_lib, name):
    cfg = I.CONFIGS[name]
    x = I.config_inputs(cfg)
    gated = "g" in x
    dev = {key: val.to(DEV) for key, val in x.items()}
    s_out = torch.empty(cfg.B, cfg.H, cfg.dk, cfg.dv, device=DEV)
    if gated:
        o = cuda_lib.gated_ret_chunkwise(dev["q"], dev["k"], dev["v"], dev["g"], cfg.chunk, state_out=s_out)
    else:
        o = cuda_lib.ret_chunkwise(dev["q"], dev["k"], dev["v"], dev["gamma"], cfg.chunk, state_out=s_out)
    torch.cuda.synchronize()
    assert cuda_lib.last_device_error() == 0
    assert torch.isfinite(o).all()
    samples = [(0, 0), (cfg.B - 1, cfg.H - 1), (cfg.B // 2, cfg.H // 2)]
    for b, h in samples:
        q, k, v = (_head(x[n], b, h) for n in ("q", "k", "v"))
        if gated:
            want_o, want_s = O.gated_chunkwise(q, k, v, _head(x["g"], b, h), cfg.chunk)
        else:
            want_o, want_s = O.ret_chunkwise(q, k, v, x["gamma"][h:h + 1], cfg.chunk)
        assert_close(o[b:b + 1, h:h + 1], want_o, cfg.dtype, f"{name} head ({b},{h})")
        assert_close(s_out[b:b + 1, h:h + 1], want_s, cfg.dtype, f"{name} state ({b},{h})")


def test_full_size_decode_sampled_heads(cuda_lib):
    cfg = I.CONFIGS["decode"]
    B, H, dk, dv = cfg.B, cfg.H, cfg.dk, cfg.dv
    gam = I.gammas(H, cfg.gamma_schedule)
    S0 = I.decode_state(B, H, dk, dv)
    Sd = S0.to(DEV)
    gd = gam.to(DEV)
    samples = [(0, 0), (B - 1, H - 1), (31, 7)]
    S_ref = {s: S0[s[0]:s[0] + 1, s[1]:s[1] + 1].double().numpy() for s in samples}
    got = {s: [] for s in samples}
    want = {s: [] for s in samples}
    for step in range(I.DECODE_STEPS):
        q, k, v = I.decode_step_inputs(B, H, dk, dv, step)
        o = cuda_lib.ret_recurrent_step(*_dev(q, k, v), gd, Sd)
        for (b, h) in samples:
            got[(b, h)].append(o[b, h].float().cpu())
            sl = (slice(b, b + 1), slice(h, h + 1))
            ow, S_ref[(b, h)] = O.ret_recurrent_step(q[sl], k[sl], v[sl], gam[h:h + 1], S_ref[(b, h)])
            want[(b, h)].append(ow[0, 0])
    assert cuda_lib.last_device_error() == 0
    for s in samples:
        assert rel_l2(torch.stack(got[s]), np.stack(want[s])) <= TOL_BF16, s
        assert rel_l2(Sd[s[0], s[1]], S_ref[s][0, 0]) <= TOL_BF16, s


def test_full_size_gated_decode_sampled_heads(cuda_lib):
    """The gated decode workload at full size (1 GiB state) for 256 steps, sampled heads
    checked against the oracle every step and in the final state."""
    cfg = I.CONFIGS["gated_decode"]
    B, H, dk, dv = cfg.B, cfg.H, cfg.dk, cfg.dv
    S0 = I.decode_state(B, H, dk, dv)
    Sd = S0.to(DEV)
    samples = [(0, 0), (B - 1, H - 1), (17, 9)]
    S_ref = {s: S0[s[0]:s[0] + 1, s[1]:s[1] + 1].double().numpy() for s in samples}
    got = {s: [] for s in samples}
    want = {s: [] for s in samples}
    for step in range(256):
        q, k, v = I.decode_step_inputs(B, H, dk, dv, step)
        g = I.decode_gate(B, H, step)
        o = cuda_lib.gated_ret_recurrent_step(*_dev(q, k, v, g), Sd)
        for (b, h) in samples:
            got[(b, h)].append(o[b, h].float().cpu())
            sl = (slice(b, b + 1), slice(h, h + 1))
            ow, S_ref[(b, h)] = O.gated_recurrent_step(q[sl], k[sl], v[sl], g[sl], S_ref[(b, h)])
            want[(b, h)].append(ow[0, 0])
    assert cuda_lib.last_device_error() == 0
    for s in samples:
        assert rel_l2(torch.stack(got[s]), np.stack(want[s])) <= TOL_BF16, s
        assert rel_l2(Sd[s[0], s[1]], S_ref[s][0, 0]) <= TOL_BF16, s


# ------------------------------------------------------------------ split sequences (few heads, long N)

SPLIT_CASES = [
    # B, H, N, dk, dv
    (1, 2, 1000, 64, 128),
    (1, 1, 2053, 128, 128),
    (2, 1, 777, 256, 256),
    # dv of several 128-column slices, dk 64 and 128
    (1, 1, 1500, 64, 256),
    (1, 2, 1100, 128, 512),
]


@pytest.mark.parametrize("gated", [False, True])
@pytest.mark.parametrize("inplace", [False, True])
@pytest.mark.parametrize("B,H,N,dk,dv", SPLIT_CASES)
def test_split_sequence_matches_oracle(cuda_lib, B, H, N, dk, dv, gated, inplace):
    """The tensor-core path cuts long sequences of few heads into segments (a
    state-only pass, then the full pass seeded per segment); the result must not
    change, including the final state and an in-place state buffer."""
    assert cuda_lib.chunkwise_launches(B, H, N, dk, dv, 64, torch.bfloat16) == 3  # state-only pass, segment prefix, full pass
    gen = torch.Generator().manual_seed(N + dk + int(gated))
    q, k, v = I.qkv(B, H, N, dk, dv, torch.bfloat16, gen=gen)
    S0 = torch.randn(B, H, dk, dv, generator=gen) * 0.05
    qd, kd, vd, S0d = _dev(q, k, v, S0)
    s_out = S0d if inplace else torch.empty_like(S0d)
    if gated:
        g = I.gate(B, H, N, gen) * 4.0
        o = cuda_lib.gated_ret_chunkwise(qd, kd, vd, g.to(DEV), 64, state_in=S0d, state_out=s_out)
        want_o, want_s = O.gated_chunkwise(q, k, v, g, 64, state_in=S0)
    else:
        gam = _gammas_with_edges(H + 2)[-H:]  # includes 1.0 and 0.9 style heads
        o = cuda_lib.ret_chunkwise(qd, kd, vd, gam.to(DEV), 64, state_in=S0d, state_out=s_out)
        want_o, want_s = O.ret_chunkwise(q, k, v, gam, 64, state_in=S0)
    assert cuda_lib.last_device_error() == 0
    assert_close(o, want_o, torch.bfloat16, "o")
    assert_close(s_out, want_s, torch.bfloat16, "state")


def test_split_sequence_gamma_zero(cuda_lib):
    """gamma = 0 makes every segment's decay exactly zero; the split must still give (q.k) v."""
    B, H, N, dk, dv = 1, 1, 900, 64, 128
    q, k, v = _rand_inputs(B, H, N, dk, dv, torch.bfloat16, seed=31)
    gam = torch.zeros(1)
    o = cuda_lib.ret_chunkwise(*_dev(q, k, v, gam), 64)
    qn, kn, vn = (t.double().numpy()[0, 0] for t in (q, k, v))
    want = np.einsum("nd,nd->n", qn, kn)[:, None] * vn
    assert rel_l2(o[0, 0], want) <= TOL_BF16
