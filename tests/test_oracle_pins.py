"""Pins for the fp64 oracle, against facts that do not come from the oracle itself.

Each test ties the oracle to something independent of its own code: hand-worked
examples, the mathematical equivalence of three differently structured forms,
closed forms (gamma = 0, gamma = 1, constant gate), invariants of the decay
matrix, linearity, and split invariance of the state. The mutation tests at the
end plant plausible mistakes in a copy of the oracle and check that a pin fails.
"""
import json
import os
import subprocess
import tempfile
import ctypes

import numpy as np
import torch
import pytest

from oracle import oracle as O

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "retention_hand_examples.json")


def _rand(shape, rng):
    return rng.standard_normal(shape)


def _inputs(B=1, H=2, N=40, dk=5, dv=3, seed=0):
    rng = np.random.default_rng(seed)
    return _rand((B, H, N, dk), rng), _rand((B, H, N, dk), rng), _rand((B, H, N, dv), rng)


def _golden():
    with open(GOLDEN) as f:
        return {e["name"]: e for e in json.load(f)["examples"]}


def _as4(a):
    a = np.asarray(a, dtype=np.float64)
    return a[None, None]


# ---------------------------------------------------------------- golden (hand-worked)

@pytest.mark.parametrize("name", ["scalar_geometric", "two_dim_integer"])
def test_golden_retention_all_forms(name):
    ex = _golden()[name]
    q, k, v = _as4(ex["q"]), _as4(ex["k"]), _as4(ex["v"])
    gam = np.asarray(ex["gamma"])
    want_o, want_s = _as4(ex["o"]), _as4(ex["state"])
    N = q.shape[2]
    np.testing.assert_allclose(O.ret_brute(q, k, v, gam), want_o, atol=1e-15)
    np.testing.assert_allclose(O.ret_parallel(q, k, v, gam), want_o, atol=1e-15)
    o, s = O.ret_recurrent(q, k, v, gam)
    np.testing.assert_allclose(o, want_o, atol=1e-15)
    np.testing.assert_allclose(s, want_s, atol=1e-15)
    for c in range(1, N + 2):
        o, s = O.ret_chunkwise(q, k, v, gam, c)
        np.testing.assert_allclose(o, want_o, atol=1e-14)
        np.testing.assert_allclose(s, want_s, atol=1e-14)


def test_golden_gated_all_forms():
    ex = _golden()["two_dim_gated"]
    q, k, v = _as4(ex["q"]), _as4(ex["k"]), _as4(ex["v"])
    g = np.log(np.asarray(ex["decay"]))[None, None]
    want_o, want_s = _as4(ex["o"]), _as4(ex["state"])
    np.testing.assert_allclose(O.gated_brute(q, k, v, g), want_o, atol=1e-14)
    np.testing.assert_allclose(O.gated_parallel(q, k, v, g), want_o, atol=1e-14)
    o, s = O.gated_recurrent(q, k, v, g)
    np.testing.assert_allclose(o, want_o, atol=1e-14)
    np.testing.assert_allclose(s, want_s, atol=1e-14)
    for c in (1, 2, 3, 4):
        o, s = O.gated_chunkwise(q, k, v, g, c)
        np.testing.assert_allclose(o, want_o, atol=1e-14)
        np.testing.assert_allclose(s, want_s, atol=1e-14)


def test_golden_decode_step():
    ex = _golden()["decode_step"]
    q = np.asarray(ex["q"], dtype=np.float64)[None, None]
    k = np.asarray(ex["k"], dtype=np.float64)[None, None]
    v = np.asarray(ex["v"], dtype=np.float64)[None, None]
    S = _as4(ex["state_in"])
    o, S2 = O.ret_recurrent_step(q, k, v, np.asarray(ex["gamma"]), S)
    np.testing.assert_allclose(o[0, 0], ex["o"], atol=1e-15)
    np.testing.assert_allclose(S2[0, 0], ex["state"], atol=1e-15)


# ---------------------------------------------------------------- decay matrix D

@pytest.mark.parametrize("gamma", [0.0, 0.3, 0.9, 0.96875, 1.0])
def test_decay_matrix_invariants(gamma):
    N = 12
    D = O.decay_matrix(gamma, N)
    # causal: zeros strictly above the diagonal; ones on it (gamma^0 = 1)
    assert np.all(D[np.triu_indices(N, 1)] == 0.0)
    assert np.all(np.diag(D) == 1.0)
    # one step further back multiplies by gamma (the recurrence), for n-1 >= m
    for n in range(1, N):
        for m in range(n):
            assert D[n, m] == pytest.approx(gamma * D[n - 1, m], rel=1e-14, abs=0)
    # semigroup: D[n,m] = D[n,j] D[j,m] for m <= j <= n (Toeplitz in n-m)
    for n in range(N):
        for m in range(n + 1):
            for j in range(m, n + 1):
                assert D[n, m] == pytest.approx(D[n, j] * D[j, m], rel=1e-14, abs=1e-300)


# ---------------------------------------------------------------- equivalence of forms

GAMMAS = np.array([0.96875, 0.6])


def test_parallel_matches_brute_force():
    q, k, v = _inputs(N=23)
    np.testing.assert_allclose(O.ret_parallel(q, k, v, GAMMAS), O.ret_brute(q, k, v, GAMMAS),
                               rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 2, 3, 7, 8, 32, 40, 64])
def test_chunkwise_matches_parallel_and_recurrent(chunk):
    q, k, v = _inputs(B=2, N=40)
    ref = O.ret_parallel(q, k, v, GAMMAS)
    o_rec, s_rec = O.ret_recurrent(q, k, v, GAMMAS)
    o_chk, s_chk = O.ret_chunkwise(q, k, v, GAMMAS, chunk)
    np.testing.assert_allclose(o_rec, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o_chk, ref, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s_chk, s_rec, rtol=1e-12, atol=1e-12)


def test_numpy_demo_shape_parallel_vs_recurrent():
    """The tutorial's demo shape: one head, n=8, d=16, gamma=0.9, projections of a
    random X by 0.05-scaled random weights; parallel and recurrent agree to 1e-6."""
    rng = np.random.default_rng(42)
    d, n = 16, 8
    Wq, Wk, Wv = (rng.standard_normal((d, d)) * 0.05 for _ in range(3))
    X = rng.standard_normal((n, d))
    q, k, v = (X @ W for W in (Wq, Wk, Wv))
    q, k, v = q[None, None], k[None, None], v[None, None]
    a = O.ret_parallel(q, k, v, np.array([0.9]))
    b, _ = O.ret_recurrent(q, k, v, np.array([0.9]))
    assert np.abs(a - b).max() < 1e-6


def test_state_split_invariance():
    q, k, v = _inputs(B=2, N=50, dk=4, dv=6, seed=3)
    o_full, s_full = O.ret_chunkwise(q, k, v, GAMMAS, 8)
    n1 = 21
    o1, s1 = O.ret_chunkwise(q[:, :, :n1], k[:, :, :n1], v[:, :, :n1], GAMMAS, 8)
    o2, s2 = O.ret_chunkwise(q[:, :, n1:], k[:, :, n1:], v[:, :, n1:], GAMMAS, 5, state_in=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), o_full, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(s2, s_full, rtol=1e-12, atol=1e-12)


def test_decode_steps_match_sequence_forms():
    rng = np.random.default_rng(5)
    B, H, N, dk, dv = 2, 2, 17, 4, 3
    q, k, v = _inputs(B, H, N, dk, dv, seed=5)
    S0 = rng.standard_normal((B, H, dk, dv)) * 0.1
    S = S0.copy()
    outs = []
    for t in range(N):
        o, S = O.ret_recurrent_step(q[:, :, t], k[:, :, t], v[:, :, t], GAMMAS, S)
        outs.append(o)
    o_steps = np.stack(outs, axis=2)
    o_rec, s_rec = O.ret_recurrent(q, k, v, GAMMAS, state_in=S0)
    o_chk, s_chk = O.ret_chunkwise(q, k, v, GAMMAS, 6, state_in=S0)
    np.testing.assert_allclose(o_steps, o_rec, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(o_chk, o_rec, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(S, s_chk, rtol=1e-12, atol=1e-12)


# ---------------------------------------------------------------- closed forms

def test_gamma_zero_is_diagonal_scores():
    """gamma = 0 keeps only m = n: o_n = (q_n . k_n) v_n."""
    q, k, v = _inputs(N=19)
    gam = np.array([0.0, 0.0])
    want = np.einsum("bhnd,bhnd->bhn", q, k)[..., None] * v
    np.testing.assert_allclose(O.ret_parallel(q, k, v, gam), want, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(O.ret_recurrent(q, k, v, gam)[0], want, rtol=1e-12, atol=1e-13)
    for c in (1, 4, 19):
        np.testing.assert_allclose(O.ret_chunkwise(q, k, v, gam, c)[0], want, rtol=1e-12, atol=1e-13)


def test_gamma_one_is_undecayed_prefix_sum():
    """gamma = 1 is linear attention without decay: o_n = q_n sum_{m<=n} k_m^T v_m."""
    q, k, v = _inputs(N=19)
    gam = np.array([1.0, 1.0])
    kv = np.cumsum(np.einsum("bhnd,bhne->bhnde", k, v), axis=2)
    want = np.einsum("bhnd,bhnde->bhne", q, kv)
    np.testing.assert_allclose(O.ret_parallel(q, k, v, gam), want, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(O.ret_chunkwise(q, k, v, gam, 5)[0], want, rtol=1e-11, atol=1e-12)


def test_linearity():
    q, k, v = _inputs(N=15, seed=9)
    _, _, v2 = _inputs(N=15, seed=10)
    a = O.ret_chunkwise(q, k, 2.0 * v - 3.0 * v2, GAMMAS, 4)[0]
    b = 2.0 * O.ret_chunkwise(q, k, v, GAMMAS, 4)[0] - 3.0 * O.ret_chunkwise(q, k, v2, GAMMAS, 4)[0]
    np.testing.assert_allclose(a, b, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(O.ret_parallel(2 * q, k, v, GAMMAS), 2 * O.ret_parallel(q, k, v, GAMMAS),
                               rtol=1e-12)


# ---------------------------------------------------------------- gated forms

def _gate(B, H, N, seed=1, scale=1.0):
    rng = np.random.default_rng(seed)
    x = rng.standard_normal((B, H, N))
    return scale * (-np.logaddexp(0.0, -x) / 16.0)  # logsigmoid(x)/16 < 0


def test_gated_constant_gate_equals_fixed_gamma():
    q, k, v = _inputs(B=2, N=33)
    g = np.broadcast_to(np.log(GAMMAS)[None, :, None], (2, 2, 33)).copy()
    ref = O.ret_parallel(q, k, v, GAMMAS)
    np.testing.assert_allclose(O.gated_parallel(q, k, v, g), ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(O.gated_brute(q, k, v, g), ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(O.gated_recurrent(q, k, v, g)[0], ref, rtol=1e-11, atol=1e-12)
    o, s = O.gated_chunkwise(q, k, v, g, 7)
    np.testing.assert_allclose(o, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s, O.ret_recurrent(q, k, v, GAMMAS)[1], rtol=1e-11, atol=1e-12)


def test_gated_zero_gate_is_prefix_sum():
    q, k, v = _inputs(N=13)
    g = np.zeros((1, 2, 13))
    kv = np.cumsum(np.einsum("bhnd,bhne->bhnde", k, v), axis=2)
    want = np.einsum("bhnd,bhnde->bhne", q, kv)
    np.testing.assert_allclose(O.gated_chunkwise(q, k, v, g, 4)[0], want, rtol=1e-11, atol=1e-12)


@pytest.mark.parametrize("chunk", [1, 3, 8, 16, 64])
def test_gated_forms_agree(chunk):
    q, k, v = _inputs(B=2, N=37, seed=4)
    g = _gate(2, 2, 37, scale=8.0)
    ref = O.gated_brute(q, k, v, g)
    np.testing.assert_allclose(O.gated_parallel(q, k, v, g), ref, rtol=1e-11, atol=1e-12)
    o_rec, s_rec = O.gated_recurrent(q, k, v, g)
    o_chk, s_chk = O.gated_chunkwise(q, k, v, g, chunk)
    np.testing.assert_allclose(o_rec, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(o_chk, ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s_chk, s_rec, rtol=1e-11, atol=1e-12)


def test_gated_step_constant_gate_equals_fixed_step():
    """A gated decode step with g = ln(gamma_h) is the fixed-gamma decode step."""
    rng = np.random.default_rng(21)
    q, k, v = rng.standard_normal((2, 2, 5)), rng.standard_normal((2, 2, 5)), rng.standard_normal((2, 2, 3))
    S = rng.standard_normal((2, 2, 5, 3))
    g = np.broadcast_to(np.log(GAMMAS)[None, :], (2, 2)).copy()
    o_g, S_g = O.gated_recurrent_step(q, k, v, g, S)
    o_f, S_f = O.ret_recurrent_step(q, k, v, GAMMAS, S)
    np.testing.assert_allclose(o_g, o_f, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(S_g, S_f, rtol=1e-12, atol=1e-13)


def test_gated_steps_equal_gated_chunkwise():
    """Twelve gated decode steps from a state equal the gated chunkwise form over the
    same twelve tokens (in-chunk cumulative sums, a different computation), per token
    and in the final state; one step by hand: S' = e^g S + k^T v, o = q S'."""
    q, k, v = _inputs(B=1, H=2, N=12, seed=22)
    g = _gate(1, 2, 12, seed=3, scale=8.0)
    S0 = np.random.default_rng(23).standard_normal((1, 2, 5, 3))
    S = S0
    outs = []
    for t in range(12):
        o, S = O.gated_recurrent_step(q[:, :, t], k[:, :, t], v[:, :, t], g[:, :, t], S)
        outs.append(o)
    o_chk, s_chk = O.gated_chunkwise(q, k, v, g, 5, state_in=S0)
    np.testing.assert_allclose(np.stack(outs, axis=2), o_chk, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(S, s_chk, rtol=1e-11, atol=1e-12)
    S1 = np.exp(g[:, :, 0])[..., None, None] * S0 + np.einsum("bhd,bhe->bhde", k[:, :, 0], v[:, :, 0])
    o1, S1_or = O.gated_recurrent_step(q[:, :, 0], k[:, :, 0], v[:, :, 0], g[:, :, 0], S0)
    np.testing.assert_allclose(S1_or, S1, rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(o1, np.einsum("bhd,bhde->bhe", q[:, :, 0], S1), rtol=1e-13, atol=1e-13)


def test_gated_long_sequence_stays_finite():
    """A long strongly decaying gate drives the global cumulative sum far below
    exp's range; the chunkwise form uses in-chunk sums only and stays finite."""
    q, k, v = _inputs(B=1, H=1, N=3000, dk=3, dv=2, seed=8)
    g = np.full((1, 1, 3000), -0.5)  # G reaches -1500: exp(G) underflows
    o_chk, s_chk = O.gated_chunkwise(q, k, v, g, 64)
    o_rec, s_rec = O.gated_recurrent(q, k, v, g)
    assert np.all(np.isfinite(o_chk)) and np.all(np.isfinite(s_chk))
    np.testing.assert_allclose(o_chk, o_rec, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(s_chk, s_rec, rtol=1e-10, atol=1e-12)


def test_gated_split_invariance():
    q, k, v = _inputs(B=1, N=45, seed=12)
    g = _gate(1, 2, 45, seed=13, scale=4.0)
    o_full, s_full = O.gated_chunkwise(q, k, v, g, 8)
    n1 = 19
    o1, s1 = O.gated_chunkwise(q[:, :, :n1], k[:, :, :n1], v[:, :, :n1], g[:, :, :n1], 8)
    o2, s2 = O.gated_chunkwise(q[:, :, n1:], k[:, :, n1:], v[:, :, n1:], g[:, :, n1:], 6, state_in=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), o_full, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(s2, s_full, rtol=1e-11, atol=1e-12)


def test_bad_arguments_rejected():
    q, k, v = _inputs(N=4)
    with pytest.raises(ValueError):
        O.ret_chunkwise(q, k, v, GAMMAS, 0)


# ---------------------------------------------------------------- planted mistakes

# ---------------------------------------------------------------- backward pass

def _fd(f, x, eps=1e-6):
    """Central finite differences of the scalar function f at x (fp64)."""
    g = np.zeros_like(x)
    for idx in np.ndindex(x.shape):
        xp, xm = x.copy(), x.copy()
        xp[idx] += eps
        xm[idx] -= eps
        g[idx] = (f(xp) - f(xm)) / (2 * eps)
    return g


def test_backward_matches_finite_differences():
    """Gradients of L = sum dO . O against central differences of the brute-force forward."""
    q, k, v = _inputs(B=1, H=2, N=7, dk=3, dv=4, seed=30)
    do = np.random.default_rng(31).standard_normal((1, 2, 7, 4))
    gam = np.array([0.9, 0.6])
    loss = lambda q_, k_, v_, g_: float(np.sum(do * O.ret_brute(q_, k_, v_, g_)))
    dq, dk, dv, dgam = O.ret_backward(q, k, v, gam, do)
    np.testing.assert_allclose(dq, _fd(lambda x: loss(x, k, v, gam), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd(lambda x: loss(q, x, v, gam), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd(lambda x: loss(q, k, x, gam), v), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dgam, _fd(lambda x: loss(q, k, v, x), gam), rtol=1e-6, atol=1e-8)


def test_gated_backward_matches_finite_differences():
    q, k, v = _inputs(B=1, H=2, N=7, dk=3, dv=4, seed=32)
    do = np.random.default_rng(33).standard_normal((1, 2, 7, 4))
    g = _gate(1, 2, 7, seed=34, scale=8.0)
    loss = lambda q_, k_, v_, g_: float(np.sum(do * O.gated_brute(q_, k_, v_, g_)))
    dq, dk, dv, dg = O.gated_backward(q, k, v, g, do)
    np.testing.assert_allclose(dq, _fd(lambda x: loss(x, k, v, g), q), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dk, _fd(lambda x: loss(q, x, v, g), k), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dv, _fd(lambda x: loss(q, k, x, g), v), rtol=1e-6, atol=1e-8)
    np.testing.assert_allclose(dg, _fd(lambda x: loss(q, k, v, x), g), rtol=1e-6, atol=1e-8)


def test_backward_gamma_zero_and_constant_gate():
    """gamma = 0 leaves only the diagonal: dq_n = (dO_n . v_n) k_n, dv_n = (q_n . k_n) dO_n;
    a constant gate g = ln gamma gives the fixed-gamma gradients."""
    q, k, v = _inputs(B=1, H=2, N=9, dk=3, dv=4, seed=35)
    do = np.random.default_rng(36).standard_normal((1, 2, 9, 4))
    dq, dk, dv, _ = O.ret_backward(q, k, v, np.array([0.0, 0.0]), do)
    a = np.einsum("bhnc,bhnc->bhn", do, v)
    s = np.einsum("bhnd,bhnd->bhn", q, k)
    np.testing.assert_allclose(dq, a[..., None] * k, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dk, a[..., None] * q, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(dv, s[..., None] * do, rtol=1e-12, atol=1e-12)
    gam = np.array([0.9, 0.75])
    g = np.broadcast_to(np.log(gam)[None, :, None], (1, 2, 9)).copy()
    ref = O.ret_backward(q, k, v, gam, do)
    got = O.gated_backward(q, k, v, g, do)
    for a_, b_ in zip(ref[:3], got[:3]):
        np.testing.assert_allclose(b_, a_, rtol=1e-11, atol=1e-12)
    # dL/dlog(gamma) = gamma dL/dgamma = sum over the sequence of dL/dg_t
    np.testing.assert_allclose(got[3].sum(axis=2)[0], gam * ref[3], rtol=1e-10, atol=1e-12)


_MUTANTS = {
    # the printed single gamma^c cross factor instead of the per-row gamma^(j+1)
    "uniform_cross_factor": ("const double r = gpow(gm, j + 1);", "const double r = gpow(gm, L);"),
    # key weights dropped from the state update
    "no_key_weight": ("const double zeta = gpow(gm, L - 1 - m);", "const double zeta = 1.0;"),
    # decay matrix transposed (upper instead of lower triangle)
    "transposed_mask": ("D[(size_t)n * N + m] = (n >= m) ? gpow(gamma, n - m) : 0.0;",
                        "D[(size_t)n * N + m] = (n <= m) ? gpow(gamma, m - n) : 0.0;"),
    # decay exponent off by one
    "exponent_off_by_one": ("const double w = gpow(gm, n - m) * qk;", "const double w = gpow(gm, n - m + 1) * qk;"),
    # gated inner mask with the sign of the log-decay difference flipped
    "gated_sign": ("A[(size_t)j * L + m] = (j >= m) ? s * exp(Gl[j] - Gl[m]) : 0.0;",
                   "A[(size_t)j * L + m] = (j >= m) ? s * exp(Gl[m] - Gl[j]) : 0.0;"),
    # gated parallel form with an exclusive instead of inclusive cumulative sum
    "gated_exclusive_cumsum": ("for (int n = 0; n < N; ++n) { acc += Gt[n]; G[n] = acc; }",
                               "for (int n = 0; n < N; ++n) { G[n] = acc; acc += Gt[n]; }"),
    # backward: decay gradient exponent off by one
    "backward_dgamma_power": ("if (n > m) dg += (double)(n - m) * gpow(gm, n - m - 1) * s * a;",
                              "if (n > m) dg += (double)(n - m) * gpow(gm, n - m) * s * a;"),
    # gated backward: gate gradient over the wrong range of t (includes t = m)
    "backward_gate_range": ("for (int t = m + 1; t <= n; ++t) DG[t] += w * s * a;",
                            "for (int t = m; t <= n; ++t) DG[t] += w * s * a;"),
    # epilogue: eps added outside the square root
    "norm_eps_outside": ("const double inv_rms = 1.0 / sqrt(ms + eps);", "const double inv_rms = 1.0 / (sqrt(ms) + eps);"),
    # epilogue: sum of squares instead of the mean
    "norm_sum_not_mean": ("    ms /= dv;\n", "\n"),
    # epilogue: the gate's sigmoid instead of its swish
    "gate_sigmoid": ("const double swish = x / (1.0 + exp(-x));", "const double swish = 1.0 / (1.0 + exp(-x));"),
    # epilogue: y written head-major like o instead of token-major
    "norm_layout": ("const size_t yoff = (((size_t)b * N + n) * H + h) * dv;",
                    "const size_t yoff = ((size_t)bh * N + n) * dv;"),
}


def _build_mutant(tmpdir, old, new):
    src = open(os.path.join(os.path.dirname(O.__file__), "oracle.c")).read()
    assert src.count(old) == 1, old
    path_c = os.path.join(tmpdir, "mut.c")
    with open(path_c, "w") as f:
        f.write(src.replace(old, new))
    path_so = os.path.join(tmpdir, "libmut.so")
    subprocess.run(["gcc", "-O1", "-fopenmp", "-fPIC", "-shared", path_c, "-o", path_so, "-lm"], check=True)
    return path_so


def _pins_pass_with(lib_path):
    """Run a subset of the pins above against a differently built oracle library."""
    real = O._lib
    try:
        lib = ctypes.CDLL(lib_path)
        O._lib = None
        sig_src = O._load()  # the real library carries the argtypes to copy
        for name in ("oracle_decay_matrix", "oracle_ret_brute", "oracle_ret_parallel", "oracle_ret_recurrent",
                     "oracle_ret_recurrent_step", "oracle_ret_chunkwise", "oracle_gated_brute",
                     "oracle_gated_parallel", "oracle_gated_recurrent", "oracle_gated_chunkwise",
                     "oracle_ret_backward", "oracle_gated_backward", "oracle_msr_norm_gate"):
            fn = getattr(lib, name)
            fn.argtypes = getattr(sig_src, name).argtypes
            fn.restype = ctypes.c_int
        lib.oracle_max_threads.restype = ctypes.c_int
        lib.oracle_set_threads.argtypes = [ctypes.c_int]
        O._lib = lib
        checks = [
            lambda: test_golden_retention_all_forms("two_dim_integer"),
            test_golden_gated_all_forms,
            lambda: test_decay_matrix_invariants(0.9),
            lambda: test_chunkwise_matches_parallel_and_recurrent(7),
            lambda: test_gated_forms_agree(8),
            test_parallel_matches_brute_force,
            test_backward_matches_finite_differences,
            test_gated_backward_matches_finite_differences,
            lambda: test_golden_msr_norm_gate("two_heads_two_tokens_eps"),
            lambda: test_golden_msr_norm_gate("one_row_eps0"),
        ]
        for check in checks:
            try:
                check()
            except AssertionError:
                return False
        return True
    finally:
        O._lib = real


@pytest.mark.parametrize("mutant", sorted(_MUTANTS))
def test_planted_mistake_is_caught(mutant):
    old, new = _MUTANTS[mutant]
    with tempfile.TemporaryDirectory() as d:
        assert not _pins_pass_with(_build_mutant(d, old, new)), f"pins missed mutant {mutant}"


def test_unmutated_copy_passes_pins():
    with tempfile.TemporaryDirectory() as d:
        assert _pins_pass_with(_build_mutant(d, "#define ORACLE_OK 0", "#define ORACLE_OK 0"))


# ---------------------------------------------------------------- multi-scale retention output epilogue

NORM_GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "msr_norm_gate_hand_examples.json")


@pytest.mark.parametrize("name", ["one_row_eps0", "two_heads_two_tokens_eps"])
def test_golden_msr_norm_gate(name):
    with open(NORM_GOLDEN, encoding="utf-8") as f:
        ex = {e["name"]: e for e in json.load(f)["examples"]}[name]
    ln3 = np.log(3.0)
    y = O.msr_norm_gate(np.array(ex["o"], dtype=float), np.array(ex["gate_ln3"], dtype=float) * ln3, ex["eps"])
    np.testing.assert_allclose(y, np.array(ex["y_ln3"]) * ln3, rtol=1e-14, atol=1e-15)


def test_msr_norm_gate_matches_library_routines():
    """Special case that reduces to library routines: torch's rms_norm (no weight) and silu, fp64."""
    rng = np.random.default_rng(40)
    o = rng.standard_normal((2, 3, 17, 24)) * 3.0
    gate = rng.standard_normal((2, 17, 3, 24)) * 2.0
    for eps in (0.0, 1e-5, 0.5):
        y = O.msr_norm_gate(o, gate, eps)
        ref = (torch.nn.functional.rms_norm(torch.from_numpy(o), (24,), eps=eps).permute(0, 2, 1, 3)
               * torch.nn.functional.silu(torch.from_numpy(gate)))
        np.testing.assert_allclose(y, ref.numpy(), rtol=1e-12, atol=1e-14)


def test_msr_norm_gate_invariants():
    """With eps = 0 the output is invariant to positive scaling of a head's row and odd in o;
    with a large gate (swish(x) -> x) each row of y / gate has unit root mean square."""
    rng = np.random.default_rng(41)
    o = rng.standard_normal((1, 2, 5, 8))
    gate = rng.standard_normal((1, 5, 2, 8))
    y = O.msr_norm_gate(o, gate, 0.0)
    np.testing.assert_allclose(O.msr_norm_gate(o * 7.5, gate, 0.0), y, rtol=1e-13)
    np.testing.assert_allclose(O.msr_norm_gate(-o, gate, 0.0), -y, rtol=1e-13)
    big = np.full((1, 5, 2, 8), 60.0)
    r = O.msr_norm_gate(o, big, 0.0) / 60.0
    np.testing.assert_allclose(np.sqrt((r ** 2).mean(axis=-1)), 1.0, rtol=1e-12)
    # eps damps small rows: a row of zeros stays zero for any eps > 0
    z = O.msr_norm_gate(np.zeros((1, 1, 2, 4)), np.ones((1, 2, 1, 4)), 1e-5)
    assert np.all(z == 0.0)
