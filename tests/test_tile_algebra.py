"""The factorisations the tensor-core kernel's fixed-decay bodies compute with, modelled in
fp64 and checked against the oracle's chunkwise form ("RetNet retention mechanism" page,
section 块级循环):

128-token body (gamma >= 2^-0.75): with zeta_m = gamma^(L-1-m) over a tile of L tokens and
the state held as S = kappa T (a scalar kappa and a matrix T),
    kappa <- kappa gamma^L                         (the decay of the carried state, on the scalar)
    o_j    = (kappa / zeta_j) [ q_j T + sum_{m<=j} (q_j . k_m) zeta_m v_m / kappa ]
    T     <- T + sum_m zeta_m k_m^T v_m / kappa
and T is rescaled (T <- kappa T, kappa <- 1) when kappa falls below 2^-40.

64-token merged accumulator (gamma in [1/2, 1]): with zeta'_j = gamma^(63-j),
    gamma^(j-m) = zeta'_m / zeta'_j  and  gamma^(j+1) = gamma^64 / zeta'_j,
so o_j = (1/zeta'_j) [ q_j (gamma^64 S) + sum_{m<=j} zeta'_m (q_j . k_m) v_m ] over 64-token chunks
(a ragged last chunk is zero padding: its rows past the end contribute nothing).
"""
import numpy as np
import pytest

from oracle import oracle as O


def _tile_model_128(q, k, v, gamma, renorm=2.0 ** -40):
    N = q.shape[0]
    T = np.zeros((q.shape[1], v.shape[1]))
    kappa = 1.0
    out = np.zeros((N, v.shape[1]))
    for t0 in range(0, N, 128):
        L = min(128, N - t0)
        qs, ks, vs = q[t0:t0 + L], k[t0:t0 + L], v[t0:t0 + L]
        zeta = gamma ** (L - 1 - np.arange(L))
        if kappa * gamma ** L < renorm:
            T, kappa = kappa * T, 1.0
        kappa *= gamma ** L
        A = np.tril(qs @ ks.T)
        zv = zeta[:, None] * vs / kappa
        out[t0:t0 + L] = (kappa / zeta)[:, None] * (qs @ T + A @ zv)
        T = T + ks.T @ zv
    return out, kappa * T


def _merged_model_64(q, k, v, gamma):
    N = q.shape[0]
    S = np.zeros((q.shape[1], v.shape[1]))
    zp = gamma ** (63 - np.arange(64))
    out = np.zeros((N, v.shape[1]))
    for t0 in range(0, N, 64):
        L = min(64, N - t0)
        qs = np.zeros((64, q.shape[1])); ks = np.zeros((64, k.shape[1])); vs = np.zeros((64, v.shape[1]))
        qs[:L], ks[:L], vs[:L] = q[t0:t0 + L], k[t0:t0 + L], v[t0:t0 + L]  # zero padding past the end
        P = np.tril(qs @ ks.T) * zp[None, :]
        acc = qs @ (gamma ** 64 * S) + P @ vs
        out[t0:t0 + L] = (acc / zp[:, None])[:L]
        # the state update over the chunk's true length L: S <- gamma^L S + sum gamma^(L-1-m) k_m^T v_m
        w = gamma ** (L - 1 - np.arange(L))
        S = gamma ** L * S + (ks[:L] * w[:, None]).T @ vs[:L]
    return out, S


@pytest.mark.parametrize("gamma", [0.999, 0.96875, 2.0 ** -0.75])
@pytest.mark.parametrize("N", [128, 300, 517])
def test_128_token_factorisation_equals_chunkwise(gamma, N):
    rng = np.random.default_rng(N)
    q, k, v = (rng.standard_normal((N, d)) / 3 for d in (6, 6, 5))
    o, s = _tile_model_128(q, k, v, gamma)
    want_o, want_s = O.ret_chunkwise(q[None, None], k[None, None], v[None, None], np.array([gamma]), 128)
    np.testing.assert_allclose(o, want_o[0, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(s, want_s[0, 0], rtol=1e-9, atol=1e-11)


def test_128_token_rescaling_keeps_the_result():
    """A sequence long enough that kappa crosses 2^-40 several times (gamma^128 = 2^-96 per tile)."""
    gamma, N = 2.0 ** -0.75, 1000
    rng = np.random.default_rng(3)
    q, k, v = (rng.standard_normal((N, 4)) for _ in range(3))
    o, s = _tile_model_128(q, k, v, gamma)
    want_o, want_s = O.ret_chunkwise(q[None, None], k[None, None], v[None, None], np.array([gamma]), 64)
    np.testing.assert_allclose(o, want_o[0, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(s, want_s[0, 0], rtol=1e-9, atol=1e-11)


@pytest.mark.parametrize("gamma", [0.5, 0.75, 0.999])
@pytest.mark.parametrize("N", [64, 100, 257])
def test_64_token_merged_accumulator_equals_chunkwise(gamma, N):
    rng = np.random.default_rng(N + 7)
    q, k, v = (rng.standard_normal((N, d)) / 3 for d in (6, 6, 5))
    o, s = _merged_model_64(q, k, v, gamma)
    want_o, want_s = O.ret_chunkwise(q[None, None], k[None, None], v[None, None], np.array([gamma]), 64)
    np.testing.assert_allclose(o, want_o[0, 0], rtol=1e-9, atol=1e-11)
    np.testing.assert_allclose(s, want_s[0, 0], rtol=1e-9, atol=1e-11)


def test_merged_factors_stay_in_range():
    """For gamma in [1/2, 1] every factor of the merged 64-token form lies in [2^-64, 2^63],
    inside the normal range of bf16 and fp32."""
    for gamma in (0.5, 0.6, 0.9, 1.0):
        zp = gamma ** (63 - np.arange(64))
        factors = np.concatenate([zp, 1 / zp, [gamma ** 64]])
        assert factors.min() >= 2.0 ** -64 and factors.max() <= 2.0 ** 63


# ---------------------------------------------------------------- anti-causal tiles (a reversed kernel)
#
# The backward's dK and dV are anti-causal sums, R_m = sum_{n>=m} w_nm (a_m . b_n) c_n (dV: a=k, b=q, c=dO;
# dK: a=v, b=dO, c=q). Without reversing the sequence in memory they can be computed over the forward's
# tiles visited from the last to the first, carrying S' = sum over later tokens of w b_n^T c_n:
#   fixed gamma, a tile of L tokens, local index j:  row factor gamma^(L-j), key weight gamma^i,
#       state decay gamma^L, intra weights gamma^(i-j) for i >= j (upper triangle);
#   gated:  row factor exp(sum of g over (j, L-1]), key weight exp(sum of g over [0, i]),
#       state decay exp(sum of g over the tile), intra weights exp(sum of g over (j, i]).

def _anticausal_model(a, b, c, tile, gamma=None, g=None):
    N = a.shape[0]
    S = np.zeros((b.shape[1], c.shape[1]))
    out = np.zeros((N, c.shape[1]))
    starts = list(range(0, N, tile))
    for t0 in reversed(starts):
        L = min(tile, N - t0)
        A, Bm, C = a[t0:t0 + L], b[t0:t0 + L], c[t0:t0 + L]
        idx = np.arange(L)
        if g is None:
            row = gamma ** (L - idx)
            key = gamma ** idx
            decay = gamma ** L
            W = np.where(idx[None, :] >= idx[:, None], gamma ** np.maximum(idx[None, :] - idx[:, None], 0), 0.0)
        else:
            gl = g[t0:t0 + L]
            inc = np.cumsum(gl)                      # sum over [0, i]
            row = np.exp(inc[-1] - inc)              # sum over (j, L-1]
            key = np.exp(inc)
            decay = np.exp(inc[-1])
            W = np.where(idx[None, :] >= idx[:, None], np.exp(inc[None, :] - inc[:, None]), 0.0)
        scores = (A @ Bm.T) * W                      # [j, i]: (a_j . b_i) w_ji for i >= j
        out[t0:t0 + L] = scores @ C + row[:, None] * (A @ S)
        S = decay * S + (Bm * key[:, None]).T @ C
    return out


@pytest.mark.parametrize("N,tile", [(128, 64), (300, 64), (517, 128), (77, 128)])
@pytest.mark.parametrize("gated", [False, True])
def test_anticausal_tiles_give_dk_and_dv(N, tile, gated):
    rng = np.random.default_rng(N + tile)
    q, k = rng.standard_normal((N, 5)), rng.standard_normal((N, 5))
    v, do = rng.standard_normal((N, 6)), rng.standard_normal((N, 6))
    if gated:
        g = -np.abs(rng.standard_normal(N)) / 4
        want = O.gated_backward(q[None, None], k[None, None], v[None, None], g[None, None], do[None, None])
        dv = _anticausal_model(k, q, do, tile, g=g)
        dk = _anticausal_model(v, do, q, tile, g=g)
    else:
        gamma = 0.97
        want = O.ret_backward(q[None, None], k[None, None], v[None, None], np.array([gamma]), do[None, None])
        dv = _anticausal_model(k, q, do, tile, gamma=gamma)
        dk = _anticausal_model(v, do, q, tile, gamma=gamma)
    np.testing.assert_allclose(dv, want[2][0, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(dk, want[1][0, 0], rtol=1e-9, atol=1e-10)


# ---------------------------------------------------------------- the reversed kernel's own factors
#
# The time-reversed kernel references its carried state at the token before the current tile
# (the convention of the gated model above): R = sum_{n >= t0} w(n, t0 - 1) b_n^T c_n, so for
# fixed gamma the key weights are gamma^(i+1), the cross-term row factors gamma^(L-1-j) and the
# tile decay gamma^L. Its two fixed-decay bodies factor these like the forward's:
#   128-token body: zeta_i = gamma^(i+1), R = kappa T, kappa T = gamma^L R_next before the update,
#       o_j = (kappa / zeta_j) [ a_j T + sum_{i>=j} (a_j . b_i) zeta_i c_i / kappa ];
#   64-token merged accumulator: zeta'_i = gamma^i, the state copy scaled by gamma^(L-1),
#       o_j = (1 / zeta'_j) [ a_j (gamma^(L-1) R_next) + sum_{i>=j} zeta'_i (a_j . b_i) c_i ].

def _rev_tile_model_128(a, b, c, gamma, renorm=2.0 ** -40):
    N = a.shape[0]
    T = np.zeros((b.shape[1], c.shape[1]))
    kappa = 1.0
    out = np.zeros((N, c.shape[1]))
    for t0 in reversed(range(0, N, 128)):
        L = min(128, N - t0)
        A_, B_, C_ = a[t0:t0 + L], b[t0:t0 + L], c[t0:t0 + L]
        zeta = gamma ** (np.arange(L) + 1)
        if kappa * gamma ** L < renorm:
            T, kappa = kappa * T, 1.0
        kappa *= gamma ** L
        scores = np.triu(A_ @ B_.T)                  # i >= j
        zc = zeta[:, None] * C_ / kappa
        out[t0:t0 + L] = (kappa / zeta)[:, None] * (A_ @ T + scores @ zc)
        T = T + B_.T @ zc
    return out


def _rev_merged_model_64(a, b, c, gamma):
    N = a.shape[0]
    R = np.zeros((b.shape[1], c.shape[1]))
    out = np.zeros((N, c.shape[1]))
    for t0 in reversed(range(0, N, 64)):
        L = min(64, N - t0)
        zp = gamma ** np.arange(L)
        A_, B_, C_ = a[t0:t0 + L], b[t0:t0 + L], c[t0:t0 + L]
        P = np.triu(A_ @ B_.T) * zp[None, :]
        acc = A_ @ (gamma ** (L - 1) * R) + P @ C_
        out[t0:t0 + L] = acc / zp[:, None]
        R = gamma ** L * R + (B_ * (gamma ** (np.arange(L) + 1))[:, None]).T @ C_
    return out


@pytest.mark.parametrize("gamma", [0.999, 0.9, 2.0 ** -0.75])
@pytest.mark.parametrize("N", [128, 300, 517, 1100])
def test_reversed_128_token_factors_give_dk_and_dv(gamma, N):
    rng = np.random.default_rng(N + 11)
    q, k = rng.standard_normal((N, 5)) / 2, rng.standard_normal((N, 5)) / 2
    v, do = rng.standard_normal((N, 6)) / 2, rng.standard_normal((N, 6)) / 2
    want = O.ret_backward(q[None, None], k[None, None], v[None, None], np.array([gamma]), do[None, None])
    np.testing.assert_allclose(_rev_tile_model_128(k, q, do, gamma), want[2][0, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(_rev_tile_model_128(v, do, q, gamma), want[1][0, 0], rtol=1e-9, atol=1e-10)


@pytest.mark.parametrize("gamma", [0.5, 0.55, 0.999])
@pytest.mark.parametrize("N", [64, 100, 257])
def test_reversed_64_token_merged_factors_give_dk_and_dv(gamma, N):
    rng = np.random.default_rng(N + 13)
    q, k = rng.standard_normal((N, 5)) / 2, rng.standard_normal((N, 5)) / 2
    v, do = rng.standard_normal((N, 6)) / 2, rng.standard_normal((N, 6)) / 2
    want = O.ret_backward(q[None, None], k[None, None], v[None, None], np.array([gamma]), do[None, None])
    np.testing.assert_allclose(_rev_merged_model_64(k, q, do, gamma), want[2][0, 0], rtol=1e-9, atol=1e-10)
    np.testing.assert_allclose(_rev_merged_model_64(v, do, q, gamma), want[1][0, 0], rtol=1e-9, atol=1e-10)


def test_reversed_factors_stay_in_range():
    """128-token body (log2 gamma >= -0.75) and merged 64-token form (gamma >= 1/2): every
    factor of the reversed direction lies within the normal range of bf16 and fp32."""
    for gamma in (2.0 ** -0.75, 0.9, 1.0):
        zeta = gamma ** (np.arange(128) + 1)
        f = np.log2(np.concatenate([zeta, 1 / zeta, [gamma ** 128]]))
        assert f.min() >= -96 - 1e-9 and f.max() <= 96 + 1e-9
    for gamma in (0.5, 0.6, 1.0):
        zp = gamma ** np.arange(64)
        f = np.log2(np.concatenate([zp, 1 / zp, [gamma ** 63]]))
        assert f.min() >= -64 - 1e-9 and f.max() <= 63 + 1e-9
