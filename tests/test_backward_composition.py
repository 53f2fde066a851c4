"""The algebra the GPU backward is built on, checked on the CPU with the oracle's forward
standing in for the kernels (the same steps the library takes, in fp64):

  dQ = forward(dO, V, K), summed over pieces of the dv contraction;
  dK = rev(forward(rev V, rev dO, rev Q)), dV = rev(forward(rev K, rev Q, rev dO)), with the
  gated form's reversed gates shifted by one (g'_0 = 0, g'_i = g_{N-i});
  a_t = q_t . dQ_t - k_t . dK_t, dgamma_h = (1/gamma_h) sum_{b,t} t a_t, dg_t = sum_{u>=t} a_u;

against the oracle's gradients by definition (themselves pinned to finite differences).
"""
import numpy as np
import pytest

from oracle import oracle as O

B, H, N, DK, DV, CHUNK = 2, 2, 37, 5, 7, 8
PIECES = [(0, 4), (4, 7)]  # the dv contraction in two pieces, as the library splits dv > 256


def _inputs(seed):
    rng = np.random.default_rng(seed)
    q, k = rng.standard_normal((B, H, N, DK)), rng.standard_normal((B, H, N, DK))
    v, do = rng.standard_normal((B, H, N, DV)), rng.standard_normal((B, H, N, DV))
    return q, k, v, do, rng


def _rev(x):
    return np.ascontiguousarray(x[:, :, ::-1])


def _composed(q, k, v, do, decay, gated):
    fwd = (lambda a, b, c, d: O.gated_chunkwise(a, b, c, d, CHUNK)[0]) if gated else \
        (lambda a, b, c, d: O.ret_chunkwise(a, b, c, d, CHUNK)[0])
    if gated:
        rdec = np.zeros_like(decay)
        rdec[:, :, 1:] = decay[:, :, :0:-1]  # g'_i = g_{N-i} for i >= 1, g'_0 = 0
    else:
        rdec = decay
    dq = sum(fwd(do[..., a:b], v[..., a:b], k, decay) for a, b in PIECES)
    dk = _rev(sum(fwd(_rev(v)[..., a:b], _rev(do)[..., a:b], _rev(q), rdec) for a, b in PIECES))
    dv = _rev(fwd(_rev(k), _rev(q), _rev(do), rdec))
    a_t = np.einsum("bhnd,bhnd->bhn", q, dq) - np.einsum("bhnd,bhnd->bhn", k, dk)
    if gated:
        dd = np.cumsum(a_t[:, :, ::-1], axis=2)[:, :, ::-1]
    else:
        t = np.arange(N)
        dd = (a_t * t).sum(axis=(0, 2)) / decay
    return dq, dk, dv, dd


def test_fixed_gamma_composition_equals_the_gradients():
    q, k, v, do, _ = _inputs(50)
    gam = np.array([0.93, 0.6])
    got = _composed(q, k, v, do, gam, gated=False)
    want = O.ret_backward(q, k, v, gam, do)
    for g, w, name in zip(got, want, ("dq", "dk", "dv", "dgamma")):
        np.testing.assert_allclose(g, w, rtol=1e-10, atol=1e-10, err_msg=name)


def test_gated_composition_equals_the_gradients():
    q, k, v, do, rng = _inputs(51)
    g = -np.abs(rng.standard_normal((B, H, N))) / 3.0
    got = _composed(q, k, v, do, g, gated=True)
    want = O.gated_backward(q, k, v, g, do)
    for a, w, name in zip(got, want, ("dq", "dk", "dv", "dg")):
        np.testing.assert_allclose(a, w, rtol=1e-10, atol=1e-10, err_msg=name)


def test_unshifted_gate_reversal_is_wrong():
    """The shift matters: reversing the gates without it gives different dk."""
    q, k, v, do, rng = _inputs(52)
    g = -np.abs(rng.standard_normal((B, H, N))) / 3.0
    wrong = O.gated_chunkwise(_rev(v), _rev(do), _rev(q), _rev(g), CHUNK)[0]
    dk_wrong = _rev(wrong)
    dk = O.gated_backward(q, k, v, g, do)[1]
    assert not np.allclose(dk_wrong, dk, rtol=1e-6, atol=1e-8)
