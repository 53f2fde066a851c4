"""Property checks of the oracle over randomly drawn shapes, chunk sizes and decays (the
fixed-case pins are in test_oracle_pins.py): the pages' three forms agree ("RetNet retention
mechanism" page, 并行训练 / 递归推理 / 块级循环; the Gated RetNet page's parallel, chunk and
recurrent gate retention), a sequence split anywhere composes through the state, and the
backward agrees with a directional finite difference of the forward."""
import numpy as np
from hypothesis import given, settings, strategies as st

from oracle import oracle as O

shapes = st.tuples(st.integers(1, 2), st.integers(1, 3), st.integers(1, 40), st.integers(1, 6), st.integers(1, 6))


def _draw(seed, B, H, N, dk, dv):
    rng = np.random.default_rng(seed)
    return (rng.standard_normal((B, H, N, dk)), rng.standard_normal((B, H, N, dk)),
            rng.standard_normal((B, H, N, dv)), rng)


@settings(max_examples=40, deadline=None)
@given(shapes, st.integers(1, 45), st.lists(st.floats(0.0, 1.0), min_size=3, max_size=3), st.integers(0, 2**31))
def test_forms_agree(shape, chunk, gammas, seed):
    B, H, N, dk, dv = shape
    q, k, v, rng = _draw(seed, B, H, N, dk, dv)
    gam = np.array(gammas[:H])
    S0 = rng.standard_normal((B, H, dk, dv))
    par = O.ret_parallel(q, k, v, gam)
    rec_o, rec_s = O.ret_recurrent(q, k, v, gam)
    chk_o, chk_s = O.ret_chunkwise(q, k, v, gam, chunk)
    np.testing.assert_allclose(rec_o, par, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(chk_o, par, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(chk_s, rec_s, rtol=1e-9, atol=1e-9)
    # with an initial state, chunkwise and recurrent still agree
    a, sa = O.ret_recurrent(q, k, v, gam, state_in=S0)
    b, sb = O.ret_chunkwise(q, k, v, gam, chunk, state_in=S0)
    np.testing.assert_allclose(b, a, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(sb, sa, rtol=1e-9, atol=1e-9)


@settings(max_examples=40, deadline=None)
@given(shapes, st.integers(1, 45), st.floats(0.0, 3.0), st.integers(0, 2**31))
def test_gated_forms_agree(shape, chunk, strength, seed):
    B, H, N, dk, dv = shape
    q, k, v, rng = _draw(seed, B, H, N, dk, dv)
    g = -np.abs(rng.standard_normal((B, H, N))) * strength
    par = O.gated_parallel(q, k, v, g)
    rec_o, rec_s = O.gated_recurrent(q, k, v, g)
    chk_o, chk_s = O.gated_chunkwise(q, k, v, g, chunk)
    np.testing.assert_allclose(rec_o, par, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(chk_o, par, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(chk_s, rec_s, rtol=1e-9, atol=1e-9)


@settings(max_examples=30, deadline=None)
@given(shapes, st.integers(1, 20), st.data(), st.integers(0, 2**31))
def test_split_anywhere_composes(shape, chunk, data, seed):
    B, H, N, dk, dv = shape
    q, k, v, rng = _draw(seed, B, H, N, dk, dv)
    gam = rng.uniform(0.0, 1.0, H)
    cut = data.draw(st.integers(0, N))
    whole_o, whole_s = O.ret_chunkwise(q, k, v, gam, chunk)
    o1, s1 = O.ret_chunkwise(q[:, :, :cut], k[:, :, :cut], v[:, :, :cut], gam, chunk)
    o2, s2 = O.ret_chunkwise(q[:, :, cut:], k[:, :, cut:], v[:, :, cut:], gam, chunk, state_in=s1)
    np.testing.assert_allclose(np.concatenate([o1, o2], axis=2), whole_o, rtol=1e-9, atol=1e-9)
    np.testing.assert_allclose(s2, whole_s, rtol=1e-9, atol=1e-9)


@settings(max_examples=25, deadline=None)
@given(st.tuples(st.integers(1, 2), st.integers(1, 2), st.integers(1, 9), st.integers(1, 4), st.integers(1, 4)),
       st.booleans(), st.integers(0, 2**31))
def test_backward_directional_derivative(shape, gated, seed):
    B, H, N, dk, dv = shape
    q, k, v, rng = _draw(seed, B, H, N, dk, dv)
    do = rng.standard_normal((B, H, N, dv))
    decay = -np.abs(rng.standard_normal((B, H, N))) if gated else rng.uniform(0.2, 1.0, H)
    dirs = [rng.standard_normal(t.shape) for t in (q, k, v, decay)]
    fwd = O.gated_brute if gated else O.ret_brute
    loss = lambda s: float(np.sum(do * fwd(*(t + s * d for t, d in zip((q, k, v, decay), dirs)))))
    eps = 1e-5
    fd = (loss(eps) - loss(-eps)) / (2 * eps)
    grads = (O.gated_backward if gated else O.ret_backward)(q, k, v, decay, do)
    an = sum(float(np.sum(g * d)) for g, d in zip(grads, dirs))
    assert abs(fd - an) <= 1e-6 * (1 + abs(an)), (fd, an)
