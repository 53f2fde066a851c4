"""The binding's argument checks on the CPU: every call the tests, the bench and the
sequence-parallel orchestration make passes the shape and dtype checks (host tensors then
stop at the CUDA check), and mismatched shapes or dtypes are refused before any pointer
reaches the library."""
import pytest
import torch

from linear_attention_ret_b200 import ret

B, H, N, DK, DV = 2, 3, 10, 8, 12
bf, f32 = torch.bfloat16, torch.float32


def _passes_shape_checks(fn, *args, **kw):
    with pytest.raises(ValueError, match="CUDA tensors"):
        fn(*args, **kw)


def _refused(fn, match, *args, **kw):
    with pytest.raises(ValueError, match=match):
        fn(*args, **kw)


def seq(dtype=bf):
    return (torch.zeros(B, H, N, DK, dtype=dtype), torch.zeros(B, H, N, DK, dtype=dtype),
            torch.zeros(B, H, N, DV, dtype=dtype))


GAM, G = torch.full((H,), 0.9), torch.zeros(B, H, N)
S = torch.zeros(B, H, DK, DV)


def test_valid_calls_pass_the_checks():
    q, k, v = seq()
    _passes_shape_checks(ret.ret_parallel, *seq(f32), GAM)
    _passes_shape_checks(ret.ret_chunkwise, q, k, v, GAM, 64)
    _passes_shape_checks(ret.ret_chunkwise, q, q, v, GAM, 64, state_in=S, state_out=S,
                         o=torch.zeros(B, H, N, DV, dtype=bf))
    _passes_shape_checks(ret.ret_chunkwise_noalloc, q, k, v, GAM, 64, state_in=S, state_out=S.clone())
    _passes_shape_checks(ret.gated_ret_chunkwise, q, k, v, G, 64, state_in=S)
    qs, ks, vs = q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous()
    _passes_shape_checks(ret.ret_recurrent_step, qs, ks, vs, GAM, S, o=torch.zeros(B, H, DV, dtype=bf))
    _passes_shape_checks(ret.gated_ret_recurrent_step, qs, ks, vs, torch.zeros(B, H), S)
    _passes_shape_checks(ret.chunkwise_state, k, v, GAM, 64)
    _passes_shape_checks(ret.chunkwise_state, k, v, G, 64, gated=True)
    _passes_shape_checks(ret.state_prefix, torch.zeros(4, B, H, DK, DV), torch.zeros(4, B, H), S)
    _passes_shape_checks(ret.state_prefix, torch.zeros(1, B, H, DK, DV), torch.zeros(1, B, H))
    _passes_shape_checks(ret.chunkwise_backward, q, k, v, GAM, torch.zeros(B, H, N, DV, dtype=bf), 64)
    _passes_shape_checks(ret.chunkwise_backward, q, k, v, G, torch.zeros(B, H, N, DV, dtype=bf), 64, gated=True,
                         ddecay=False)
    _passes_shape_checks(ret.msr_norm_gate, v, torch.zeros(B, N, H, DV, dtype=bf))


def test_mismatches_are_refused():
    q, k, v = seq()
    _refused(ret.ret_chunkwise, "k must have shape", q, k[:, :, :5].contiguous(), v, GAM, 64)
    _refused(ret.ret_chunkwise, "v must be", q, k, v.float(), GAM, 64)
    _refused(ret.ret_chunkwise, "gamma must have shape", q, k, v, torch.full((H - 1,), 0.9), 64)
    _refused(ret.ret_chunkwise, "gamma must be", q, k, v, GAM.double(), 64)
    _refused(ret.ret_chunkwise, "state_in must have shape", q, k, v, GAM, 64, state_in=torch.zeros(B, H, DK, DK))
    _refused(ret.ret_chunkwise, "state_out must be", q, k, v, GAM, 64, state_out=S.to(bf))
    _refused(ret.ret_chunkwise, "o must have shape", q, k, v, GAM, 64, o=torch.zeros(B, H, N, DK, dtype=bf))
    _refused(ret.gated_ret_chunkwise, "g must have shape", q, k, v, torch.zeros(B, H, N + 1), 64)
    _refused(ret.ret_parallel, "q must have 4 dimensions", q[0], k[0], v[0], GAM)
    qs, ks, vs = q[:, :, 0].contiguous(), k[:, :, 0].contiguous(), v[:, :, 0].contiguous()
    _refused(ret.ret_recurrent_step, "state must have shape", qs, ks, vs, GAM, torch.zeros(B, H, DV, DK))
    _refused(ret.gated_ret_recurrent_step, "g must have shape", qs, ks, vs, torch.zeros(H), S)
    _refused(ret.chunkwise_state, "gamma must have shape", k, v, G, 64)
    _refused(ret.state_prefix, "seg_log2_decay must have shape", torch.zeros(4, B, H, DK, DV), torch.zeros(3, B, H))
    _refused(ret.chunkwise_backward, "dout must have shape", q, k, v, GAM, torch.zeros(B, H, N, DK, dtype=bf), 64)
    _refused(ret.msr_norm_gate, "gate must be", v, torch.zeros(B, H, N, DV, dtype=bf))
