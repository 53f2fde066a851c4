"""B200-native (sm_100a) RetNet retention operator.

The compute lives in libret.so (C ABI, include/ret.h); `ret` is its thin
binding. Importing the package does not load the library: call
``linear_attention_ret_b200.ret.load()`` (the binding's functions do it).

What the binding offers (CUDA tensors in, CUDA tensors out; q, k [B, H, N, dk],
v and o [B, H, N, dv], states [B, H, dk, dv] fp32, bf16 or fp32 inputs):

* ``ret.ret_chunkwise`` / ``ret.gated_ret_chunkwise``: chunkwise retention with a
  fixed decay per head (gamma [H]) or a per-token log-decay (g [B, H, N]), with an
  optional initial state and final state (prefill).
* ``ret.ret_recurrent_step`` / ``ret.gated_ret_recurrent_step``: one decode step,
  updating the state in place.
* ``ret.ret_parallel``: the parallel form, for checking.
* ``ret.chunkwise_backward``: dq, dk, dv and dgamma (or dg) of either chunkwise form;
  ``autograd.chunkwise_retention`` wraps forward and backward as a differentiable torch op.
* ``ret.msr_norm_gate``: the output epilogue, swish(gate) * per-head RMSNorm(o),
  token-major.
* ``ret.chunkwise_state`` and ``ret.state_prefix``: segment end states and start
  states for a sequence split across calls or GPUs; ``seqpar.sequence_parallel_chunkwise``
  runs the whole split over a torch.distributed group.
* ``ret.ret_chunkwise_host`` / ``ret.gated_ret_chunkwise_host`` and
  ``ret.chunkwise_backward_host``: the forward and the backward on host (CPU) tensors,
  page-locked for overlap; the library copies them in and the results out, pipelined
  with the compute over groups of heads.
"""
__all__ = ["ret", "inputs", "build", "seqpar", "autograd"]
