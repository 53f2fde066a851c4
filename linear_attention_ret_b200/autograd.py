"""Chunkwise retention as a differentiable torch op: the forward is ret_chunkwise (or
gated_ret_chunkwise), the backward is ret_chunkwise_backward (or its gated form). Both run
in the library's kernels; this module only routes tensors. The gradients are those of the
operator from a zero initial state ("RetNet retention mechanism" page, 保留机制初识;
the Gated RetNet page's parallel_gate_retention weights for the gated form)."""
from __future__ import annotations

import torch

from . import ret


class ChunkwiseRetention(torch.autograd.Function):
    """o = retention(q, k, v; decay). decay: gamma [H] (gated=False) or g [B, H, N] (gated=True)."""

    @staticmethod
    def forward(ctx, q, k, v, decay, chunk: int, gated: bool):
        q, k, v, decay = (t.contiguous() for t in (q, k, v, decay))
        if gated:
            o = ret.gated_ret_chunkwise(q, k, v, decay, chunk)
        else:
            o = ret.ret_chunkwise(q, k, v, decay, chunk)
        ctx.save_for_backward(q, k, v, decay)
        ctx.chunk, ctx.gated = chunk, gated
        return o

    @staticmethod
    def backward(ctx, do):
        q, k, v, decay = ctx.saved_tensors
        want_decay = ctx.needs_input_grad[3]
        dq, dk, dv, dd = ret.chunkwise_backward(q, k, v, decay, do.contiguous(), ctx.chunk, gated=ctx.gated,
                                                ddecay=want_decay)
        return dq, dk, dv, dd, None, None


def chunkwise_retention(q, k, v, decay, chunk: int = 64, gated: bool = False):
    """Differentiable chunkwise retention (see ChunkwiseRetention); o has v's layout and q's dtype."""
    return ChunkwiseRetention.apply(q, k, v, decay, chunk, gated)
