"""Sequence-parallel chunkwise retention: one long sequence split across the ranks of
a process group, with one exchange of states.

The chunkwise recurrence ("RetNet retention mechanism" (aiqz.cc), section 块级循环;
the Gated RetNet page's cross_chunk state update) composes over consecutive segments:

    S_in(0) = state_in,    S_in(r + 1) = D_r S_in(r) + U_r,

with U_r the end state of segment r from a zero start and D_r its total decay. Rank r
holds segment r (its slice of the tokens, in rank order). It computes (U_r, log2 D_r)
with the state-only kernel, the ranks all-gather them (B*H*dk*dv*4 bytes per rank over
NCCL), every rank forms the start states with the prefix kernel, and rank r runs the
chunkwise kernel on its segment from S_in(r). The outputs are exactly the whole
sequence's outputs for that segment; S_in(R) is the final state, on every rank.

All arithmetic runs in the library's kernels; torch.distributed only moves states.
"""
from __future__ import annotations

import torch

from . import ret


class LibraryOps:
    """The three steps as calls of the C ABI (the only implementation the product uses)."""

    @staticmethod
    def state(k, v, decay, chunk, gated):
        return ret.chunkwise_state(k, v, decay, chunk, gated=gated)

    @staticmethod
    def prefix(seg_states, seg_log2_decay, state_in):
        return ret.state_prefix(seg_states, seg_log2_decay, state_in)

    @staticmethod
    def chunkwise(q, k, v, decay, chunk, state_in, gated):
        if gated:
            return ret.gated_ret_chunkwise(q, k, v, decay, chunk, state_in=state_in)
        return ret.ret_chunkwise(q, k, v, decay, chunk, state_in=state_in)


def sequence_parallel_chunkwise(q, k, v, decay, chunk, gated=False, state_in=None, group=None, ops=None):
    """This rank's part of chunkwise retention over a sequence split across `group`.

    q, k [B, H, N_r, dk], v [B, H, N_r, dv]: this rank's tokens (rank order = sequence
    order; segments may differ in length). decay: gamma [H], or this rank's gates
    g [B, H, N_r] with gated=True. state_in: the sequence's initial state [B, H, dk, dv]
    (the same on every rank) or None. Returns (o [B, H, N_r, dv], final state after the
    whole sequence). `ops` replaces the library's kernels (tests only).
    """
    import torch.distributed as dist
    ops = ops or LibraryOps
    single = not dist.is_initialized()  # one process: the whole sequence is one segment
    world = 1 if single else dist.get_world_size(group)
    rank = 0 if single else dist.get_rank(group)
    U, ld = ops.state(k, v, decay, chunk, gated)
    all_U = torch.empty((world,) + tuple(U.shape), dtype=U.dtype, device=U.device)
    all_ld = torch.empty((world,) + tuple(ld.shape), dtype=ld.dtype, device=ld.device)
    if single:
        all_U[0].copy_(U)
        all_ld[0].copy_(ld)
    else:
        dist.all_gather(list(all_U.unbind(0)), U.contiguous(), group=group)
        dist.all_gather(list(all_ld.unbind(0)), ld.contiguous(), group=group)
    starts, end = ops.prefix(all_U, all_ld, state_in)
    o = ops.chunkwise(q, k, v, decay, chunk, starts[rank].contiguous(), gated)
    return o, end
