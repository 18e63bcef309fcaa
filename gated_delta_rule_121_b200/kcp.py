"""KDA context parallelism across ranks (KCP).

The digest's co-design section ("KDA context parallelism (KCP)" paragraph)
splits one long sequence over the ranks of a context-parallel group.  With
``M_t = (I - beta_t k_t k_t^T) Diag(alpha_t)`` the recurrence reads
``S_t = M_t S_{t-1} + beta_t k_t v_t^T``, so the effect of a rank's tokens on
the state is the pair (M, S~): the rank's transition and its state from a zero
start.  Both come from the local tokens alone.  One fixed-size all-gather of
the pairs lets every rank compose the incoming state of its own tokens by a
prefix over the ranks before it, and the final state of the sequence.

Per rank (tokens [B, T_local, H, d] of B sequences, rank r holding the r-th
consecutive slice of every sequence):

    pieces   kda_segment_fwd: zero-start outputs o~, S~, qhat, M      (GPU)
    gather   all_gather of M [B,H,dk,dk] and S~ [B,H,dk,dv]           (NCCL)
    compose  kda_state_compose over the ranks in rank order           (GPU)
    finish   kda_output_correct: o = o~ + S_in^T qhat                 (GPU)

Every rank returns its own outputs and the sequence's final state (the same
on every rank).  The exchange is 4 B x H x dk x (dk + dv) per sequence per
rank, independent of the sequence length.

The step functions take an ``ops`` object whose defaults are this package's
CUDA entry points; the host logic (which rank holds which piece, the order of
the gathered pieces) is the same whatever computes the pieces.
"""
from __future__ import annotations

import types

import torch

from . import kda_output_correct, kda_segment_fwd, kda_state_compose

CUDA_OPS = types.SimpleNamespace(segment_fwd=kda_segment_fwd, state_compose=kda_state_compose,
                                 output_correct=kda_output_correct)


def kcp_pieces(q, k, v, log_alpha, beta, ops=CUDA_OPS):
    """The rank-local quantities: (out_zero, qhat, transition, state_zero)."""
    out_zero, state_zero, qhat, transition = ops.segment_fwd(q, k, v, log_alpha, beta)
    return out_zero, qhat, transition, state_zero


def kcp_combine(transitions, states_zero, world, init_state=None, ops=CUDA_OPS):
    """Incoming state of every rank's piece and the final state, from the
    gathered pieces in rank order ([world * B, H, ...], rank-major)."""
    return ops.state_compose(transitions, states_zero, world, init_state=init_state, rank_major=True)


def kcp_finish(out_zero, qhat, state_in_rank, dtype, ops=CUDA_OPS):
    """This rank's outputs once its incoming states are known."""
    return ops.output_correct(out_zero, qhat, state_in_rank, dtype=dtype)


def all_gather_rank_major(t, group=None):
    """[world * B, ...] from every rank's [B, ...] (one fixed-size all-gather)."""
    import torch.distributed as dist
    world = dist.get_world_size(group)
    out = torch.empty((world * t.shape[0],) + tuple(t.shape[1:]), dtype=t.dtype, device=t.device)
    if dist.get_backend(group) == "nccl":
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    else:
        parts = list(out.chunk(world, 0))
        dist.all_gather(parts, t.contiguous(), group=group)
        out = torch.cat(parts, 0)
    return out


def kcp_fwd(q, k, v, log_alpha, beta, init_state=None, group=None, ops=CUDA_OPS, gather=None):
    """KDA forward of sequences whose tokens are split over the ranks of
    ``group``: this rank passes its consecutive slice [B, T_local, H, d] of
    each of the B sequences (rank 0 the first slice); ``init_state`` is the
    state before rank 0's slice (the same tensor on every rank, or None).
    Returns (this rank's outputs, the final state of every sequence)."""
    import torch.distributed as dist
    rank, world = dist.get_rank(group), dist.get_world_size(group)
    gather = gather or (lambda t: all_gather_rank_major(t, group))
    out_zero, qhat, transition, state_zero = kcp_pieces(q, k, v, log_alpha, beta, ops)
    transitions = gather(transition)
    states_zero = gather(state_zero)
    state_in, final_state = kcp_combine(transitions, states_zero, world, init_state, ops)
    B = q.shape[0]
    out = kcp_finish(out_zero, qhat, state_in[rank * B:(rank + 1) * B].contiguous(), q.dtype, ops)
    return out, final_state
