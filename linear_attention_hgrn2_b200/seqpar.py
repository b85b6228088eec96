"""One sequence across several GPUs: sequence parallelism for the HGRN2 recurrence.

Each rank of a process group holds one contiguous slice of the tokens of every
(batch, head) sequence, in rank order.  Over a slice the recurrence
("HGRN2: Gated Linear RNNs with State Expansion", §3.2) is affine in the state
entering the slice, and its backward is affine in the gradient leaving it:

    S_out    = Diag(g) S_in     + U        (forward map)
    dL/dS_in = Diag(g) dL/dS_out + W       (backward map)

so a step is: every rank computes its slice's maps (hgrn2_state_map /
hgrn2_state_map_bwd), one all-gather exchanges them, an fp32 scan of the maps in
rank order (reverse rank order for the backward) gives each rank its boundary
state (hgrn2_affine_scan), and each rank runs the ordinary chunkwise forward or
backward on its slice from those boundary states.  The exchange is the one
collective on the path: B*H*(dk + dk*dv) float32 per rank and direction (64.5 KB
per 128 x 128 head).  The pages cite linear-attention sequence parallelism
(LASP) for running the chunkwise state passing across devices.

Every compute step runs in the library's kernels; this module only slices,
exchanges (torch.distributed) and orders.  The phases are also exposed one by
one (``*_local`` then ``*_finish``), so that all ranks can be emulated one after
the other in a single process.  ``ops`` selects the implementation of the
compute steps (the library by default).
"""
from __future__ import annotations

from dataclasses import dataclass

import torch


class LibraryOps:
    """The compute steps of a sequence-parallel pass, on the library's kernels."""

    @staticmethod
    def state_map(log_f, i):
        from . import state_map
        return state_map(log_f, i)

    @staticmethod
    def state_map_bwd(q, log_f, dO):
        from . import state_map_bwd
        return state_map_bwd(q, log_f, dO)

    @staticmethod
    def affine_scan(g, M, first, count, step, init=None):
        from . import affine_scan
        return affine_scan(g, M, first, count, step, init=init)

    @staticmethod
    def fwd(q, log_f, i, h0, saved=None, chunk=64):
        from . import fwd
        return fwd(q, log_f, i, h0, want_hT=True, chunk=chunk, saved=saved)

    @staticmethod
    def bwd(q, log_f, i, dO, h0, dhT, want_dh0, saved=None, chunk=64):
        from . import bwd
        return bwd(q, log_f, i, dO, h0, dhT, want_dh0=want_dh0, chunk=chunk, saved=saved)


@dataclass
class SliceContext:
    """What a rank keeps from its forward for its backward."""
    g_all: torch.Tensor      # [R, B, H, dk]: every slice's decay product
    S_in: torch.Tensor       # [B, H, dk, dv]: the state entering this rank's slice
    rank: int
    world: int


# ------------------------------------------------------------------ phases (one rank each)
def fwd_local(q, log_f, i, ops=LibraryOps):
    """This slice's forward map (g, U)."""
    return ops.state_map(log_f, i)


def fwd_finish(q, log_f, i, g_all, U_all, rank, h0=None, ops=LibraryOps, saved=None, chunk=64):
    """Given every slice's map (stacked in rank order): the state entering this slice (scan of
    the maps of the ranks before it from h0), this slice's output from it, and the state after
    the whole sequence (scan of all maps).  Returns (o, hT, context)."""
    R = g_all.shape[0]
    S_in = ops.affine_scan(g_all, U_all, 0, rank, 1, init=h0)
    o, _ = ops.fwd(q, log_f, i, S_in, saved=saved, chunk=chunk)
    hT = ops.affine_scan(g_all, U_all, 0, R, 1, init=h0)
    return o, hT, SliceContext(g_all, S_in, rank, R)


def bwd_local(q, log_f, dO, ops=LibraryOps):
    """This slice's backward map W (its g is the forward's)."""
    return ops.state_map_bwd(q, log_f, dO)[1]


def bwd_finish(q, log_f, i, dO, ctx: SliceContext, W_all, dhT=None, ops=LibraryOps, saved=None, chunk=64):
    """Given every slice's backward map: the gradient leaving this slice (scan of the maps of
    the ranks after it, last first, from dhT), then this slice's gradients from its boundary
    states.  Returns (dq, dlog_f, di, dh0): dh0 (the gradient of the sequence's initial state)
    on rank 0, None elsewhere."""
    R, r = ctx.world, ctx.rank
    dS_out = ops.affine_scan(ctx.g_all, W_all, R - 1, R - 1 - r, -1, init=dhT)
    dq, dlf, di, dh0 = ops.bwd(q, log_f, i, dO, ctx.S_in, dS_out, want_dh0=(r == 0), saved=saved, chunk=chunk)
    return dq, dlf, di, (dh0 if r == 0 else None)


# ------------------------------------------------------------------ across a process group
def _all_gather(t: torch.Tensor, group) -> torch.Tensor:
    """[world, *t.shape]: every rank's t in rank order."""
    import torch.distributed as dist
    parts = [torch.empty_like(t) for _ in range(dist.get_world_size(group))]
    dist.all_gather(parts, t.contiguous(), group=group)
    return torch.stack(parts)


def forward(q, log_f, i, h0=None, group=None, ops=LibraryOps, saved=None, chunk=64):
    """Sequence-parallel forward.  Each rank passes its own slice of q, log_f, i
    ([B, T_rank, H, *], slices in rank order) and the same h0 (the state before the whole
    sequence, or None).  Returns (o of this slice, hT of the whole sequence, context)."""
    import torch.distributed as dist
    rank = dist.get_rank(group)
    g, U = fwd_local(q, log_f, i, ops)
    return fwd_finish(q, log_f, i, _all_gather(g, group), _all_gather(U, group), rank, h0, ops, saved, chunk)


def backward(q, log_f, i, dO, ctx: SliceContext, dhT=None, group=None, ops=LibraryOps, saved=None, chunk=64):
    """Sequence-parallel backward of forward(): this rank's slice of dO, and dhT (the gradient
    of the whole sequence's final state, the same on every rank, or None).  Returns this slice's
    (dq, dlog_f, di) and dh0 on rank 0."""
    W = bwd_local(q, log_f, dO, ops)
    return bwd_finish(q, log_f, i, dO, ctx, _all_gather(W, group), dhT, ops, saved, chunk)
