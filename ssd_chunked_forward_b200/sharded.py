"""Sequence-sharded forward and backward: one sequence split along T over the
ranks of a process group (rank r holds tokens [r T/W, (r+1) T/W) of every
batch row).

Each rank first forms the state its segment builds from a zero start and the
segment's total log-decay (ssd.segment_state: one pass over x, a and Bm, no
outputs), the ranks exchange those in one all-gather, every rank combines
them into the state entering its own segment, and then runs its segment's
forward once, from that state -- the passing of one summarised state between
pieces, as the chunked algorithm does between chunks ("State Space Duality",
"Two algorithms for one operator"), one level up.  The backward runs the same
exchange for the entering states, then the adjoint's exchange in the other
direction (sequence_sharded_backward).  All arithmetic runs in the library's
kernels (ssd.segment_state, ssd.state_combine, ssd.forward, ssd.backward) and
in the collectives; this module only orders the calls.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist

from . import ssd


@dataclass
class SegmentOps:
    """The computations a rank performs; the defaults are the library's (tests
    on machines without a GPU substitute the fp64 oracle)."""
    forward: Callable = None        # (x, a, Bm, Cm, D, chunk, initial_state) -> (y, final)
    segment_state: Callable = None  # (x, a, Bm, chunk) -> (final state from zero, total log-decay)
    state_combine: Callable = None  # (finals [W,...], totals [W,...], h0) -> h_in [W+1,...]
    backward: Callable = None       # (x, a, Bm, Cm, D, dy, chunk, dfinal, init) -> dict of gradients

    def __post_init__(self):
        if self.forward is None:
            self.forward = lambda x, a, Bm, Cm, D, chunk, init: ssd.forward(
                x, a, Bm, Cm, D, chunk, initial_state=init)
        if self.segment_state is None:
            self.segment_state = lambda x, a, Bm, chunk: ssd.segment_state(x, a, Bm, chunk)
        if self.state_combine is None:
            self.state_combine = ssd.state_combine
        if self.backward is None:
            self.backward = lambda x, a, Bm, Cm, D, dy, chunk, dfinal, init: ssd.backward(
                x, a, Bm, Cm, D, dy, chunk, dfinal=dfinal, initial_state=init)


def _all_gather(t: torch.Tensor, group) -> torch.Tensor:
    """[W, *t.shape] on every rank (one collective)."""
    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    if t.is_cuda:
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


def _entering_states(x, a, Bm, chunk, group, initial_state, ops):
    """Each segment's total decay and the state entering every segment
    (h_in [W+1, ...]; h_in[W] is the sequence's final state), through one
    all-gather of the segments' own states (from zero) and totals."""
    fin, tot = ops.segment_state(x, a, Bm, chunk)
    packed = torch.cat([fin.reshape(-1), tot.reshape(-1).to(fin.dtype)])
    gathered = _all_gather(packed, group)
    nf = fin.numel()
    finals = gathered[:, :nf].reshape((gathered.shape[0],) + tuple(fin.shape)).contiguous()
    totals = gathered[:, nf:].reshape((gathered.shape[0],) + tuple(tot.shape)).contiguous()
    return totals, ops.state_combine(finals, totals, initial_state)


def sequence_sharded_forward(x, a, Bm, Cm, D, chunk, *, group=None, initial_state=None,
                             ops: SegmentOps | None = None):
    """This rank's segment of y, and the final state of the whole sequence.

    x [B,T_r,H,P], a [B,T_r,H] (or [B,T_r,H,N]), Bm/Cm [B,T_r,G,N] hold this
    rank's tokens; initial_state [B,H,N,P] (optional, the same on every rank)
    enters the first segment.  Every rank takes part in the same single
    all-gather (of the segment states and of the total decays, packed), and
    runs its forward once, from the state entering its segment."""
    ops = ops or SegmentOps()
    rank = dist.get_rank(group)
    _, h_in = _entering_states(x, a, Bm, chunk, group, initial_state, ops)
    init = h_in[rank].contiguous() if (rank > 0 or initial_state is not None) else None
    y, _ = ops.forward(x, a, Bm, Cm, D, chunk, init)
    return y, h_in[-1]


def sequence_sharded_backward(x, a, Bm, Cm, D, dy, chunk, *, group=None, initial_state=None,
                              dfinal=None, ops: SegmentOps | None = None):
    """Gradients of sum(dy * y) + <dfinal, final state> over the whole
    sequence, for this rank's segment (dx, da, dBm, dCm) and for the shared
    inputs (dD, d initial state; the same on every rank).

    The state entering each segment comes from the forward's exchange.  The
    adjoint runs the other way: the adjoint at the end of segment r is the
    adjoint entering segment r+1, which is that segment's own contribution
    (its backward with no loss on its end, started from its entering state)
    plus its total decay times the adjoint at its end -- the forward's
    combine run over the segments in reverse order, from dfinal.  So each
    rank runs its backward once with no end loss, one all-gather exchanges
    the entering-state adjoints and one all-reduce sums the segments' shares
    of dD, every rank combines the adjoints, and the ranks before the last
    (or all, given dfinal) rerun their backward with the adjoint at their end."""
    ops = ops or SegmentOps()
    rank = dist.get_rank(group)
    totals, h_in = _entering_states(x, a, Bm, chunk, group, initial_state, ops)
    init = h_in[rank].contiguous()
    g = ops.backward(x, a, Bm, Cm, D, dy, chunk, None, init)
    din = g["dinit"]
    dinits = _all_gather(din, group)
    world = dinits.shape[0]
    # dD: every segment's share, summed by the collective itself
    dD_all = g["dD"].clone()
    dist.all_reduce(dD_all, op=dist.ReduceOp.SUM, group=group)
    # reverse combine: adj[s] = adjoint at the end of segment W-1-s; adj[W] = d initial
    adj = ops.state_combine(dinits.flip(0).contiguous(), totals.flip(0).contiguous(), dfinal)
    g_end = adj[world - 1 - rank].contiguous()
    if rank < world - 1 or dfinal is not None:
        g = ops.backward(x, a, Bm, Cm, D, dy, chunk, g_end, init)
    return {"dx": g["dx"], "da": g["da"], "dBm": g["dBm"], "dCm": g["dCm"],
            "dD": dD_all, "dinit": adj[world]}
