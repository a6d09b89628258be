"""Sequence-sharded forward: one sequence split along T over the ranks of a
process group (rank r holds tokens [r T/W, (r+1) T/W) of every batch row).

Each rank runs its segment from a zero state, the ranks exchange each
segment's final state and total log-decay in one all-gather, every rank
combines them into the state entering its own segment, and the ranks after
the first rerun their segment from that state -- the passing of one
summarised state between pieces, as the chunked algorithm does between chunks
("State Space Duality", "Two algorithms for one operator"), one level up.
All arithmetic runs in the library's kernels (ssd.forward, ssd.decay_total,
ssd.state_combine); this module only orders the calls and the collective.
"""
from __future__ import annotations

from dataclasses import dataclass
from typing import Callable

import torch
import torch.distributed as dist

from . import ssd


@dataclass
class SegmentOps:
    """The three computations a rank performs; the defaults are the library's
    (tests on machines without a GPU substitute the fp64 oracle)."""
    forward: Callable = None        # (x, a, Bm, Cm, D, chunk, initial_state) -> (y, final)
    decay_total: Callable = None    # a -> total log-decay per chain
    state_combine: Callable = None  # (finals [W,...], totals [W,...], h0) -> h_in [W+1,...]

    def __post_init__(self):
        if self.forward is None:
            self.forward = lambda x, a, Bm, Cm, D, chunk, init: ssd.forward(
                x, a, Bm, Cm, D, chunk, initial_state=init)
        if self.decay_total is None:
            self.decay_total = ssd.decay_total
        if self.state_combine is None:
            self.state_combine = ssd.state_combine


def _all_gather(t: torch.Tensor, group) -> torch.Tensor:
    """[W, *t.shape] on every rank (one collective)."""
    world = dist.get_world_size(group)
    out = torch.empty((world,) + tuple(t.shape), dtype=t.dtype, device=t.device)
    if t.is_cuda:
        dist.all_gather_into_tensor(out, t.contiguous(), group=group)
    else:
        dist.all_gather(list(out.unbind(0)), t.contiguous(), group=group)
    return out


def sequence_sharded_forward(x, a, Bm, Cm, D, chunk, *, group=None, initial_state=None,
                             ops: SegmentOps | None = None):
    """This rank's segment of y, and the final state of the whole sequence.

    x [B,T_r,H,P], a [B,T_r,H] (or [B,T_r,H,N]), Bm/Cm [B,T_r,G,N] hold this
    rank's tokens; initial_state [B,H,N,P] (optional, the same on every rank)
    enters the first segment.  Every rank takes part in the same single
    all-gather (of the final states and of the total decays, packed)."""
    ops = ops or SegmentOps()
    rank = dist.get_rank(group)
    y, fin = ops.forward(x, a, Bm, Cm, D, chunk, None)
    tot = ops.decay_total(a)
    # one collective: final state and total decay of every segment, packed
    packed = torch.cat([fin.reshape(-1), tot.reshape(-1).to(fin.dtype)])
    gathered = _all_gather(packed, group)
    nf = fin.numel()
    finals = gathered[:, :nf].reshape((gathered.shape[0],) + tuple(fin.shape)).contiguous()
    totals = gathered[:, nf:].reshape((gathered.shape[0],) + tuple(tot.shape)).contiguous()
    h_in = ops.state_combine(finals, totals, initial_state)
    if rank > 0 or initial_state is not None:
        y, _ = ops.forward(x, a, Bm, Cm, D, chunk, h_in[rank].contiguous())
    return y, h_in[-1]
