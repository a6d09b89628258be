"""PyTorch autograd for the chunked SSD forward: y, final = ssd_autograd(...)
takes part in a torch graph, and its backward is the library's ssd_backward
(the gradients of sum(dy * y) + <dfinal, final> that autograd asks for).

The forward keeps only its inputs for the backward, which rebuilds the chunk
states from them instead of storing them during the forward (the memory
trade named on llms.blog "State Space Models and Mamba ...", section
"Hardware-Aware Parallel Associative Scan").  All arithmetic runs in the
library's kernels; this module only passes tensors.
"""
from __future__ import annotations

import torch

from . import ssd


class _Ops:
    """The two computations the function calls (tests without a GPU pass the
    fp64 oracle instead)."""

    @staticmethod
    def forward(x, a, Bm, Cm, D, chunk, init):
        return ssd.forward(x, a, Bm, Cm, D, chunk, initial_state=init)

    @staticmethod
    def backward(x, a, Bm, Cm, D, dy, chunk, dfinal, init):
        return ssd.backward(x, a, Bm, Cm, D, dy, chunk, dfinal=dfinal, initial_state=init)


class SSDFunction(torch.autograd.Function):
    @staticmethod
    def forward(ctx, x, a, Bm, Cm, D, initial_state, chunk, ops):
        y, final = ops.forward(x, a, Bm, Cm, D, chunk, initial_state)
        ctx.save_for_backward(x, a, Bm, Cm, D, initial_state)
        ctx.chunk, ctx.ops = chunk, ops
        return y, final

    @staticmethod
    def backward(ctx, dy, dfinal):
        x, a, Bm, Cm, D, init = ctx.saved_tensors
        if dy is None:
            dy = torch.zeros_like(x)
        g = ctx.ops.backward(x, a, Bm, Cm, D, dy.contiguous().to(x.dtype), ctx.chunk,
                             None if dfinal is None else dfinal.contiguous().to(torch.float32), init)
        return (g["dx"], g["da"], g["dBm"], g["dCm"],
                g["dD"] if D is not None and ctx.needs_input_grad[4] else None,
                g["dinit"] if init is not None and ctx.needs_input_grad[5] else None,
                None, None)


def ssd_autograd(x, a, Bm, Cm, D=None, chunk=256, initial_state=None, *, ops=None):
    """(y, final_state) of the forward as a differentiable torch operation.
    Shapes and dtypes as for ssd.forward; gradients flow to x, a, Bm, Cm, D
    and initial_state (whichever require them)."""
    return SSDFunction.apply(x, a, Bm, Cm, D, initial_state, chunk, ops or _Ops)
