"""The autograd wrapper's plumbing on the CPU: the fp64 oracle stands in for
the library's forward and backward, and torch.autograd.gradcheck compares the
function's gradients (the oracle's adjoint, routed through the wrapper) with
finite differences of its forward -- argument order, the optional D and
initial state, and losses on y alone or on the final state alone."""
import numpy as np
import pytest
import torch

from oracle import ssd_oracle as O
from ssd_chunked_forward_b200.autograd import ssd_autograd


class OracleOps:
    @staticmethod
    def forward(x, a, Bm, Cm, D, chunk, init):
        f = lambda t: None if t is None else t.detach().numpy()
        prob = O.Problem(f(x), f(a), f(Bm), f(Cm), f(D))
        B, T, H, P = x.shape
        N = Bm.shape[3]
        r = O.recurrence(prob, initial=f(init), nthreads=1)
        y = r["y"].reshape(B, H, T, P).transpose(0, 2, 1, 3)
        return torch.from_numpy(np.ascontiguousarray(y)), torch.from_numpy(r["final"].reshape(B, H, N, P))

    @staticmethod
    def backward(x, a, Bm, Cm, D, dy, chunk, dfinal, init):
        f = lambda t: None if t is None else t.detach().numpy()
        prob = O.Problem(f(x), f(a), f(Bm), f(Cm), f(D))
        g = O.backward(prob, f(dy), dfinal=f(dfinal), initial=f(init))
        return {k: torch.from_numpy(np.ascontiguousarray(g[k])) for k in ("dx", "da", "dBm", "dCm", "dD", "dinit")}


def _inputs(per_state, with_D=True, with_init=True, seed=0):
    g = torch.Generator().manual_seed(seed)
    B, T, H, P, G, N = 1, 6, 2, 2, 1, 3
    x = torch.randn((B, T, H, P), generator=g, dtype=torch.float64)
    a = -torch.rand((B, T, H, N) if per_state else (B, T, H), generator=g, dtype=torch.float64) * 0.5
    Bm = torch.randn((B, T, G, N), generator=g, dtype=torch.float64) / 2
    Cm = torch.randn((B, T, G, N), generator=g, dtype=torch.float64) / 2
    D = torch.randn((H,), generator=g, dtype=torch.float64) if with_D else None
    h0 = torch.randn((B, H, N, P), generator=g, dtype=torch.float64) if with_init else None
    return [t.requires_grad_() if t is not None else None for t in (x, a, Bm, Cm, D, h0)]


@pytest.mark.parametrize("per_state", [False, True])
@pytest.mark.parametrize("with_D,with_init", [(True, True), (False, False)])
def test_gradcheck_through_the_wrapper(per_state, with_D, with_init):
    x, a, Bm, Cm, D, h0 = _inputs(per_state, with_D, with_init)
    args = [t for t in (x, a, Bm, Cm, D, h0) if t is not None]

    def fn(*ts):
        it = iter(ts)
        xx, aa, bb, cc = next(it), next(it), next(it), next(it)
        dd = next(it) if with_D else None
        hh = next(it) if with_init else None
        return ssd_autograd(xx, aa, bb, cc, dd, 4, hh, ops=OracleOps)

    assert torch.autograd.gradcheck(fn, tuple(args), eps=1e-6, atol=1e-7, rtol=1e-5)


def test_loss_on_one_output_only():
    """A loss on y alone (the final state's gradient is zero) and on the final
    state alone (y's gradient is zero) both match the oracle's backward."""
    x, a, Bm, Cm, D, h0 = _inputs(False, seed=3)
    y, fin = ssd_autograd(x, a, Bm, Cm, D, 4, h0, ops=OracleOps)
    y.sum().backward()
    ref = OracleOps.backward(x, a, Bm, Cm, D, torch.ones_like(x), 4, None, h0)
    assert torch.allclose(x.grad, ref["dx"]) and torch.allclose(a.grad, ref["da"])
    assert torch.allclose(h0.grad, ref["dinit"]) and torch.allclose(D.grad, ref["dD"])
    for t in (x, a, Bm, Cm, D, h0):
        t.grad = None
    y, fin = ssd_autograd(x, a, Bm, Cm, D, 4, h0, ops=OracleOps)
    (fin * 2).sum().backward()
    ref = OracleOps.backward(x, a, Bm, Cm, D, torch.zeros_like(x), 4, torch.full_like(h0, 2.0), h0)
    assert torch.allclose(Bm.grad, ref["dBm"]) and torch.allclose(Cm.grad, ref["dCm"])
    assert torch.allclose(D.grad, ref["dD"])
