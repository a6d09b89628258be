"""Pins of the oracle's backward (oracle.ssd_oracle.backward), on the CPU.

The backward is the gradient of l = sum_t dy_t . y_t + <dfinal, h_{T-1}>.
It is pinned against the forward oracle (the C recurrence, itself pinned in
test_oracle_pins.py) by central finite differences on every input element,
by the Euler identities of the parts of l that are linear in one input, and
by the memoryless closed form -- none of which retypes the adjoint.
"""
from __future__ import annotations

import numpy as np
import pytest

from oracle import ssd_oracle as O
from tests.oracle_cases import random_problem, rel_inf


def _loss(prob, dy, dfinal, init):
    """l through the forward oracle: y [B,H,T,P] and final [B,H,N,P]."""
    B, T, H, P = prob.x.shape
    N = prob.Bm.shape[3]
    r = O.recurrence(prob, initial=init, nthreads=1)
    y = O.to_bthp(r["y"], r["chains"], B, H)
    fin = r["final"].reshape(B, H, N, P)
    return float(np.sum(dy * y) + (0.0 if dfinal is None else np.sum(dfinal * fin)))


def _setup(per_state, seed, B=1, T=5, H=2, P=2, G=1, N=3, with_init=True, with_dfinal=True):
    rng = np.random.default_rng(seed)
    prob = random_problem(rng, B=B, T=T, H=H, P=P, G=G, N=N, per_state=per_state)
    dy = rng.standard_normal(prob.x.shape)
    init = rng.standard_normal((B, H, N, P)) if with_init else None
    dfinal = rng.standard_normal((B, H, N, P)) if with_dfinal else None
    return prob, dy, init, dfinal


@pytest.mark.parametrize("per_state", [False, True])
@pytest.mark.parametrize("G,H", [(1, 2), (2, 4)])
def test_backward_matches_finite_differences(per_state, G, H):
    """Every element of every gradient equals the central difference of l
    (step 1e-6; fp64 truncation and rounding stay far below 1e-6)."""
    prob, dy, init, dfinal = _setup(per_state, 3 + G + 2 * per_state, H=H, G=G)
    g = O.backward(prob, dy, dfinal=dfinal, initial=init)
    eps = 1e-6
    fields = {"x": "dx", "a": "da", "Bm": "dBm", "Cm": "dCm", "D": "dD", "init": "dinit"}
    for name, gname in fields.items():
        base = init if name == "init" else getattr(prob, name)
        fd = np.zeros_like(base)
        for idx in np.ndindex(base.shape):
            vals = []
            for s in (+eps, -eps):
                arr = base.copy()
                arr[idx] += s
                if name == "init":
                    vals.append(_loss(prob, dy, dfinal, arr))
                else:
                    kw = dict(x=prob.x, a=prob.a, Bm=prob.Bm, Cm=prob.Cm, D=prob.D)
                    kw[name] = arr
                    vals.append(_loss(O.Problem(**kw), dy, dfinal, init))
            fd[idx] = (vals[0] - vals[1]) / (2 * eps)
        err = np.max(np.abs(fd - g[gname])) / max(1.0, np.max(np.abs(fd)))
        assert err < 1e-6, (name, err)


@pytest.mark.parametrize("per_state", [False, True])
def test_backward_euler_identities(per_state):
    """l minus its D term is linear in C, jointly linear in (x, initial state),
    and (from a zero initial state) linear in B, so by Euler's theorem it
    equals <dC, C>, <dx - D dy, x> + <d initial, initial> and <dB, B>."""
    prob, dy, init, dfinal = _setup(per_state, 17, B=2, T=9, H=4, P=3, G=2, N=4)
    B, T, H, P = prob.x.shape
    Dv = prob.D
    skip = float(np.sum(dy * Dv[None, None, :, None] * prob.x))
    l_init = _loss(prob, dy, dfinal, init) - skip
    g = O.backward(prob, dy, dfinal=dfinal, initial=init)
    dx_state = g["dx"] - Dv[None, None, :, None] * dy
    # the final state does not depend on C: only the output part is linear in C
    l_out = _loss(prob, dy, None, init) - skip
    assert abs(np.sum(g["dCm"] * prob.Cm) - l_out) < 1e-10 * max(1.0, abs(l_out))
    assert abs(np.sum(dx_state * prob.x) + np.sum(g["dinit"] * init) - l_init) < 1e-10 * max(1.0, abs(l_init))
    l_zero = _loss(prob, dy, dfinal, None) - skip
    g0 = O.backward(prob, dy, dfinal=dfinal)
    assert abs(np.sum(g0["dBm"] * prob.Bm) - l_zero) < 1e-10 * max(1.0, abs(l_zero))
    assert abs(np.sum(g["dD"] * Dv) - skip) < 1e-10 * max(1.0, abs(skip))


def test_backward_memoryless_limit():
    """e^{a} = 0 (a = -1e4 underflows to exactly 0): y_t = (C_t . B_t) x_t + D x_t,
    so dx_t = (C_t . B_t + D) dy_t, dB_t = C_t (dy_t . x_t), dC_t = B_t (dy_t . x_t)
    summed over the group's heads, da = 0 and the initial state gets nothing."""
    prob, dy, init, _ = _setup(False, 23, B=2, T=6, H=4, P=3, G=2, N=5, with_dfinal=False)
    prob = O.Problem(prob.x, np.full_like(prob.a, -1e4), prob.Bm, prob.Cm, prob.D)
    g = O.backward(prob, dy, initial=init)
    B, T, H, P = prob.x.shape
    G = prob.Bm.shape[2]
    grp = np.arange(H) // (H // G)
    cb = np.einsum("btgn,btgn->btg", prob.Cm, prob.Bm)[:, :, grp]          # [B,T,H]
    dot = np.einsum("bthp,bthp->bth", dy, prob.x)                           # [B,T,H]
    assert rel_inf(g["dx"], (cb + prob.D[None, None, :])[..., None] * dy) < 1e-12
    dBm = np.zeros_like(prob.Bm)
    dCm = np.zeros_like(prob.Cm)
    for h in range(H):
        dBm[:, :, grp[h]] += prob.Cm[:, :, grp[h]] * dot[:, :, h, None]
        dCm[:, :, grp[h]] += prob.Bm[:, :, grp[h]] * dot[:, :, h, None]
    assert rel_inf(g["dBm"], dBm) < 1e-12
    assert rel_inf(g["dCm"], dCm) < 1e-12
    assert np.all(g["da"] == 0) and np.all(g["dinit"] == 0)
