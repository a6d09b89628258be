"""GPU parity of the backward (ssd_backward, through the C ABI) against the
oracle's adjoint of the recurrence, on the same seeded inputs.

Every gradient (dx, da, dBm, dCm, dD, d initial) is compared with the parity
metric ||g - g_ref||_inf / ||g_ref||_inf: 1e-4 for fp32 inputs, 2e-2 for bf16
inputs (fp32 arithmetic; dx, dB, dC rounded to bf16 on output).  Cases span
several chunks and row tiles, a partial last chunk, grouped B/C, a loss on
the final state and a given initial state.
"""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from oracle import ssd_oracle as O
from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.workloads import generate, small_case
from tests.gpu_helpers import TOL_BF16, rel_err, to_dev, tol_for

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load()


CASES = [
    small_case(B=2, T=96, H=3, P=24, N=20, G=1, chunk=32, dtype="f32", seed=81),
    small_case(B=1, T=150, H=4, P=70, N=33, G=2, chunk=64, dtype="f32", seed=82),
    small_case(B=1, T=512, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=83),
    small_case(B=2, T=300, H=4, P=64, N=128, G=2, chunk=128, dtype="bf16", seed=84),
    # tensor-core forms: 256-token chunks, grouped B/C, a last chunk of 8 rows
    small_case(B=2, T=520, H=4, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=87),
    # the group-summing forms over longer head loops (8 and 4 heads per group)
    small_case(B=1, T=1000, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=88),
    small_case(B=2, T=384, H=12, P=64, N=128, G=3, chunk=128, dtype="bf16", seed=89),
    small_case(B=1, T=7, H=2, P=5, N=3, G=1, chunk=7, dtype="f32", seed=85),
    small_case(B=1, T=5, H=1, P=3, N=2, G=1, chunk=1, dtype="f32", seed=86),
]


# per-state decay (a [B,T,H,N]); served up to N = 128
DIAG_CASES = [
    small_case(B=1, T=150, H=2, P=20, N=12, G=1, chunk=64, dtype="f32", a_per_state=True, seed=93),
    small_case(B=2, T=256, H=2, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=94),
    small_case(B=2, T=200, H=4, P=16, N=24, G=2, chunk=128, dtype="f32", a_per_state=True, seed=95),
    small_case(B=1, T=130, H=2, P=64, N=128, G=1, chunk=64, dtype="bf16", a_per_state=True, seed=96),
    small_case(B=1, T=70, H=2, P=256, N=32, G=1, chunk=64, dtype="f32", a_per_state=True, seed=97),
    small_case(B=1, T=5, H=1, P=3, N=2, G=1, chunk=1, dtype="f32", a_per_state=True, seed=98),
]


def _ids(cases):
    return [c.name + ("_diag" if c.a_per_state else "") + "_" + c.dtype for c in cases]


def _extras(w, with_init, with_dfinal):
    g = torch.Generator().manual_seed(w.seed + 101)
    dt = torch.float32 if w.dtype == "f32" else torch.bfloat16
    dy = torch.randn((w.B, w.T, w.H, w.P), generator=g).to(dt)
    init = torch.randn((w.B, w.H, w.N, w.P), generator=g) if with_init else None
    dfin = torch.randn((w.B, w.H, w.N, w.P), generator=g) if with_dfinal else None
    return dy, init, dfin


def _run(w, with_init, with_dfinal):
    inp = generate(w)
    dy, init, dfin = _extras(w, with_init, with_dfinal)
    dev = to_dev(inp)
    got = ssd.backward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], dy.cuda(), w.chunk,
                       dfinal=None if dfin is None else dfin.cuda(),
                       initial_state=None if init is None else init.cuda())
    torch.cuda.synchronize()
    f = lambda t: None if t is None else t.to(torch.float64).numpy()
    prob = O.Problem(*(f(inp[k]) for k in ("x", "a", "Bm", "Cm", "D")))
    ref = O.backward(prob, f(dy), dfinal=f(dfin), initial=f(init))
    return got, ref


@pytest.mark.parametrize("w", CASES + DIAG_CASES, ids=_ids(CASES + DIAG_CASES))
@pytest.mark.parametrize("with_init,with_dfinal", [(False, False), (True, True)],
                         ids=["plain", "init_dfinal"])
def test_backward_matches_oracle(w, with_init, with_dfinal):
    got, ref = _run(w, with_init, with_dfinal)
    tol = tol_for(w)
    errs = {}
    for k in ("dx", "da", "dBm", "dCm", "dD", "dinit"):
        g = got[k].float().cpu().numpy().astype(np.float64)
        errs[k] = rel_err(g, ref[k])
    assert all(e <= tol for e in errs.values()), errs


@pytest.mark.parametrize("dtype", ["f32", "bf16"])
def test_backward_maximum_sizes(dtype):
    """N = P = 256 (the largest the boundary takes: the widest shared tiles)
    with a partial last chunk."""
    w = small_case(B=1, T=200, H=2, P=256, N=256, G=1, chunk=128, dtype=dtype, seed=91)
    got, ref = _run(w, True, True)
    errs = {k: rel_err(got[k].float().cpu().numpy().astype(np.float64), ref[k])
            for k in ("dx", "da", "dBm", "dCm", "dD", "dinit")}
    assert all(e <= tol_for(w) for e in errs.values()), errs


def test_backward_without_D_and_deterministic():
    """D = NULL is D = 0 (dx carries no skip term; dD is still sum dy.x), two
    calls on the same inputs give bit-identical gradients, and the call leaves
    SSD_OK in its workspace's status word."""
    w = small_case(B=2, T=256, H=4, P=64, N=128, G=2, chunk=128, dtype="bf16", seed=92)
    inp = generate(w)
    dev = to_dev(inp)
    dy, _, dfin = _extras(w, False, True)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    ws = torch.full((ssd.backward_workspace_size(shape),), 7, dtype=torch.uint8, device="cuda")
    run = lambda: ssd.backward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], None, dy.cuda(), w.chunk,
                               dfinal=dfin.cuda(), workspace=ws)
    g1 = run()
    assert ssd.device_status(ws) == ssd.SSD_OK
    g2 = run()
    torch.cuda.synchronize()
    for k in ("dx", "da", "dBm", "dCm", "dD", "dinit"):
        assert torch.equal(g1[k], g2[k]), k
    f = lambda t: t.to(torch.float64).numpy()
    prob = O.Problem(f(inp["x"]), f(inp["a"]), f(inp["Bm"]), f(inp["Cm"]), None)
    ref = O.backward(prob, f(dy), dfinal=f(dfin))
    errs = {k: rel_err(g1[k].float().cpu().numpy().astype(np.float64), ref[k])
            for k in ("dx", "da", "dBm", "dCm", "dD", "dinit")}
    assert all(e <= tol_for(w) for e in errs.values()), errs


def test_backward_rejects_per_state_and_bad_workspace():
    """The per-state variant above N = 128 is not served (SSD_ERR_UNSUPPORTED)
    and a short workspace is refused before any launch."""
    w = small_case(B=1, T=64, H=2, P=16, N=256, G=1, chunk=32, dtype="f32", a_per_state=True, seed=87)
    dev = to_dev(generate(w))
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    assert ssd.backward_workspace_size(shape) == 0
    with pytest.raises(ssd.SSDError) as e:
        ssd.backward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], dev["x"].clone(), w.chunk)
    assert e.value.code == ssd.SSD_ERR_UNSUPPORTED
    w2 = small_case(B=1, T=64, H=2, P=16, N=16, G=1, chunk=32, dtype="f32", seed=88)
    dev = to_dev(generate(w2))
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w2.chunk)
    need = ssd.backward_workspace_size(shape)
    ws = torch.empty(need - 256, dtype=torch.uint8, device="cuda")
    outs = [torch.empty_like(dev[k]) for k in ("x", "a", "Bm", "Cm")]
    code = ssd.load().ssd_backward(
        ctypes.byref(shape), dev["x"].data_ptr(), dev["a"].data_ptr(), dev["Bm"].data_ptr(),
        dev["Cm"].data_ptr(), None, None, dev["x"].data_ptr(), None, outs[0].data_ptr(),
        outs[1].data_ptr(), outs[2].data_ptr(), outs[3].data_ptr(), None, None, ws.data_ptr(),
        ws.numel(), None)
    assert code == ssd.SSD_ERR_WORKSPACE


@pytest.mark.parametrize("per_state", [False, True], ids=["scalar", "per_state"])
def test_backward_over_segments_with_library_kernels(per_state):
    """The sharded backward's steps on one GPU, the sequence cut into 4
    segments: entering states by ssd_state_combine, each segment's backward
    with no end loss, the entering-state adjoints combined in reverse order
    from dfinal, and each segment's backward rerun with the adjoint at its
    end -- equal to the fp64 adjoint of the whole sequence (the oracle)."""
    if per_state:
        w = small_case(B=2, T=1024, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=105)
    else:
        w = small_case(B=2, T=2048, H=4, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=106)
    inp = generate(w)
    dev = to_dev(inp)
    dy, _, dfin = _extras(w, False, True)
    dy, dfin = dy.cuda(), dfin.cuda()
    S = 4
    Ts = w.T // S
    seg = lambda t, s: t[:, s * Ts:(s + 1) * Ts].clone()  # aligned copies, as each rank holds
    parts = [[seg(t, s) for t in (dev["x"], dev["a"], dev["Bm"], dev["Cm"], dy)] for s in range(S)]
    st = [ssd.segment_state(x, a, Bm, w.chunk) for x, a, Bm, Cm, _ in parts]
    fins = [f for f, _ in st]
    tots = torch.stack([t for _, t in st]).contiguous()
    h_in = ssd.state_combine(torch.stack(fins).contiguous(), tots)
    g1 = [ssd.backward(x, a, Bm, Cm, dev["D"], g, w.chunk, initial_state=h_in[s].contiguous())
          for s, (x, a, Bm, Cm, g) in enumerate(parts)]
    dinits = torch.stack([g["dinit"] for g in g1])
    adj = ssd.state_combine(dinits.flip(0).contiguous(), tots.flip(0).contiguous(), dfin)
    g2 = [ssd.backward(x, a, Bm, Cm, dev["D"], g, w.chunk, dfinal=adj[S - 1 - s].contiguous(),
                       initial_state=h_in[s].contiguous())
          for s, (x, a, Bm, Cm, g) in enumerate(parts)]
    torch.cuda.synchronize()
    f = lambda t: t.float().cpu().numpy().astype(np.float64)
    f64 = lambda t: t.to(torch.float64).cpu().numpy()
    full = O.backward(O.Problem(*(f64(inp[k]) for k in ("x", "a", "Bm", "Cm", "D"))), f64(dy),
                      dfinal=f64(dfin))
    errs = {k: rel_err(f(torch.cat([g[k] for g in g2], dim=1)), full[k])
            for k in ("dx", "da", "dBm", "dCm")}
    errs["dD"] = rel_err(f(sum(g["dD"] for g in g1)), full["dD"])
    errs["dinit"] = rel_err(f(adj[S]), full["dinit"])
    assert all(e <= TOL_BF16 for e in errs.values()), errs
