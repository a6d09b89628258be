"""GPU parity of libssd against the fp64 oracle, through the C ABI.

Per-step parity (each kernel fed the oracle's own fp64 intermediates, cast to
fp32), end-to-end parity on small cases that span several tiles with ragged
edges, the library's invariants, and edge shapes.  Full-size workloads are in
test_gpu_workloads.py.  Tolerances: 1e-4 for fp32 inputs, 2e-2 for bf16
inputs with fp32 accumulation, as ||y - y_ref||_inf / ||y_ref||_inf.
"""
from __future__ import annotations

import math

import numpy as np
import pytest
import torch

from oracle import ssd_oracle as O
from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.workloads import generate, small_case
from tests.gpu_helpers import (TOL_BF16, TOL_F32, chain_problem, parity_on_chains, rel_err,
                               run_forward, to_dev, tol_for)

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load()  # a missing library is an error, not a skip


CASES = [
    small_case(B=2, T=96, H=3, P=24, N=20, G=1, chunk=32, dtype="f32", seed=1),
    small_case(B=1, T=150, H=2, P=70, N=33, G=2, chunk=30, dtype="f32", seed=2),
    small_case(B=1, T=192, H=4, P=64, N=128, G=2, chunk=64, dtype="bf16", seed=3),
    small_case(B=2, T=768, H=3, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=4),
    small_case(B=1, T=384, H=5, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=5),
    small_case(B=2, T=1024, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=13, u_mean=-4.0),
    small_case(B=1, T=2048, H=16, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=14),
    small_case(B=2, T=256, H=2, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=6),
    small_case(B=1, T=60, H=2, P=10, N=12, G=1, chunk=20, dtype="f32", a_per_state=True, seed=7),
    # per-state tensor-core steps: an odd number of 128-token blocks; groups, a
    # partial last block and fast decay (a sub-block's decay far beyond fp32's range)
    small_case(B=1, T=384, H=3, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=31),
    small_case(B=2, T=1000, H=4, P=64, N=64, G=2, chunk=128, dtype="bf16", a_per_state=True, seed=32,
               u_mean=-1.0),
]
EDGE = [
    small_case(B=1, T=1, H=1, P=1, N=1, G=1, chunk=1, dtype="f32", seed=8),
    small_case(B=1, T=5, H=1, P=3, N=2, G=1, chunk=1, dtype="f32", seed=9),
    small_case(B=1, T=7, H=2, P=5, N=3, G=2, chunk=7, dtype="f32", seed=10),
    small_case(B=3, T=64, H=1, P=1, N=1, G=1, chunk=64, dtype="bf16", seed=11),
    small_case(B=1, T=1024, H=1, P=8, N=8, G=1, chunk=1024, dtype="f32", seed=12),
]

# T % chunk != 0: the last chunk (and, on the tensor-core paths, the last
# 128-token block) holds the remaining tokens; the kernels read zeros past T
# and write nothing there
RAGGED = [
    small_case(B=1, T=384, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=71),
    small_case(B=1, T=1000, H=2, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=73),
    small_case(B=2, T=77, H=3, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=72),
    small_case(B=2, T=4000, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=76),
    small_case(B=1, T=997, H=2, P=12, N=10, G=1, chunk=256, dtype="f32", seed=74),
    small_case(B=2, T=200, H=2, P=16, N=24, G=2, chunk=128, dtype="f32", a_per_state=True, seed=75),
]
# per-step cases with a partial last chunk (tensor-core steps take chunk 128)
STEP_RAGGED = [
    small_case(B=2, T=333, H=3, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=77),
    small_case(B=1, T=150, H=2, P=20, N=12, G=1, chunk=64, dtype="f32", a_per_state=True, seed=78),
]


def _ids(cases):
    return [c.name + ("_diag" if c.a_per_state else "") + "_" + c.dtype for c in cases]


def _all_chains(w):
    return [(b, h) for b in range(w.B) for h in range(w.H)]


def _paths():
    return [ssd.PATH_SIMT, ssd.PATH_MODULAR, ssd.PATH_AUTO, ssd.PATH_FUSED]


@pytest.mark.parametrize("w", CASES + EDGE + RAGGED, ids=_ids(CASES + EDGE + RAGGED))
@pytest.mark.parametrize("path", _paths(), ids=["simt", "modular", "auto", "fused"])
def test_forward_matches_oracle(w, path):
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    if not ssd.path_supported(shape, path):
        pytest.skip("path does not serve this shape")
    y, fin = run_forward(w, dev, path=path)
    ey, ef = parity_on_chains(inp, y, fin, _all_chains(w))
    tol = tol_for(w)
    assert ey <= tol, f"y rel err {ey:.3e}"
    assert ef <= tol, f"final-state rel err {ef:.3e}"


def _oracle_chunked(inp, w):
    """O3 per chain, as [B,H,...] float64 arrays.  A partial last chunk is
    the input padded with a = 0 and x = B = C = 0 (the padding is pinned on
    the CPU to leave y[:T] and the final state unchanged)."""
    arrs = [inp[k].to(torch.float64).numpy() for k in ("x", "a", "Bm", "Cm")]
    nc = -(-w.T // w.chunk)
    Tp = nc * w.chunk
    if Tp != w.T:
        arrs = [np.pad(v, [(0, 0), (0, Tp - w.T)] + [(0, 0)] * (v.ndim - 2)) for v in arrs]
    prob = O.Problem(*arrs, inp["D"].to(torch.float64).numpy())
    r = O.chunked(prob, w.chunk)
    cum = r["cum"].reshape(w.B, w.H, nc, w.chunk, -1)
    if not w.a_per_state:
        cum = cum[..., 0]
    S = r["S"].reshape(w.B, w.H, nc, w.N, w.P)
    Hin = r["Hin"].reshape(w.B, w.H, nc, w.N, w.P)
    y = r["y"].reshape(w.B, w.H, Tp, w.P).transpose(0, 2, 1, 3)[:, : w.T]
    fin = r["final"].reshape(w.B, w.H, w.N, w.P)
    return cum, S, Hin, y, fin


@pytest.mark.parametrize("w", CASES + STEP_RAGGED, ids=_ids(CASES + STEP_RAGGED))
def test_step_chunk_cumsum(w):
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    cum = ssd.chunk_cumsum(shape, dev["a"])
    torch.cuda.synchronize()
    ref = _oracle_chunked(inp, w)[0]
    assert rel_err(cum.cpu().numpy().astype(np.float64), ref) < 1e-5


@pytest.mark.parametrize("w", CASES + STEP_RAGGED, ids=_ids(CASES + STEP_RAGGED))
@pytest.mark.parametrize("impl", [ssd.IMPL_SIMT, ssd.IMPL_TC], ids=["simt", "tc"])
def test_step_chunk_state(w, impl):
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    cum, S, _, _, _ = _oracle_chunked(inp, w)
    cum_d = torch.from_numpy(cum.astype(np.float32)).cuda().contiguous()
    try:
        got = ssd.chunk_state(shape, dev["x"], dev["Bm"], cum_d, impl=impl)
    except ssd.SSDError as e:
        if e.code == ssd.SSD_ERR_UNSUPPORTED:
            pytest.skip("tensor-core chunk_state does not serve this shape")
        raise
    torch.cuda.synchronize()
    assert rel_err(got.cpu().numpy().astype(np.float64), S) <= tol_for(w)


@pytest.mark.parametrize("w", CASES + STEP_RAGGED, ids=_ids(CASES + STEP_RAGGED))
def test_step_state_pass(w):
    inp = generate(w)
    shape = ssd.make_shape(w.B, w.T, w.H, w.P, w.G, w.N, w.chunk, w.a_per_state, w.dtype)
    cum, S, Hin, _, fin = _oracle_chunked(inp, w)
    cum_d = torch.from_numpy(cum.astype(np.float32)).cuda().contiguous()
    st = torch.from_numpy(S.astype(np.float32)).cuda().contiguous()
    fin_d = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device="cuda")
    ssd.state_pass(shape, cum_d, st, fin_d)
    torch.cuda.synchronize()
    assert rel_err(st.cpu().numpy().astype(np.float64), Hin) < 1e-5
    assert rel_err(fin_d.cpu().numpy().astype(np.float64), fin) < 1e-5


@pytest.mark.parametrize("w", CASES + STEP_RAGGED, ids=_ids(CASES + STEP_RAGGED))
@pytest.mark.parametrize("impl", [ssd.IMPL_SIMT, ssd.IMPL_TC], ids=["simt", "tc"])
def test_step_chunk_scan(w, impl):
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    cum, _, Hin, y_ref, _ = _oracle_chunked(inp, w)
    cum_d = torch.from_numpy(cum.astype(np.float32)).cuda().contiguous()
    Hin_d = torch.from_numpy(Hin.astype(np.float32)).cuda().contiguous()
    try:
        y = ssd.chunk_scan(shape, dev["x"], dev["Bm"], dev["Cm"], cum_d, Hin_d, dev["D"], impl=impl)
    except ssd.SSDError as e:
        if e.code == ssd.SSD_ERR_UNSUPPORTED:
            pytest.skip("tensor-core scan does not serve this shape")
        raise
    torch.cuda.synchronize()
    assert rel_err(y.float().cpu().numpy().astype(np.float64), y_ref) <= tol_for(w)


# ------------------------------------------------------------ invariants ----

def _bf16_case(T=1024, H=4, G=1, seed=21, u_mean=-2.0):
    return small_case(B=2, T=T, H=H, P=64, N=128, G=G, chunk=256, dtype="bf16", seed=seed,
                      u_mean=u_mean)


def test_chunk_size_invariance():
    """The result does not depend on the chunk size ("State Space Duality":
    the chunk boundary separates the two forms and nothing else)."""
    w = _bf16_case()
    dev = to_dev(generate(w))
    outs = [ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], q)
            for q in (32, 64, 128, 256)]
    torch.cuda.synchronize()
    ref = outs[0][0].float().cpu().numpy()
    for y, fin in outs[1:]:
        assert rel_err(y.float().cpu().numpy(), ref) <= TOL_BF16
        # the tensor-core paths round the decay-weighted x to bf16 for the state
        assert rel_err(fin.cpu().numpy(), outs[0][1].cpu().numpy()) <= TOL_BF16


def test_diag_broadcast_equals_scalar():
    """Per-state decays equal across n give the scalar result."""
    w = small_case(B=1, T=512, H=2, P=64, N=64, G=1, chunk=128, dtype="bf16", seed=22)
    dev = to_dev(generate(w))
    y1, f1 = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    a4 = dev["a"].unsqueeze(-1).expand(*dev["a"].shape, w.N).contiguous()
    y2, f2 = ssd.forward(dev["x"], a4, dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    torch.cuda.synchronize()
    # the per-state path rounds its tensor-core operands (B o w) to bf16, the
    # scalar path for N = 64 runs on CUDA cores in fp32: both within the bf16 bar
    assert rel_err(y2.float().cpu().numpy(), y1.float().cpu().numpy()) <= TOL_BF16
    assert rel_err(f2.cpu().numpy(), f1.cpu().numpy()) <= TOL_BF16


def test_grouping_equals_replication():
    w = _bf16_case(H=8, G=2, seed=23)
    dev = to_dev(generate(w))
    y1, f1 = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    rep = lambda m: m.repeat_interleave(w.H // w.G, dim=2).contiguous()
    y2, f2 = ssd.forward(dev["x"], dev["a"], rep(dev["Bm"]), rep(dev["Cm"]), dev["D"], w.chunk)
    torch.cuda.synchronize()
    assert rel_err(y2.float().cpu().numpy(), y1.float().cpu().numpy()) <= 1e-6
    assert rel_err(f2.cpu().numpy(), f1.cpu().numpy()) <= 1e-6


@pytest.mark.parametrize("dtype,tol", [("f32", 1e-5), ("bf16", 4e-3)])
def test_first_decay_and_causality(dtype, tol):
    """a_0 multiplies nothing (the product in M_{i,j} runs over k = j+1..i):
    changing it moves y only by rounding (cum values shift, so the fp32
    differences round differently; bf16 outputs may flip one ulp).  Outputs
    before a perturbed input are bitwise unchanged (causal masking)."""
    w = small_case(B=2, T=1024, H=4, P=64, N=128, G=1, chunk=256, dtype=dtype, seed=24)
    dev = to_dev(generate(w))
    y0, _ = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    a2 = dev["a"].clone()
    a2[:, 0] = -9.0
    y1, _ = ssd.forward(dev["x"], a2, dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    x2 = dev["x"].clone()
    s = 700
    x2[:, s] += 3.0
    y2, _ = ssd.forward(x2, dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    torch.cuda.synchronize()
    assert rel_err(y1.float().cpu().numpy(), y0.float().cpu().numpy()) <= tol
    assert torch.equal(y2[:, :s], y0[:, :s])
    assert not torch.equal(y2[:, s:], y0[:, s:])


@pytest.mark.parametrize("path", [ssd.PATH_SIMT, ssd.PATH_AUTO], ids=["simt", "auto"])
def test_deterministic(path):
    w = _bf16_case(seed=25)
    dev = to_dev(generate(w))
    r1 = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=path)
    r2 = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=path)
    torch.cuda.synchronize()
    assert torch.equal(r1[0], r2[0]) and torch.equal(r1[1], r2[1])


def test_host_buffer_entry_point():
    """ssd_forward_host (host inputs and outputs, copies queued by the library)
    gives the device forward's result bit for bit."""
    w = _bf16_case(seed=26)
    inp = generate(w)
    dev = to_dev(inp)
    y_ref, f_ref = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    pin = {k: v.pin_memory() for k, v in inp.items()}
    y_h = torch.empty_like(inp["x"]).pin_memory()
    f_h = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32).pin_memory()
    buf = torch.empty(ssd.forward_host_bytes(shape), dtype=torch.uint8, device="cuda")
    ssd.forward_host(shape, pin["x"], pin["a"], pin["Bm"], pin["Cm"], pin["D"], y_h, f_h, buf)
    torch.cuda.synchronize()
    assert torch.equal(y_h, y_ref.cpu()) and torch.equal(f_h, f_ref.cpu())


def test_fused_bounded_wait_reports_timeout():
    """The fused path's hand-off wait is bounded: with the test flag that keeps
    the first block of chain 0 from publishing its state, the waiting block
    gives up, the device status reads SSD_ERR_TIMEOUT, and the context stays
    usable (a normal call right after is correct)."""
    w = small_case(B=1, T=512, H=8, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=27)
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    if not ssd.path_supported(shape, ssd.PATH_FUSED):
        pytest.skip("fused path not built for this shape")
    ws = ssd.alloc_workspace(shape)
    ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, workspace=ws,
                path=ssd.PATH_FUSED, flags=ssd.FLAG_TEST_STALL)
    assert ssd.device_status(ws) == ssd.SSD_ERR_TIMEOUT
    st, line, block, thread = ssd.device_status_where(ws)
    assert st == ssd.SSD_ERR_TIMEOUT and line > 0 and 0 <= block and 0 <= thread < 1024
    y, fin = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, workspace=ws,
                         path=ssd.PATH_FUSED)
    assert ssd.device_status(ws) == ssd.SSD_OK
    assert ssd.device_status_where(ws) == (ssd.SSD_OK, 0, 0, 0)
    ey, ef = parity_on_chains(inp, y, fin, _all_chains(w))
    assert ey <= TOL_BF16 and ef <= TOL_BF16


def test_fused_on_two_streams():
    """Forwards issued on two streams at once (each with its own workspace):
    the library orders the fused launches, so both finish with SSD_OK and give
    the single-stream result bit for bit."""
    w = small_case(B=2, T=2048, H=16, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=21)
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    if not ssd.path_supported(shape, ssd.PATH_FUSED):
        pytest.skip("fused path does not serve this shape")
    y_ref, f_ref = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk,
                               path=ssd.PATH_FUSED)
    torch.cuda.synchronize()
    streams = [torch.cuda.Stream(), torch.cuda.Stream()]
    wss = [ssd.alloc_workspace(shape) for _ in streams]
    outs = []
    for r in range(6):
        s = r % 2
        with torch.cuda.stream(streams[s]):
            outs.append(ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk,
                                    workspace=wss[s], path=ssd.PATH_FUSED, stream=streams[s]))
    torch.cuda.synchronize()
    for s in range(2):
        assert ssd.device_status(wss[s], streams[s]) == ssd.SSD_OK
    for y, f in outs:
        assert torch.equal(y, y_ref) and torch.equal(f, f_ref)


INIT_CASES = [
    small_case(B=2, T=1024, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=61),
    small_case(B=1, T=384, H=5, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=62),
    small_case(B=1, T=150, H=2, P=70, N=33, G=2, chunk=30, dtype="f32", seed=63),
    small_case(B=2, T=256, H=2, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=64),
]


@pytest.mark.parametrize("w", INIT_CASES + RAGGED[:3], ids=_ids(INIT_CASES + RAGGED[:3]))
@pytest.mark.parametrize("path", _paths(), ids=["simt", "modular", "auto", "fused"])
def test_initial_state_matches_oracle(w, path):
    """ssd_forward_init: every chain starts from a given state h_{-1}; y and the
    final state match the oracle's recurrence started from the same state."""
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    if not ssd.path_supported(shape, path):
        pytest.skip("path does not serve this shape")
    g = torch.Generator().manual_seed(w.seed + 7)
    h0 = torch.randn((w.B, w.H, w.N, w.P), generator=g, dtype=torch.float64)
    y, fin = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=path,
                         initial_state=h0.to(torch.float32).cuda())
    torch.cuda.synchronize()
    prob = O.Problem(*(inp[k].to(torch.float64).numpy() for k in ("x", "a", "Bm", "Cm", "D")))
    ref = O.recurrence(prob, initial=h0.to(torch.float32).to(torch.float64).numpy())
    yr = ref["y"].reshape(w.B, w.H, w.T, w.P).transpose(0, 2, 1, 3)
    ey = rel_err(y.float().cpu().numpy().astype(np.float64), yr)
    ef = rel_err(fin.cpu().numpy().astype(np.float64), ref["final"].reshape(w.B, w.H, w.N, w.P))
    tol = tol_for(w)
    assert ey <= tol, f"y rel err {ey:.3e}"
    assert ef <= tol, f"final rel err {ef:.3e}"


@pytest.mark.parametrize("path", [ssd.PATH_AUTO, ssd.PATH_FUSED, ssd.PATH_MODULAR], ids=["auto", "fused", "modular"])
def test_split_sequence_resumes(path):
    """A sequence run in two calls -- the second from the first's final state,
    passed in place (initial_state aliases final_state) -- gives the one-call
    result up to rounding."""
    w = small_case(B=2, T=2048, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=65)
    inp = generate(w)
    dev = to_dev(inp)
    y_full, f_full = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=path)
    t1 = 768
    part = lambda t, sl: t[:, sl].contiguous()
    y1, f1 = ssd.forward(part(dev["x"], slice(0, t1)), part(dev["a"], slice(0, t1)),
                         part(dev["Bm"], slice(0, t1)), part(dev["Cm"], slice(0, t1)), dev["D"], w.chunk,
                         path=path)
    y2, f2 = ssd.forward(part(dev["x"], slice(t1, None)), part(dev["a"], slice(t1, None)),
                         part(dev["Bm"], slice(t1, None)), part(dev["Cm"], slice(t1, None)), dev["D"],
                         w.chunk, path=path, initial_state=f1, final_state=f1)
    torch.cuda.synchronize()
    y = torch.cat([y1, y2], dim=1).float()
    assert rel_err(y.cpu().numpy(), y_full.float().cpu().numpy()) <= TOL_BF16
    assert rel_err(f1.cpu().numpy(), f_full.cpu().numpy()) <= TOL_BF16


DECODE_CASES = [
    small_case(B=3, T=1, H=8, P=64, N=128, G=2, chunk=1, dtype="bf16", seed=71),
    small_case(B=2, T=1, H=3, P=70, N=33, G=3, chunk=1, dtype="f32", seed=72),
    small_case(B=2, T=1, H=4, P=64, N=64, G=1, chunk=1, dtype="bf16", a_per_state=True, seed=73),
    small_case(B=1, T=1, H=2, P=250, N=20, G=1, chunk=1, dtype="f32", seed=74),
    # 16-byte kernel with the columns split over 4, 2 and 3 blocks (N = 256, P = 12)
    small_case(B=2, T=1, H=3, P=128, N=256, G=1, chunk=1, dtype="f32", seed=76),
    small_case(B=2, T=1, H=2, P=64, N=256, G=2, chunk=1, dtype="bf16", seed=77),
    small_case(B=1, T=1, H=2, P=12, N=16, G=1, chunk=1, dtype="f32", a_per_state=True, seed=78),
]


@pytest.mark.parametrize("w", DECODE_CASES, ids=_ids(DECODE_CASES))
def test_decode_step_matches_oracle(w):
    """One decode step from a given state equals one step of the oracle's
    recurrence from that state (y and the updated state)."""
    inp = generate(w)
    dev = to_dev(inp)
    g = torch.Generator().manual_seed(w.seed + 3)
    h0 = torch.randn((w.B, w.H, w.N, w.P), generator=g).to(torch.float32)
    state = h0.cuda()
    y = ssd.decode_step(dev["x"][:, 0].contiguous(), dev["a"][:, 0].contiguous(),
                        dev["Bm"][:, 0].contiguous(), dev["Cm"][:, 0].contiguous(), dev["D"], state)
    torch.cuda.synchronize()
    prob = O.Problem(*(inp[k].to(torch.float64).numpy() for k in ("x", "a", "Bm", "Cm", "D")))
    ref = O.recurrence(prob, initial=h0.to(torch.float64).numpy())
    yr = ref["y"].reshape(w.B, w.H, 1, w.P)[:, :, 0]
    tol = tol_for(w)
    assert rel_err(y.float().cpu().numpy().astype(np.float64), yr) <= tol
    assert rel_err(state.cpu().numpy().astype(np.float64), ref["final"].reshape(w.B, w.H, w.N, w.P)) <= tol


def test_prefill_then_decode_continues_the_sequence():
    """ssd_forward over the first T0 tokens, then one decode step per token
    from its final state, reproduces the forward over all tokens."""
    w = small_case(B=2, T=512 + 16, H=4, P=64, N=128, G=1, chunk=16, dtype="bf16", seed=75)
    inp = generate(w)
    dev = to_dev(inp)
    T0 = 512
    y_all, f_all = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], 16)
    _, state = ssd.forward(dev["x"][:, :T0].contiguous(), dev["a"][:, :T0].contiguous(),
                           dev["Bm"][:, :T0].contiguous(), dev["Cm"][:, :T0].contiguous(), dev["D"], 256)
    ys = []
    for t in range(T0, w.T):
        ys.append(ssd.decode_step(dev["x"][:, t].contiguous(), dev["a"][:, t].contiguous(),
                                  dev["Bm"][:, t].contiguous(), dev["Cm"][:, t].contiguous(), dev["D"],
                                  state))
    torch.cuda.synchronize()
    y_dec = torch.stack(ys, dim=1).float().cpu().numpy()
    assert rel_err(y_dec, y_all[:, T0:].float().cpu().numpy()) <= TOL_BF16
    assert rel_err(state.cpu().numpy(), f_all.cpu().numpy()) <= TOL_BF16


@pytest.mark.parametrize("path", [ssd.PATH_FUSED, ssd.PATH_MODULAR], ids=["fused", "modular"])
def test_cuda_graph_capture_and_replay(path):
    """The forward records into a CUDA graph (workspace reset, TMA descriptors
    and launches all captured) and each replay computes on the inputs' current
    contents, matching an eager call bit for bit."""
    w = small_case(B=2, T=1024, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=81)
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    ws = ssd.alloc_workspace(shape)
    y = torch.empty_like(dev["x"])
    fin = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device="cuda")
    run = lambda: ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, y=y,
                              final_state=fin, workspace=ws, path=path)
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(side):
        run()  # warm-up outside the capture
    torch.cuda.current_stream().wait_stream(side)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        run()
    for seed in (82, 83):
        new = generate(small_case(B=2, T=1024, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=seed))
        for k in dev:
            dev[k].copy_(new[k].cuda())
        graph.replay()
        torch.cuda.synchronize()
        assert ssd.device_status(ws) == ssd.SSD_OK
        y_g, f_g = y.clone(), fin.clone()
        y_e, f_e = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=path)
        torch.cuda.synchronize()
        assert torch.equal(y_g, y_e) and torch.equal(f_g, f_e)


@pytest.mark.parametrize("per_state,dtype", [(False, "bf16"), (True, "bf16"), (False, "f32")],
                         ids=["scalar_bf16", "per_state_bf16", "scalar_f32"])
def test_discretize_matches_oracle(per_state, dtype):
    """ssd_discretize against the oracle's fp64 discretisation, then the forward
    on its outputs against the oracle recurrence on the oracle's outputs."""
    B, T, H, P, N, G = 2, 512, 4, 64, 128 if not per_state else 64, 1
    g = torch.Generator().manual_seed(93 + per_state)
    dt_raw = (torch.randn((B, T, H), generator=g, dtype=torch.float64) * 1.5 - 2.0).to(torch.float32)
    dt_bias = torch.randn((H,), generator=g, dtype=torch.float64).to(torch.float32)
    A_log = (torch.rand((H, N) if per_state else (H,), generator=g, dtype=torch.float64) * math.log(16)).to(torch.float32)
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    x = torch.randn((B, T, H, P), generator=g, dtype=torch.float64).to(tdt)
    Bm = (torch.randn((B, T, G, N), generator=g, dtype=torch.float64) / math.sqrt(N)).to(tdt)
    Cm = (torch.randn((B, T, G, N), generator=g, dtype=torch.float64) / math.sqrt(N)).to(tdt)
    D = torch.randn((H,), generator=g, dtype=torch.float64).to(torch.float32)
    a_g, x_g = ssd.discretize(dt_raw.cuda(), dt_bias.cuda(), A_log.cuda(), x.cuda())
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    a_r, x_r, _ = O.discretize(f64(dt_raw), f64(dt_bias), f64(A_log), f64(x))
    assert rel_err(a_g.cpu().numpy().astype(np.float64), a_r) <= 1e-6
    assert rel_err(x_g.float().cpu().numpy().astype(np.float64), x_r) <= (4e-3 if dtype == "bf16" else 1e-6)
    # in place on x gives the same
    xc = x.cuda()
    ssd.discretize(dt_raw.cuda(), dt_bias.cuda(), A_log.cuda(), xc, x_out=xc)
    torch.cuda.synchronize()
    assert torch.equal(xc, x_g)
    # the forward on the discretised inputs
    y, fin = ssd.forward(x_g, a_g, Bm.cuda(), Cm.cuda(), D.cuda(), 256 if not per_state else 128)
    torch.cuda.synchronize()
    ref = O.recurrence(O.Problem(x_r, a_r, f64(Bm), f64(Cm), f64(D)))
    yr = ref["y"].reshape(B, H, T, P).transpose(0, 2, 1, 3)
    tol = TOL_BF16 if dtype == "bf16" else 1e-4
    assert rel_err(y.float().cpu().numpy().astype(np.float64), yr) <= tol
    assert rel_err(fin.cpu().numpy().astype(np.float64), ref["final"].reshape(B, H, N, P)) <= tol


FUSED_DISC_CASES = [
    (2, 512, 4, 1, True),    # B, T, H, G, with dt_bias
    (1, 1000, 8, 2, False),  # ragged last block, grouped, no bias
    (2, 384, 3, 1, True),    # three heads per item (scalar decay loads)
]


@pytest.mark.parametrize("case", FUSED_DISC_CASES, ids=[f"B{c[0]}_T{c[1]}_H{c[2]}_G{c[3]}" for c in FUSED_DISC_CASES])
def test_forward_discretized_matches_oracle(case):
    """ssd_forward_discretized (the discretisation inside the fused forward)
    against the oracle's fp64 discretisation followed by its recurrence, and
    against the library's two launches (ssd_discretize, then ssd_forward)."""
    B, T, H, G, with_bias = case
    P, N = 64, 128
    g = torch.Generator().manual_seed(97 + T)
    dt_raw = (torch.randn((B, T, H), generator=g, dtype=torch.float64) * 1.5 - 2.0).to(torch.float32)
    dt_bias = torch.randn((H,), generator=g, dtype=torch.float64).to(torch.float32) if with_bias else None
    A_log = (torch.rand((H,), generator=g, dtype=torch.float64) * math.log(16)).to(torch.float32)
    x = torch.randn((B, T, H, P), generator=g, dtype=torch.float64).to(torch.bfloat16)
    Bm = (torch.randn((B, T, G, N), generator=g, dtype=torch.float64) / math.sqrt(N)).to(torch.bfloat16)
    Cm = (torch.randn((B, T, G, N), generator=g, dtype=torch.float64) / math.sqrt(N)).to(torch.bfloat16)
    D = torch.randn((H,), generator=g, dtype=torch.float64).to(torch.float32)
    dev = lambda t: t.cuda() if t is not None else None
    y, fin = ssd.forward_discretized(dev(x), dev(dt_raw), dev(dt_bias), dev(A_log), dev(Bm), dev(Cm), dev(D), 256)
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    bias64 = f64(dt_bias) if dt_bias is not None else np.zeros((H,))
    a_r, x_r, _ = O.discretize(f64(dt_raw), bias64, f64(A_log), f64(x))
    ref = O.recurrence(O.Problem(x_r, a_r, f64(Bm), f64(Cm), f64(D)))
    yr = ref["y"].reshape(B, H, T, P).transpose(0, 2, 1, 3)
    assert rel_err(y.float().cpu().numpy().astype(np.float64), yr) <= TOL_BF16
    assert rel_err(fin.cpu().numpy().astype(np.float64), ref["final"].reshape(B, H, N, P)) <= TOL_BF16
    # the two-launch form of the same computation
    a2, x2 = ssd.discretize(dev(dt_raw), dev(dt_bias), dev(A_log), dev(x))
    y2, f2 = ssd.forward(x2, a2, dev(Bm), dev(Cm), dev(D), 256, path=ssd.PATH_FUSED)
    torch.cuda.synchronize()
    assert rel_err(y.float().cpu().numpy().astype(np.float64), y2.float().cpu().numpy().astype(np.float64)) <= TOL_BF16
    assert rel_err(fin.cpu().numpy().astype(np.float64), f2.cpu().numpy().astype(np.float64)) <= TOL_BF16


def test_forward_discretized_unsupported_shape():
    """Shapes the fused path does not serve are refused before any launch."""
    B, T, H, P, N = 1, 256, 2, 64, 128
    x = torch.zeros((B, T, H, P), dtype=torch.float32, device="cuda")
    dt_raw = torch.zeros((B, T, H), dtype=torch.float32, device="cuda")
    A_log = torch.zeros((H,), dtype=torch.float32, device="cuda")
    Bm = torch.zeros((B, T, 1, N), dtype=torch.float32, device="cuda")
    with pytest.raises(ssd.SSDError) as e:
        ssd.forward_discretized(x, dt_raw, None, A_log, Bm, Bm, None, 256)
    assert e.value.code == ssd.SSD_ERR_UNSUPPORTED


def test_discretize_odd_rows():
    """Rows whose length is not a multiple of 16 bytes (the per-row path)."""
    B, T, H, P, N = 1, 33, 3, 70, 5
    g = torch.Generator().manual_seed(95)
    dt_raw = torch.randn((B, T, H), generator=g, dtype=torch.float64).to(torch.float32)
    A_log = torch.rand((H, N), generator=g, dtype=torch.float64).to(torch.float32)
    x = torch.randn((B, T, H, P), generator=g, dtype=torch.float64).to(torch.float32)
    a_g, x_g = ssd.discretize(dt_raw.cuda(), None, A_log.cuda(), x.cuda())
    torch.cuda.synchronize()
    f64 = lambda t: t.to(torch.float64).numpy()
    a_r, x_r, _ = O.discretize(f64(dt_raw), None, f64(A_log), f64(x))
    assert rel_err(a_g.cpu().numpy().astype(np.float64), a_r) <= 1e-6
    assert rel_err(x_g.cpu().numpy().astype(np.float64), x_r) <= 1e-6


SEGMENT_CASES = [
    small_case(B=2, T=4096, H=8, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=104),
    small_case(B=1, T=4000, H=4, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=105, u_mean=-4.0),
    small_case(B=2, T=1024, H=4, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=103),
    small_case(B=1, T=600, H=3, P=20, N=12, G=1, chunk=64, dtype="f32", seed=106),
]


@pytest.mark.parametrize("w", SEGMENT_CASES, ids=_ids(SEGMENT_CASES))
@pytest.mark.parametrize("with_init", [False, True], ids=["zero", "init"])
def test_sequence_segments_with_library_kernels(w, with_init):
    """What every rank of the sequence-sharded forward does, with the
    library's kernels, for a sequence cut into 4 segments: each segment's
    state from zero and total decay (ssd_segment_state), their combine into
    the state entering every segment (ssd_state_combine), and one forward per
    segment from that state (ssd_forward_init).  The segments' y, joined, and
    the combine's last state equal the fp64 recurrence over the whole
    sequence (the oracle, not the library's whole-sequence forward); the
    segment states and totals equal the oracle's too."""
    inp = generate(w)
    dev = to_dev(inp)
    S = 4
    bounds = [round(s * w.T / S) for s in range(S + 1)]
    # a fresh (16-byte aligned) copy per segment, as each rank would hold
    seg = lambda t, s: t[:, bounds[s]:bounds[s + 1]].clone()
    parts = [[seg(dev[k], s) for k in ("x", "a", "Bm", "Cm")] for s in range(S)]
    h0 = None
    if with_init:
        g = torch.Generator().manual_seed(w.seed + 3)
        h0 = torch.randn((w.B, w.H, w.N, w.P), generator=g, dtype=torch.float64).to(torch.float32)
    fins, tots = [], []
    for x, a, Bm, Cm in parts:
        f, tot = ssd.segment_state(x, a, Bm, w.chunk)
        fins.append(f)
        tots.append(tot)
    totals = torch.stack(tots).contiguous()
    h_in = ssd.state_combine(torch.stack(fins).contiguous(), totals, None if h0 is None else h0.cuda())
    ys = [ssd.forward(x, a, Bm, Cm, dev["D"], w.chunk, initial_state=h_in[s].contiguous())[0]
          for s, (x, a, Bm, Cm) in enumerate(parts)]
    torch.cuda.synchronize()
    tol = tol_for(w)
    f64 = lambda t: t.to(torch.float64).numpy()
    prob = O.Problem(*(f64(inp[k]) for k in ("x", "a", "Bm", "Cm", "D")))
    ref = O.recurrence(prob, initial=None if h0 is None else f64(h0))
    yr = ref["y"].reshape(w.B, w.H, w.T, w.P).transpose(0, 2, 1, 3)
    y = torch.cat(ys, dim=1).float().cpu().numpy().astype(np.float64)
    assert rel_err(y, yr) <= tol, f"y rel err {rel_err(y, yr):.3e}"
    fr = ref["final"].reshape(w.B, w.H, w.N, w.P)
    assert rel_err(h_in[S].cpu().numpy().astype(np.float64), fr) <= tol
    # each segment's own state from zero and total log-decay against the oracle
    for s in range(S):
        sub = O.Problem(*(f64(seg(inp[k], s)) for k in ("x", "a", "Bm", "Cm")), f64(inp["D"]))
        rs = O.recurrence(sub, want_y=False)
        assert rel_err(fins[s].cpu().numpy().astype(np.float64),
                       rs["final"].reshape(w.B, w.H, w.N, w.P)) <= tol, f"segment {s} state"
        a64 = f64(seg(inp["a"], s))
        assert rel_err(tots[s].cpu().numpy().astype(np.float64), a64.sum(axis=1)) <= 1e-5


# few long sequences: SSD_PATH_SPLIT cuts each into pieces (the piece states
# from zero, their combine, then the fused kernel over all pieces); pieces of
# 4100 tokens end inside a 128-token block
SPLIT_CASES = [
    small_case(B=1, T=16384, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=81, u_mean=-4.0),
    small_case(B=2, T=12288, H=2, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=82),
    small_case(B=1, T=8200, H=3, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=83, u_mean=-5.0),
]


@pytest.mark.parametrize("w", SPLIT_CASES, ids=_ids(SPLIT_CASES))
@pytest.mark.parametrize("with_init", [False, True], ids=["zero", "init"])
def test_split_path_matches_oracle(w, with_init):
    """The split path equals the fp64 recurrence over the whole sequence, from
    a zero or a given initial state; AUTO takes it for these shapes."""
    inp = generate(w)
    dev = to_dev(inp)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    assert ssd.path_supported(shape, ssd.PATH_SPLIT)
    assert ssd.auto_path(shape) == ssd.PATH_SPLIT
    h0 = None
    if with_init:
        g = torch.Generator().manual_seed(w.seed + 9)
        h0 = torch.randn((w.B, w.H, w.N, w.P), generator=g, dtype=torch.float64).to(torch.float32)
    y, fin = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=ssd.PATH_SPLIT,
                         initial_state=None if h0 is None else h0.cuda())
    torch.cuda.synchronize()
    prob = O.Problem(*(inp[k].to(torch.float64).numpy() for k in ("x", "a", "Bm", "Cm", "D")))
    ref = O.recurrence(prob, initial=None if h0 is None else h0.to(torch.float64).numpy())
    yr = ref["y"].reshape(w.B, w.H, w.T, w.P).transpose(0, 2, 1, 3)
    ey = rel_err(y.float().cpu().numpy().astype(np.float64), yr)
    ef = rel_err(fin.cpu().numpy().astype(np.float64), ref["final"].reshape(w.B, w.H, w.N, w.P))
    assert ey <= TOL_BF16, f"y rel err {ey:.3e}"
    assert ef <= TOL_BF16, f"final rel err {ef:.3e}"


def test_per_state_extreme_decay():
    """Per-state decays down to -1e4 (the state forgets at once) mixed with
    slow ones: the tensor-core steps stay finite and match the oracle (every
    weight they form is a product of factors <= 1)."""
    w = small_case(B=1, T=512, H=2, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True, seed=33)
    inp = generate(w)
    g = torch.Generator().manual_seed(34)
    mask = torch.rand(inp["a"].shape, generator=g) < 0.05
    inp["a"] = torch.where(mask, torch.full_like(inp["a"], -1e4), inp["a"]).contiguous()
    dev = to_dev(inp)
    for path in (ssd.PATH_MODULAR, ssd.PATH_AUTO):
        y, fin = run_forward(w, dev, path=path)
        assert torch.isfinite(y.float()).all() and torch.isfinite(fin).all()
        ey, ef = parity_on_chains(inp, y, fin, _all_chains(w))
        assert ey <= TOL_BF16 and ef <= TOL_BF16, (path, ey, ef)
