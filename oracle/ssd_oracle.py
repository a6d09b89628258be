"""Python face of the fp64 CPU oracle (ssd_oracle.c) -- TEST INFRASTRUCTURE.

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this module.  It shares nothing with the CUDA library:
it loads ``liboracle.so`` (built from ``ssd_oracle.c`` by ``build_oracle``)
and passes plain float64 numpy arrays.

Routes (see the C file for the equations and their sources):
  recurrence(...)  O1, the step recurrence h_t = e^{a_t} h_{t-1} + B_t x_t^T
  brute(...)       O2, the materialised 1-semiseparable matrix (tiny T)
  chunked(...)     O3, the chunked algorithm with every intermediate
  backward(...)    O4, gradients of the recurrence by its adjoint (numpy fp64)
  discretize(...)  the selective discretisation in front of the operator (numpy)

Parity is pinned for every route (tests/test_oracle_pins.py); nothing here is
"parity unpinned".
"""
from __future__ import annotations

import ctypes
import os
import subprocess
from dataclasses import dataclass

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "liboracle.so")


def build_oracle(force: bool = False) -> str:
    """Compile ssd_oracle.c with gcc into liboracle.so (next to the source)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(
            ["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-pthread", _SRC, "-o", tmp, "-lm"]
        )
        os.replace(tmp, _LIB)
    return _LIB


class _Shape(ctypes.Structure):
    _fields_ = [(n, ctypes.c_int) for n in ("B", "T", "H", "P", "G", "N", "chunk", "a_per_state")]


_lib = None


def _load():
    global _lib
    if _lib is None:
        build_oracle()
        lib = ctypes.CDLL(_LIB)
        dp = ctypes.POINTER(ctypes.c_double)
        ip = ctypes.POINTER(ctypes.c_int)
        sp = ctypes.POINTER(_Shape)
        lib.oracle_recurrence.argtypes = [sp, dp, dp, dp, dp, dp, ip, ctypes.c_int, ctypes.c_int,
                                          dp, dp, dp, ctypes.c_int]
        lib.oracle_recurrence_init.argtypes = [sp, dp, dp, dp, dp, dp, dp, ip, ctypes.c_int, ctypes.c_int,
                                               dp, dp, dp, ctypes.c_int]
        lib.oracle_brute.argtypes = [sp, dp, dp, dp, dp, dp, ip, ctypes.c_int, dp, dp, ctypes.c_int]
        lib.oracle_chunked.argtypes = [sp, dp, dp, dp, dp, dp, ip, ctypes.c_int, dp, dp, dp, dp, dp,
                                       ctypes.c_int]
        for f in (lib.oracle_recurrence, lib.oracle_recurrence_init, lib.oracle_brute, lib.oracle_chunked):
            f.restype = ctypes.c_int
        lib.oracle_set_mutation.argtypes = [ctypes.c_int]
        lib.oracle_set_mutation.restype = None
        lib.oracle_get_mutation.restype = ctypes.c_int
        _lib = lib
    return _lib


def set_mutation(m: int) -> None:
    """Plant mistake number ``m`` in every oracle route (0 = none).  Tests only."""
    _load().oracle_set_mutation(int(m))


def default_threads() -> int:
    return max(1, os.cpu_count() or 1)


@dataclass
class Problem:
    """One SSD problem as float64 arrays, exactly the values a device receives."""

    x: np.ndarray  # [B,T,H,P]
    a: np.ndarray  # [B,T,H] or [B,T,H,N]
    Bm: np.ndarray  # [B,T,G,N]
    Cm: np.ndarray  # [B,T,G,N]
    D: np.ndarray | None  # [H]

    @property
    def dims(self):
        B, T, H, P = self.x.shape
        G, N = self.Bm.shape[2], self.Bm.shape[3]
        return B, T, H, P, G, N

    @property
    def a_per_state(self) -> bool:
        return self.a.ndim == 4


def _f64(arr):
    if arr is None:
        return None
    out = np.ascontiguousarray(np.asarray(arr, dtype=np.float64))
    return out


def _ptr(arr):
    if arr is None:
        return ctypes.POINTER(ctypes.c_double)()
    return arr.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _shape(prob: Problem, chunk: int) -> _Shape:
    B, T, H, P, G, N = prob.dims
    return _Shape(B, T, H, P, G, N, int(chunk), int(prob.a_per_state))


def _chains(prob: Problem, chains):
    B, T, H, P, G, N = prob.dims
    if chains is None:
        chains = [(b, h) for b in range(B) for h in range(H)]
    arr = np.ascontiguousarray(np.asarray(chains, dtype=np.int32).reshape(-1, 2))
    if arr.size and (arr[:, 0].max() >= B or arr[:, 1].max() >= H or arr.min() < 0):
        raise ValueError("chain index out of range")
    return arr


def _prep(prob: Problem):
    p = Problem(_f64(prob.x), _f64(prob.a), _f64(prob.Bm), _f64(prob.Cm), _f64(prob.D))
    B, T, H, P, G, N = p.dims
    if H % G:
        raise ValueError("H must be a multiple of G")
    if p.a.shape[:3] != (B, T, H) or (p.a.ndim == 4 and p.a.shape[3] != N):
        raise ValueError("a has the wrong shape")
    if p.Cm.shape != p.Bm.shape:
        raise ValueError("Bm and Cm differ in shape")
    return p


def recurrence(prob: Problem, chains=None, t_end=None, chunk=0, want_y=True, nthreads=None,
               initial=None):
    """O1.  Returns dict(y=[C,T,P] (rows >= t_end are zero), final=[C,N,P],
    bounds=[C,nc,N,P] state after each chunk when chunk>0).  ``initial``
    [B,H,N,P]: the state h_{-1} each chain starts from (default zero)."""
    lib = _load()
    p = _prep(prob)
    B, T, H, P, G, N = p.dims
    init = _f64(initial)
    if init is not None and init.shape != (B, H, N, P):
        raise ValueError("initial state must be [B,H,N,P]")
    ch = _chains(p, chains)
    C = ch.shape[0]
    t_end = T if t_end is None else int(t_end)
    y = np.zeros((C, T, P)) if want_y else None
    fin = np.zeros((C, N, P))
    bounds = np.zeros((C, T // chunk, N, P)) if chunk else None
    rc = lib.oracle_recurrence_init(ctypes.byref(_shape(p, chunk)), _ptr(p.x), _ptr(p.a), _ptr(p.Bm),
                                    _ptr(p.Cm), _ptr(p.D), _ptr(init),
                                    ch.ctypes.data_as(ctypes.POINTER(ctypes.c_int)),
                                    C, t_end, _ptr(y), _ptr(fin), _ptr(bounds),
                                    nthreads or default_threads())
    if rc:
        raise ValueError("oracle_recurrence rejected its arguments")
    return {"y": y, "final": fin, "bounds": bounds, "chains": ch}


def brute(prob: Problem, chains=None, nthreads=None):
    """O2 (O(T^3 N) per chain).  Returns dict(y=[C,T,P], final=[C,N,P])."""
    lib = _load()
    p = _prep(prob)
    B, T, H, P, G, N = p.dims
    if T > 512:
        raise ValueError("brute force is for tiny T")
    ch = _chains(p, chains)
    C = ch.shape[0]
    y = np.zeros((C, T, P))
    fin = np.zeros((C, N, P))
    rc = lib.oracle_brute(ctypes.byref(_shape(p, 0)), _ptr(p.x), _ptr(p.a), _ptr(p.Bm), _ptr(p.Cm),
                          _ptr(p.D), ch.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), C, _ptr(y),
                          _ptr(fin), nthreads or default_threads())
    if rc:
        raise ValueError("oracle_brute rejected its arguments")
    return {"y": y, "final": fin, "chains": ch}


def chunked(prob: Problem, chunk: int, chains=None, nthreads=None):
    """O3.  Returns dict(cum=[C,nc,Q,Na], S=[C,nc,N,P], Hin=[C,nc,N,P], y=[C,T,P],
    final=[C,N,P]); Na = N for per-state decay, else 1."""
    lib = _load()
    p = _prep(prob)
    B, T, H, P, G, N = p.dims
    if chunk <= 0 or T % chunk:
        raise ValueError("chunk must divide T")
    ch = _chains(p, chains)
    C = ch.shape[0]
    nc = T // chunk
    Na = N if p.a_per_state else 1
    cum = np.zeros((C, nc, chunk, Na))
    S = np.zeros((C, nc, N, P))
    Hin = np.zeros((C, nc, N, P))
    y = np.zeros((C, T, P))
    fin = np.zeros((C, N, P))
    rc = lib.oracle_chunked(ctypes.byref(_shape(p, chunk)), _ptr(p.x), _ptr(p.a), _ptr(p.Bm),
                            _ptr(p.Cm), _ptr(p.D), ch.ctypes.data_as(ctypes.POINTER(ctypes.c_int)), C,
                            _ptr(cum), _ptr(S), _ptr(Hin), _ptr(y), _ptr(fin),
                            nthreads or default_threads())
    if rc:
        raise ValueError("oracle_chunked rejected its arguments")
    return {"cum": cum, "S": S, "Hin": Hin, "y": y, "final": fin, "chains": ch}


def to_bthp(res_y: np.ndarray, chains: np.ndarray, B: int, H: int) -> np.ndarray:
    """Scatter per-chain y [C,T,P] into [B,T,H,P] (all chains must be present)."""
    C, T, P = res_y.shape
    out = np.zeros((B, T, H, P))
    for c, (b, h) in enumerate(chains):
        out[b, :, h, :] = res_y[c]
    return out


def discretize(dt_raw, dt_bias, A_log, x):
    """The selective discretisation in front of the operator, plain fp64 numpy
    (llms.blog "The Selection Mechanism": Delta_t = softplus(Parameter +
    W_Delta x_t), Abar_t = exp(Delta_t A), Bbar_t = Delta_t B_t; and
    "Continuous-to-Discrete Discretization": Bbar ~ Delta B).  With the
    operator's inputs as log-decays and the per-head step folded into the
    input (Bbar_t x_t = B_t (Delta_t x_t)):
        dt = softplus(dt_raw + dt_bias)                  [B,T,H]
        a  = dt * A,  A = -exp(A_log)                    [B,T,H] (A_log [H])
                                                         or [B,T,H,N] (A_log [H,N])
        xd = dt * x                                      [B,T,H,P]
    softplus(z) = log(1 + e^z), evaluated as max(z, 0) + log1p(e^{-|z|}).
    Returns (a, xd, dt)."""
    z = np.asarray(dt_raw, dtype=np.float64)
    if dt_bias is not None:
        z = z + np.asarray(dt_bias, dtype=np.float64)[None, None, :]
    dt = np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))
    A = -np.exp(np.asarray(A_log, dtype=np.float64))
    if A.ndim == 1:
        a = dt * A[None, None, :]
    else:
        a = dt[..., None] * A[None, None, :, :]
    xd = dt[..., None] * np.asarray(x, dtype=np.float64)
    return a, xd, dt


_BACKWARD_MUTATION = 0


def set_backward_mutation(m: int) -> None:
    """Plant mistake number ``m`` in backward() (0 = none).  Tests only."""
    global _BACKWARD_MUTATION
    _BACKWARD_MUTATION = int(m)


def backward(prob: Problem, dy, dfinal=None, initial=None):
    """Gradients of the scalar l = sum_t dy_t . y_t + <dfinal, h_{T-1}> with
    respect to every input, by reverse-mode differentiation of the step
    recurrence (O1): the plain definition, in fp64 numpy, with every state
    h_t kept (the pages' kernels recompute the states in the backward pass
    instead of storing them -- llms.blog "State Space Models and Mamba ...",
    "Hardware-Aware Parallel Associative Scan", item on the direct output
    projection).

    Forward   h_t = e^{a_t} o h_{t-1} + B_t x_t^T,  y_t = h_t^T C_t + D x_t
    Adjoint   g_t = dl/dh_t = C_t dy_t^T + e^{a_{t+1}} o g_{t+1},
              g_{T-1} = C_{T-1} dy_{T-1}^T + dfinal
    then      dx_t = g_t^T B_t + D dy_t        dB_t = g_t x_t (summed over a group's heads)
              dC_t = h_t dy_t                  da_t = <g_t, e^{a_t} o h_{t-1}>  (per n if per-state)
              dD   = sum_t dy_t . x_t          d initial = e^{a_0} o g_0
    dy [B,T,H,P], dfinal / initial [B,H,N,P] or None (zero).  Returns a dict
    dx, da, dBm, dCm, dD, dinit with the inputs' shapes."""
    p = _prep(prob)
    B, T, H, P, G, N = p.dims
    hg = H // G
    dy = _f64(dy)
    per_state = p.a_per_state
    grp = np.arange(H) // hg
    h = np.zeros((B, H, N, P)) if initial is None else _f64(initial).copy()
    hs = np.zeros((T + 1, B, H, N, P))  # hs[t + 1] = h_t, hs[0] = h_{-1}
    hs[0] = h
    for t in range(T):
        e = np.exp(p.a[:, t])                                  # [B,H] or [B,H,N]
        e = e[..., None, None] if not per_state else e[..., None]
        Bt = p.Bm[:, t][:, grp]                                # [B,H,N]
        h = e * h + Bt[..., None] * p.x[:, t][:, :, None, :]
        hs[t + 1] = h
    mut = _BACKWARD_MUTATION
    g = np.zeros((B, H, N, P)) if (dfinal is None or mut == 1) else _f64(dfinal).copy()
    dx = np.zeros_like(p.x)
    da = np.zeros_like(p.a)
    dBh = np.zeros((B, T, H, N))
    dCh = np.zeros((B, T, H, N))
    Dv = np.zeros(H) if p.D is None else p.D
    for t in range(T - 1, -1, -1):
        Ct = p.Cm[:, t][:, grp]                                # [B,H,N]
        Bt = p.Bm[:, t][:, grp]
        g = g + (Bt if mut == 2 else Ct)[..., None] * dy[:, t][:, :, None, :]  # g_t
        dx[:, t] = np.einsum("bhnp,bhn->bhp", g, Bt) + (0 if mut == 3 else Dv[None, :, None] * dy[:, t])
        dBh[:, t] = np.einsum("bhnp,bhp->bhn", hs[t + 1] if mut == 4 else g, p.x[:, t])
        dCh[:, t] = np.einsum("bhnp,bhp->bhn", hs[t] if mut == 5 else hs[t + 1], dy[:, t])
        e = np.exp(p.a[:, t])
        if per_state:
            da[:, t] = np.einsum("bhnp,bhnp->bhn", g, (1 if mut == 6 else e[..., None]) * hs[t])
            g = (1 if mut == 7 else e[..., None]) * g
        else:
            da[:, t] = np.einsum("bhnp,bhnp->bh", g, hs[t]) * (1 if mut == 6 else e)
            g = (1 if mut == 7 else e[..., None, None]) * g
    dBm = dBh.reshape(B, T, G, hg, N).sum(axis=3)
    dCm = dCh.reshape(B, T, G, hg, N).sum(axis=3)
    dD = np.einsum("bthp,bthp->h", dy, p.x)
    return {"dx": dx, "da": da, "dBm": dBm, "dCm": dCm, "dD": dD, "dinit": g,
            "y": np.einsum("tbhnp,bthn->bthp", hs[1:], p.Cm[:, :, grp]) + Dv[None, None, :, None] * p.x,
            "final": hs[T]}
