"""Helpers for the GPU parity tests: run the library, run the oracle on the
same seeded inputs, compare with the parity metric
||y - y_ref||_inf / ||y_ref||_inf over the compared outputs."""
from __future__ import annotations

import numpy as np
import torch

from oracle import ssd_oracle as O
from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.workloads import Workload, generate

TOL_F32 = 1e-4
TOL_BF16 = 2e-2


def tol_for(w: Workload) -> float:
    return TOL_F32 if w.dtype == "f32" else TOL_BF16


def to_dev(inp):
    return {k: v.cuda() for k, v in inp.items()}


def chain_problem(inp, b: int, h: int, t_end: int | None = None) -> O.Problem:
    """float64 single-chain problem (B=H=G=1) holding exactly the values the
    device received for chain (b, h)."""
    x, a, Bm, Cm, D = inp["x"], inp["a"], inp["Bm"], inp["Cm"], inp["D"]
    H, G = x.shape[2], Bm.shape[2]
    g = h // (H // G)
    T = x.shape[1] if t_end is None else t_end
    f = lambda t: t.to(torch.float64).numpy()
    xa = f(x[b:b + 1, :T, h:h + 1, :].contiguous())
    aa = f(a[b:b + 1, :T, h:h + 1].contiguous())
    ba = f(Bm[b:b + 1, :T, g:g + 1, :].contiguous())
    ca = f(Cm[b:b + 1, :T, g:g + 1, :].contiguous())
    da = f(D[h:h + 1].contiguous())
    return O.Problem(xa, aa, ba, ca, da)


def oracle_chains(inp, chains, t_end=None, chunk=0, nthreads=None):
    """O1 per chain -> list of (y [t_end,P], final [N,P], bounds or None)."""
    out = []
    for (b, h) in chains:
        prob = chain_problem(inp, b, h, t_end)
        r = O.recurrence(prob, chunk=chunk, nthreads=nthreads)
        out.append((r["y"][0], r["final"][0], None if r["bounds"] is None else r["bounds"][0]))
    return out


def rel_err(got: np.ndarray, ref: np.ndarray) -> float:
    den = float(np.max(np.abs(ref)))
    return float(np.max(np.abs(got - ref))) / (den if den > 0 else 1.0)


def run_forward(w: Workload, dev, path=ssd.PATH_AUTO, chunk=None):
    y, fin = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"],
                         w.chunk if chunk is None else chunk, path=path)
    torch.cuda.synchronize()
    return y, fin


def parity_on_chains(inp, y, fin, chains, t_end=None):
    """max relative error of y (and of the final state when t_end is None)
    over the given chains, both against O1."""
    refs = oracle_chains(inp, chains, t_end)
    T = inp["x"].shape[1] if t_end is None else t_end
    ys = np.concatenate([y[b, :T, h, :].float().cpu().numpy().astype(np.float64)[None]
                         for (b, h) in chains])
    yr = np.concatenate([r[0][None] for r in refs])
    ey = rel_err(ys, yr)
    ef = None
    if t_end is None and fin is not None:
        fs = np.concatenate([fin[b, h].cpu().numpy().astype(np.float64)[None] for (b, h) in chains])
        fr = np.concatenate([r[1][None] for r in refs])
        ef = rel_err(fs, fr)
    return ey, ef


def whole_tensor_parity(inp, y, fin, nthreads=None, budget_bytes=3 << 30):
    """||y - y_ref||_inf / ||y_ref||_inf over the WHOLE output tensor, and the
    same metric over the whole final state, against O1 (fp64 recurrence).

    The oracle runs on batches of consecutive B/C groups of one batch row (a
    group's heads share Bm/Cm, so a sub-problem of whole groups keeps the
    head-to-group map), and the comparison streams chain by chain, so neither
    the fp64 y nor the fp64 inputs are ever held whole.  Returns
    (y_err, final_err, max|y_ref|)."""
    import os
    x, a, Bm, Cm, D = inp["x"], inp["a"], inp["Bm"], inp["Cm"], inp["D"]
    B, T, H, P = x.shape
    G, N = Bm.shape[2], Bm.shape[3]
    HG = H // G
    nthreads = nthreads or (os.cpu_count() or 1)
    # fp64 bytes one chain costs: x and y, its share of B/C and a
    per_chain = 8 * T * (2 * P + 2 * N / HG + (N if a.dim() == 4 else 1))
    groups_per_batch = max(1, min(G, max(1, nthreads // HG), int(budget_bytes // (per_chain * HG))))
    f = lambda t: t.to(torch.float64).numpy()
    dmax = rmax = fdmax = frmax = 0.0
    yc = y.cpu() if y.is_cuda else y
    fc = (fin.cpu() if fin.is_cuda else fin) if fin is not None else None
    for b in range(B):
        for g0 in range(0, G, groups_per_batch):
            g1 = min(G, g0 + groups_per_batch)
            h0, h1 = g0 * HG, g1 * HG
            prob = O.Problem(f(x[b:b + 1, :, h0:h1].contiguous()), f(a[b:b + 1, :, h0:h1].contiguous()),
                             f(Bm[b:b + 1, :, g0:g1].contiguous()), f(Cm[b:b + 1, :, g0:g1].contiguous()),
                             f(D[h0:h1].contiguous()))
            r = O.recurrence(prob, nthreads=nthreads)
            del prob
            for c in range(h1 - h0):
                ref = r["y"][c]
                got = yc[b, :, h0 + c, :].to(torch.float64).numpy()
                dmax = max(dmax, float(np.max(np.abs(got - ref))))
                rmax = max(rmax, float(np.max(np.abs(ref))))
                if fc is not None:
                    fr = r["final"][c]
                    fdmax = max(fdmax, float(np.max(np.abs(fc[b, h0 + c].numpy().astype(np.float64) - fr))))
                    frmax = max(frmax, float(np.max(np.abs(fr))))
            del r
    ey = dmax / (rmax if rmax > 0 else 1.0)
    ef = None if fc is None else fdmax / (frmax if frmax > 0 else 1.0)
    return ey, ef, rmax
