"""Seeded synthetic inputs for the chunked SSD forward.

This module only draws random numbers and casts them: it holds none of the
SSD arithmetic, and both the CUDA path and the CPU oracle take their inputs
from it.  The value recipes follow the Mamba-2-shaped workloads this library
is measured on (x ~ N(0,1); B, C ~ N(0, 1/N) in variance; log-decays
a = -softplus(u) * exp(A_log) with u ~ N(mu, 1) per (b, t, h) and
A_log ~ U(0, log 16) per head (per (head, state) for the per-state variant);
D ~ N(0, 1) per head).  The discretisation the pages describe (Abar =
exp(Delta A), "State Space Models and Mamba ...", "The Selection Mechanism")
is what these log-decays stand for; it is applied here, at input synthesis,
not inside the library.

Draw order is fixed (x, Bm, Cm, u or dt, A_log, D), every draw is float64
from one ``torch.Generator('cpu')`` seeded per workload, and large tensors are
drawn in blocks of whole batch rows so memory stays bounded.
"""
from __future__ import annotations

import math
from dataclasses import dataclass, field, replace

import torch


@dataclass(frozen=True)
class Workload:
    name: str
    B: int
    T: int
    H: int
    P: int
    N: int
    G: int
    chunk: int
    dtype: str  # "f32" or "bf16": the type of x, Bm, Cm and y
    a_per_state: bool = False
    seed: int = 0
    decay: str = "softplus"  # "softplus" (a = -softplus(u) exp(A_log)) or "uniform_dt" (a = -dt)
    u_mean: float = -2.0
    with_D: bool = True
    note: str = ""

    @property
    def nc(self) -> int:
        return -(-self.T // self.chunk)

    @property
    def tokens(self) -> int:
        return self.B * self.T

    def scaled(self, **kw) -> "Workload":
        return replace(self, **kw)


WORKLOADS = {
    "tiny_f32": Workload("tiny_f32", B=1, T=256, H=1, P=16, N=16, G=1, chunk=64, dtype="f32",
                         seed=0, decay="uniform_dt", with_D=False,
                         note="fp32 end to end; a=-dt, dt~U(0.001,0.2); D=0"),
    "mamba2_130m": Workload("mamba2_130m", B=8, T=2048, H=24, P=64, N=128, G=1, chunk=256,
                            dtype="bf16", seed=1, u_mean=-2.0,
                            note="Mamba-2-130M-shaped layer"),
    "mamba2_2p7b": Workload("mamba2_2p7b", B=4, T=8192, H=80, P=64, N=128, G=1, chunk=256,
                            dtype="bf16", seed=2, u_mean=-2.0,
                            note="Mamba-2-2.7B-shaped layer, returns the final state"),
    "long_seq": Workload("long_seq", B=1, T=262144, H=32, P=64, N=128, G=8, chunk=256,
                         dtype="bf16", seed=3, u_mean=-4.0,
                         note="long sequence, 4 heads per B/C group, slow decay"),
    "diag_ssm": Workload("diag_ssm", B=4, T=4096, H=16, P=64, N=64, G=1, chunk=128,
                         dtype="bf16", a_per_state=True, seed=4, u_mean=-2.0,
                         note="per-state log-decay a[B,T,H,N]"),
}
# the order in which the workloads are listed in the measurement contract
ORDER = ["tiny_f32", "mamba2_130m", "mamba2_2p7b", "long_seq", "diag_ssm"]


def torch_dtype(w: Workload) -> torch.dtype:
    return torch.float32 if w.dtype == "f32" else torch.bfloat16


def _softplus64(u: torch.Tensor) -> torch.Tensor:
    # log(1 + e^u) in float64, overflow-safe
    return torch.where(u > 30, u, torch.log1p(torch.exp(torch.clamp(u, max=30.0))))


def generate(w: Workload, seed: int | None = None, rows_per_block: int = 1 << 22):
    """Draw the inputs of workload ``w`` on the CPU.

    Returns a dict of CPU tensors: x [B,T,H,P], Bm/Cm [B,T,G,N] in the
    workload dtype; a [B,T,H] (or [B,T,H,N]) float32 log-decays; D [H] float32
    (zeros when the workload has no skip term).
    """
    g = torch.Generator(device="cpu")
    g.manual_seed(w.seed if seed is None else seed)
    dt = torch_dtype(w)
    B, T, H, P, N, G = w.B, w.T, w.H, w.P, w.N, w.G

    def normal(shape, std):
        # drawn as float64 in blocks along the leading (token) axes
        out = torch.empty(shape, dtype=dt)
        flat = out.view(-1, shape[-1] * shape[-2])  # [B*T, inner]
        rows = flat.shape[0]
        step = max(1, rows_per_block // flat.shape[1])
        for r0 in range(0, rows, step):
            r1 = min(rows, r0 + step)
            blk = torch.randn((r1 - r0, flat.shape[1]), generator=g, dtype=torch.float64)
            flat[r0:r1] = (blk * std).to(dt)
        return out

    x = normal((B, T, H, P), 1.0)
    Bm = normal((B, T, G, N), 1.0 / math.sqrt(N))
    Cm = normal((B, T, G, N), 1.0 / math.sqrt(N))
    if w.decay == "uniform_dt":
        dtv = torch.rand((B, T, H), generator=g, dtype=torch.float64) * (0.2 - 0.001) + 0.001
        a = (-dtv).to(torch.float32)
        if w.a_per_state:
            a = a.unsqueeze(-1).expand(B, T, H, N).contiguous()
    else:
        u = torch.randn((B, T, H), generator=g, dtype=torch.float64) + w.u_mean
        dtv = _softplus64(u)
        if w.a_per_state:
            A_log = torch.rand((H, N), generator=g, dtype=torch.float64) * math.log(16.0)
            a = (-(dtv.unsqueeze(-1) * torch.exp(A_log))).to(torch.float32)
        else:
            A_log = torch.rand((H,), generator=g, dtype=torch.float64) * math.log(16.0)
            a = (-(dtv * torch.exp(A_log))).to(torch.float32)
    Dv = torch.randn((H,), generator=g, dtype=torch.float64)
    D = Dv.to(torch.float32) if w.with_D else torch.zeros(H, dtype=torch.float32)
    return {"x": x, "a": a.contiguous(), "Bm": Bm, "Cm": Cm, "D": D}


def small_case(B=1, T=96, H=2, P=16, N=16, G=1, chunk=32, dtype="f32", a_per_state=False,
               seed=123, decay="softplus", u_mean=-2.0, with_D=True) -> Workload:
    """A free-form small workload with the same value recipe (tests)."""
    return Workload(f"case_B{B}_T{T}_H{H}_P{P}_N{N}_G{G}_Q{chunk}", B=B, T=T, H=H, P=P, N=N, G=G,
                    chunk=chunk, dtype=dtype, a_per_state=a_per_state, seed=seed, decay=decay,
                    u_mean=u_mean, with_D=with_D)
