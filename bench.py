"""Throughput of the chunked SSD forward on B200 (tokens/s and roofline fraction).

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload NAME]
                    [--path auto|modular|simt|fused] [--impl ours|reference]

One step = one ssd_forward over one batch of the workload's synthetic inputs
(already resident in HBM); the L2 is flushed (a 256 MB write) before every
timed step.  Each step is timed with CUDA events on the launching stream; the
K steps are bracketed by a barrier and a device synchronise; the slowest rank
sets the time.  Under torchrun every rank runs its own independent batch of
the same workload (weak scaling, no collective on the data path).

Rank 0 prints ONE JSON line.  ``--impl reference`` times the fp64 CPU oracle
(the reference arm: a bounded sample of the same workload per step).
"""
from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import sys
import threading
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

from ssd_chunked_forward_b200 import ssd  # noqa: E402
from ssd_chunked_forward_b200.workloads import WORKLOADS, generate  # noqa: E402

DEFAULT_WORKLOAD = "mamba2_2p7b"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
PATHS = {"auto": ssd.PATH_AUTO, "modular": ssd.PATH_MODULAR, "simt": ssd.PATH_SIMT,
         "fused": ssd.PATH_FUSED, "split": ssd.PATH_SPLIT}


# ----------------------------------------------------------------- model ----

def algorithmic(w):
    """Algorithmic FLOPs and HBM bytes of one forward.

    Per token-head: FLOPs = 2NP (chunk state) + 2NP (incoming-state term)
    + Q*P (causal half of the masked product with X) + Q*N*G/H (causal half
    of C B^T, shared by the heads of a group).  Bytes: x and y once, B and C
    once per group, a, D and the final state."""
    B, T, H, P, N, G, Q = w.B, w.T, w.H, w.P, w.N, w.G, w.chunk
    el = 2 if w.dtype == "bf16" else 4
    th = B * T * H
    flops = th * (4 * N * P + Q * P + Q * N * G / H)
    a_bytes = B * T * H * (N if w.a_per_state else 1) * 4
    byts = (2 * B * T * H * P * el + 2 * B * T * G * N * el + a_bytes + H * 4 + B * H * N * P * 4)
    return flops, byts


def kernel_bytes(w, name):
    """Algorithmic bytes of one launch of a step kernel: each tensor it must
    read or write, once."""
    B, T, H, P, N, G, Q = w.B, w.T, w.H, w.P, w.N, w.G, w.chunk
    nc = -(-T // Q)
    el = 2 if w.dtype == "bf16" else 4
    na = N if w.a_per_state else 1
    x = B * T * H * P * el
    bc = B * T * G * N * el
    a = B * T * H * na * 4
    cum = B * H * nc * Q * na * 4
    st = B * H * nc * N * P * 4
    fin = B * H * N * P * 4
    if name == "chunk_cumsum":
        return a + cum
    if name == "chunk_state":
        return x + bc + cum + st
    if name == "state_pass":
        return st + st + B * H * nc * na * 4 + fin
    if name in ("chunk_scan", "diag_scan"):
        return x + 2 * bc + cum + st + x + H * 4
    if name == "fused":
        return algorithmic(w)[1]
    if name == "segment_state":
        return x + bc // 2 + a + B * H * N * P * 4  # x, Bm, a once; a state per piece (small)
    if name == "state_combine":
        return 0
    raise KeyError(name)


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            pk = json.load(f)
        return pk, "measured"
    return dict(FALLBACK_PEAKS), "fallback"


def traffic_record(kernel, workload):
    """dram bytes per launch from a committed ncu capture, valid only while the
    kernel's source is unchanged (hash recorded with the capture)."""
    path = os.path.join(ROOT, "profiles", "traffic.json")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f)
    r = rec.get(kernel, {}).get(workload)
    if not r:
        return None
    src = os.path.join(ROOT, r["source"])
    if not os.path.exists(src):
        return None
    h = hashlib.sha256(open(src, "rb").read()).hexdigest()[:16]
    return r["bytes_per_launch"] if h == r["source_sha256_16"] else None


# ---------------------------------------------------------------- clocks ----

class ClockSampler:
    """Samples SM clock and throttle reasons through NVML every ~2 ms."""

    REASONS = {
        0x1: "gpu_idle", 0x2: "applications_clocks_setting", 0x4: "sw_power_cap",
        0x8: "hw_slowdown", 0x10: "sync_boost", 0x20: "sw_thermal_slowdown",
        0x40: "hw_thermal_slowdown", 0x80: "hw_power_brake_slowdown",
        0x100: "display_clock_setting",
    }

    def __init__(self, device_index):
        self.samples, self.reasons = [], 0
        self.ok = False
        self.max_mhz = None
        try:
            import pynvml
            pynvml.nvmlInit()
            uuid = "GPU-" + str(torch.cuda.get_device_properties(device_index).uuid)
            self.h = pynvml.nvmlDeviceGetHandleByUUID(uuid)
            self.nv = pynvml
            self.max_mhz = pynvml.nvmlDeviceGetMaxClockInfo(self.h, pynvml.NVML_CLOCK_SM)
            self.ok = True
        except Exception as e:  # no NVML: report that, never guess
            self.err = repr(e)
        self._stop = threading.Event()

    def _sample(self):
        try:
            self.samples.append(self.nv.nvmlDeviceGetClockInfo(self.h, self.nv.NVML_CLOCK_SM))
            self.reasons |= self.nv.nvmlDeviceGetCurrentClocksEventReasons(self.h)
        except Exception:
            pass

    def _run(self):
        # every ~2 ms, so that even a timed region of a few milliseconds gets
        # several samples; one more when the region ends
        while not self._stop.is_set():
            self._sample()
            time.sleep(0.002)
        self._sample()

    def __enter__(self):
        if self.ok:
            self.t = threading.Thread(target=self._run, daemon=True)
            self.t.start()
        return self

    def __exit__(self, *exc):
        if self.ok:
            self._stop.set()
            self.t.join()

    def summary(self):
        if not self.ok:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "note": "NVML unavailable"}
        names = [n for bit, n in self.REASONS.items() if self.reasons & bit and n != "gpu_idle"]
        return {"sm_mhz": statistics.median(self.samples) if self.samples else None,
                "sm_max_mhz": self.max_mhz, "reasons": names, "samples": len(self.samples)}


# ------------------------------------------------------------ oracle leg ----

def chain_problem(inp, b, h, t_end):
    """float64 copy of chain (b, h)'s first t_end tokens: the exact values the
    device receives (bf16/fp32 widen exactly to float64)."""
    from oracle import ssd_oracle as O
    H, G = inp["x"].shape[2], inp["Bm"].shape[2]
    g = h // (H // G)
    f = lambda t: t.to(torch.float64).numpy()
    return O.Problem(f(inp["x"][b:b + 1, :t_end, h:h + 1].contiguous()),
                     f(inp["a"][b:b + 1, :t_end, h:h + 1].contiguous()),
                     f(inp["Bm"][b:b + 1, :t_end, g:g + 1].contiguous()),
                     f(inp["Cm"][b:b + 1, :t_end, g:g + 1].contiguous()),
                     f(inp["D"][h:h + 1].contiguous()))


def oracle_sample(w, inp, budget_s, nthreads):
    """Time the fp64 oracle recurrence on a bounded sample of the workload:
    whole-width chains (b, h) in b-major order over their first t_end tokens,
    sized from a short calibration run to take about budget_s seconds."""
    from oracle import ssd_oracle as O

    chains = [(b, h) for b in range(w.B) for h in range(w.H)]
    t_cal = min(w.T, 256)
    p = chain_problem(inp, 0, 0, t_cal)
    t0 = time.perf_counter()
    O.recurrence(p, nthreads=1)
    per_token_chain = (time.perf_counter() - t0) / t_cal
    par = max(1, nthreads)
    n_chains = min(len(chains), max(par, 1))
    t_end = int(min(w.T, max(16, budget_s * par / (per_token_chain * n_chains))))
    if t_end == w.T:  # room for more chains
        n_chains = int(min(len(chains), max(n_chains, budget_s * par / (per_token_chain * w.T))))
    sel = chains[:n_chains]
    # one multi-chain problem: stack the chains as heads of one batch row
    import numpy as np
    probs = [chain_problem(inp, b, h, t_end) for (b, h) in sel]
    x = np.concatenate([q.x for q in probs], axis=2)
    a = np.concatenate([q.a for q in probs], axis=2)
    Bm = np.concatenate([q.Bm for q in probs], axis=2)
    Cm = np.concatenate([q.Cm for q in probs], axis=2)
    D = np.concatenate([q.D for q in probs])
    prob = O.Problem(x, a, Bm, Cm, D)
    t0 = time.perf_counter()
    O.recurrence(prob, nthreads=par)
    dt = time.perf_counter() - t0
    tokens = n_chains * t_end / w.H  # a token carries all H heads
    return {"value": tokens / dt, "unit": "tokens/s", "cores": min(par, n_chains), "kind": "oracle",
            "sample": f"{n_chains} of {w.B * w.H} (batch, head) chains x first {t_end} of {w.T} "
                      f"tokens, fp64 recurrence, {dt:.2f} s"}


def run_reference(args, rank, world):
    if rank != 0:
        return 0
    w = WORKLOADS[args.workload]
    inp = generate(w)
    nthreads = os.cpu_count() or 1
    per_step = max(0.2, min(2.0, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        oracle_sample(w, inp, per_step, nthreads)
    vals = [oracle_sample(w, inp, per_step, nthreads) for _ in range(args.steps)]
    v = statistics.median(r["value"] for r in vals)
    line = {
        "impl": "reference", "metric": "SSD forward tokens/s (B*T per second)", "value": v,
        "unit": "tokens/s", "n_gpus": world, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1000.0 * w.tokens / v, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "P": w.P, "N": w.N, "G": w.G,
                   "chunk": w.chunk, "parallelism": "none (CPU oracle)"},
        "cpu_baseline": {"kind": "oracle", "cores": vals[0]["cores"], "sample": vals[0]["sample"],
                         "value": v, "unit": "tokens/s"},
        "e2e": {"value": v, "unit": "tokens/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
        "gpu_launches": 0,
    }
    print(json.dumps(line))
    return 0


# ------------------------------------------------------------ multi-rank ----

def rank_seed(w, rank: int) -> int:
    """Seed of rank `rank`'s batch: every rank runs its own independent batch
    of the same workload (weak scaling)."""
    return w.seed + 1000 * rank


def max_over_ranks(value: float, dist=None, device="cpu") -> float:
    """The slowest rank's figure; every rank takes part (identity without a
    process group)."""
    if dist is None:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def step_stats(step_ms):
    """Median, 10th and 90th percentile and mean of the per-step device times
    (ms); the median is the step time the metric uses."""
    v = sorted(step_ms)
    def pct(q):
        if len(v) == 1:
            return v[0]
        pos = q * (len(v) - 1)
        lo = int(pos)
        hi = min(lo + 1, len(v) - 1)
        return v[lo] + (v[hi] - v[lo]) * (pos - lo)
    return {"median": statistics.median(v), "p10": pct(0.10), "p90": pct(0.90),
            "mean": statistics.mean(v)}


def whole_job_rate(tokens_per_rank: int, world: int, ms: float) -> float:
    """Tokens per second of the whole job: every rank's tokens over the
    slowest rank's time per step."""
    return tokens_per_rank * world / (ms / 1e3)


# ---------------------------------------------------------------- GPU leg ----

def per_state_tc(w):
    """The per-state shapes whose modular path runs on tensor cores (three
    launches: block states with the decay sums inside, the pass, the outputs)."""
    return w.a_per_state and w.dtype == "bf16" and w.N == 64 and w.P == 64


def step_kernels(w, path_used):
    if path_used == "fused":
        return ["fused"]
    if path_used == "split":
        return ["segment_state", "state_combine", "fused"]
    if path_used == "modular" and per_state_tc(w):
        return ["chunk_state", "state_pass", "diag_scan"]
    return ["chunk_cumsum", "chunk_state", "state_pass", "diag_scan" if w.a_per_state else "chunk_scan"]


def time_split_path(w, dev, flush, reps, S):
    """Device times (ms) of the split path's three launches, called one by one
    through the library on the [B*S][T/S] view of the inputs: the pieces'
    states from zero (ssd_segment_state), their combine (ssd_state_combine),
    and the forward over all pieces from their entering states
    (ssd_forward_init; the fused kernel)."""
    B, T = w.B, w.T
    L = T // S
    view = {k: dev[k].view((B * S, L) + tuple(dev[k].shape[2:])) for k in ("x", "a", "Bm", "Cm")}
    st = torch.cuda.current_stream()
    times = {"segment_state": [], "state_combine": [], "fused": []}
    for r in range(reps):
        flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(4)]
        ev[0].record(st)
        fin, tot = ssd.segment_state(view["x"], view["a"], view["Bm"], w.chunk)
        ev[1].record(st)
        finals = fin.view(B, S, w.H, w.N, w.P).transpose(0, 1).contiguous()
        totals = tot.view(B, S, w.H).transpose(0, 1).contiguous()
        h_in = ssd.state_combine(finals, totals)
        ev[2].record(st)
        init = h_in[:S].transpose(0, 1).reshape(B * S, w.H, w.N, w.P).contiguous()
        ssd.forward(view["x"], view["a"], view["Bm"], view["Cm"], dev["D"], w.chunk, initial_state=init,
                    path=ssd.PATH_FUSED)
        ev[3].record(st)
        torch.cuda.synchronize()
        if r == 0:
            continue
        for i, n in enumerate(times):
            times[n].append(ev[i].elapsed_time(ev[i + 1]))
    return {n: statistics.median(v) for n, v in times.items()}


def step_workload(w, impl):
    """The shape the modular path's steps run on: where the tensor-core kernels
    serve the workload and the chunk is a multiple of 128, the library runs
    the steps on 128-token blocks (the same result up to rounding)."""
    if (impl != ssd.IMPL_SIMT and w.dtype == "bf16" and not w.a_per_state and w.N == 128
            and w.P == 64 and w.chunk % 128 == 0 and w.chunk > 128):
        return w.scaled(chunk=128)
    return w


def time_steps_split(w, dev, flush, reps, impl):
    """Per-kernel device times (ms) of the modular path, by calling the step
    entry points one by one with events between them on one stream, on the
    shape the library's modular path uses (step_workload)."""
    w = step_workload(w, impl)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    st = torch.cuda.current_stream()
    nc = -(-w.T // w.chunk)
    cum_t = torch.empty(w.B * w.H * nc * w.chunk * (w.N if w.a_per_state else 1),
                        dtype=torch.float32, device=dev["x"].device)
    states = torch.empty((w.B, w.H, nc, w.N, w.P), dtype=torch.float32, device=dev["x"].device)
    fin = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device=dev["x"].device)
    y = torch.empty_like(dev["x"])
    # the four step entry points; for the per-state tensor-core shapes the
    # forward itself folds the prefix sums into the other kernels, and its
    # block-state and output kernels are these steps' kernels reading a instead
    # of the prefix sums (the same bytes)
    names = ["chunk_cumsum", "chunk_state", "state_pass", "diag_scan" if w.a_per_state else "chunk_scan"]
    times = {n: [] for n in names}
    for r in range(reps):
        flush()
        ev = [torch.cuda.Event(enable_timing=True) for _ in range(5)]
        ev[0].record(st)
        ssd.chunk_cumsum(shape, dev["a"], cum_t)
        ev[1].record(st)
        ssd.chunk_state(shape, dev["x"], dev["Bm"], cum_t, states, impl=impl)
        ev[2].record(st)
        ssd.state_pass(shape, cum_t, states, fin)
        ev[3].record(st)
        ssd.chunk_scan(shape, dev["x"], dev["Bm"], dev["Cm"], cum_t, states, dev["D"], y, impl=impl)
        ev[4].record(st)
        torch.cuda.synchronize()
        if r == 0:
            continue  # warm-up
        for i, n in enumerate(names):
            times[n].append(ev[i].elapsed_time(ev[i + 1]))
    del cum_t, states, fin, y
    out = {n: statistics.median(v) for n, v in times.items()}
    if impl != ssd.IMPL_SIMT and per_state_tc(w):
        out.pop("chunk_cumsum")  # not launched by the forward
    return out


def run_decode(args, device):
    """The decode step (ssd_decode_step) on the workload's batch and heads: one
    token per (batch, head) chain, the fp32 state read and written in place.
    Algorithmic bytes: the state twice plus x, y, a, B and C of one token."""
    w = WORKLOADS[args.workload]
    g = torch.Generator().manual_seed(w.seed + 500)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    x = torch.randn((w.B, w.H, w.P), generator=g).to(dt).to(device)
    a = (-torch.rand((w.B, w.H) + ((w.N,) if w.a_per_state else ()), generator=g)).to(device)
    Bm = (torch.randn((w.B, w.G, w.N), generator=g) / w.N ** 0.5).to(dt).to(device)
    Cm = (torch.randn((w.B, w.G, w.N), generator=g) / w.N ** 0.5).to(dt).to(device)
    D = torch.randn((w.H,), generator=g).to(device)
    state = torch.randn((w.B, w.H, w.N, w.P), generator=g).to(device)
    y = torch.empty_like(x)
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        scratch.fill_(1)
        ssd.decode_step(x, a, Bm, Cm, D, state, y=y)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        scratch.fill_(1)
        e0.record(st)
        ssd.decode_step(x, a, Bm, Cm, D, state, y=y)
        e1.record(st)
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    el = 2 if w.dtype == "bf16" else 4
    byts = (2 * w.B * w.H * w.N * w.P * 4 + 2 * w.B * w.H * w.P * el
            + w.B * w.H * (w.N if w.a_per_state else 1) * 4 + 2 * w.B * w.G * w.N * el + w.H * 4)
    peaks, src = load_peaks()
    achieved = byts / (ms / 1e3) / 1e9
    print(json.dumps({
        "metric": "SSD decode step tokens/s (one token per batch row)", "value": w.B / (ms / 1e3),
        "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
        "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name + "_decode", "B": w.B, "H": w.H, "P": w.P, "N": w.N, "G": w.G,
                   "a_per_state": w.a_per_state, "l2": "flushed (256 MB write) before every step"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": byts,
                     "kernel": "ssd_decode_step", "peak_source": f"{src} (hbm_gbs)"},
        "gpu_launches": args.steps}))
    return 0


# fp32 FMA issue rate of the CUDA cores: 148 SMs x 128 fp32 lanes x 2 flops
# x 1.965 GHz (the part's maximum SM clock)
FP32_ALU_TFLOPS = 148 * 128 * 2 * 1.965e9 / 1e12


def backward_flops(w):
    """Algorithmic flops of the chunked backward: per chain and chunk, four
    quadratic forms (pair scores over K plus pair-weighted sums over Mc, with
    K + Mc = N + P, on the Q (Q + 1) / 2 causal pairs, plus the Q x K x Mc
    boundary term) and three chunk-state contractions (the recomputed states,
    the adjoint readout states; Q x N x P each, the boundary terms counted
    above)."""
    Q, N, P = w.chunk, w.N, w.P
    nc = -(-w.T // Q)
    per_chunk = 4 * (Q * (Q + 1) * (N + P) + 2 * Q * N * P) + 2 * (2 * Q * N * P)
    return w.B * w.H * nc * per_chunk


def run_backward(args, device):
    """ssd_backward on the workload: dy (and a loss on the final state) in, the
    six gradients out; L2 flushed before every step.  Its roofline is the bf16
    tensor rate where the quadratic forms run on tensor cores, else the fp32
    FMA rate of the CUDA cores."""
    w = WORKLOADS[args.workload]
    if args.B or args.T:
        w = w.scaled(B=args.B or w.B, T=args.T or w.T, name=w.name + f"_B{args.B or w.B}_T{args.T or w.T}")
    dev = {k: (v.to(device) if v is not None else None) for k, v in generate(w).items()}
    g = torch.Generator().manual_seed(w.seed + 700)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    dy = torch.randn((w.B, w.T, w.H, w.P), generator=g).to(dt).to(device)
    dfin = torch.randn((w.B, w.H, w.N, w.P), generator=g).to(device)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    ws = torch.empty(ssd.backward_workspace_size(shape), dtype=torch.uint8, device=device)
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream()
    call = lambda: ssd.backward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], dy, w.chunk,
                                dfinal=dfin, workspace=ws)
    for _ in range(args.warmup):
        scratch.fill_(1)
        call()
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        scratch.fill_(1)
        e0.record(st)
        call()
        e1.record(st)
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    el = 2 if w.dtype == "bf16" else 4
    tok = w.B * w.T
    byts = (2 * 2 * tok * w.H * w.P * el + 2 * tok * w.H * 4 + 2 * 2 * tok * w.G * w.N * el
            + 2 * w.B * w.H * w.N * w.P * 4 + 2 * w.H * 4)
    flops = backward_flops(w)
    achieved = flops / (ms / 1e3) / 1e12
    peaks, src = load_peaks()
    # bf16 heads with N = 128, P = 64 and 128/256-token chunks run the forms and
    # the chunk states on tensor cores: the roofline is then the bf16 tensor rate
    tc = (w.dtype == "bf16" and not w.a_per_state and w.N == 128 and w.P == 64
          and w.chunk in (128, 256))
    if tc:
        roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"], "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16_tflops"], "algorithmic_flops_per_step": flops,
                "kernel": "ssd_backward (13 launches; the four forms and both chunk-state "
                          "contractions on tensor cores)",
                "peak_source": f"{src} (bf16_tflops)"}
    else:
        roof = {"bound": "alu", "achieved": achieved, "peak": FP32_ALU_TFLOPS, "unit": "TFLOP/s",
                "frac": achieved / FP32_ALU_TFLOPS, "algorithmic_flops_per_step": flops,
                "kernel": "ssd_backward (13 launches)",
                "peak_source": "fp32 FMA rate from unit counts and the maximum SM clock"}
    print(json.dumps({
        "metric": "SSD backward tokens/s", "value": tok / (ms / 1e3), "unit": "tokens/s",
        "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup, "dtype": w.dtype,
        "data": "synthetic",
        "config": {"workload": w.name + "_backward", "B": w.B, "T": w.T, "H": w.H, "P": w.P,
                   "N": w.N, "G": w.G, "chunk": w.chunk, "loss": "sum(dy * y) + <dfinal, final>",
                   "l2": "flushed (256 MB write) before every step"},
        "roofline": roof,
        "hbm_view": {"algorithmic_bytes_per_step": byts, "achieved_gbs": byts / (ms / 1e3) / 1e9,
                     "frac_of_measured_hbm": byts / (ms / 1e3) / 1e9 / peaks["hbm_gbs"]},
        "gpu_launches": 13 * args.steps}))
    return 0


def run_discretize(args, device):
    """ssd_discretize on the workload's shape: dt_raw and x in, a and x_out out,
    each once (algorithmic bytes); L2 flushed before every step."""
    w = WORKLOADS[args.workload]
    g = torch.Generator().manual_seed(w.seed + 600)
    dt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    raw = torch.randn((w.B, w.T, w.H), generator=g).to(device)
    bias = torch.randn((w.H,), generator=g).to(device)
    A_log = torch.rand((w.H, w.N) if w.a_per_state else (w.H,), generator=g).to(device)
    x = torch.randn((w.B, w.T, w.H, w.P), generator=g).to(dt).to(device)
    a_out = torch.empty((w.B, w.T, w.H) + ((w.N,) if w.a_per_state else ()), dtype=torch.float32,
                        device=device)
    x_out = torch.empty_like(x)
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=device)
    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        scratch.fill_(1)
        ssd.discretize(raw, bias, A_log, x, a_out=a_out, x_out=x_out)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    torch.cuda.synchronize()
    for e0, e1 in ev:
        scratch.fill_(1)
        e0.record(st)
        ssd.discretize(raw, bias, A_log, x, a_out=a_out, x_out=x_out)
        e1.record(st)
    torch.cuda.synchronize()
    ms = statistics.median(e0.elapsed_time(e1) for e0, e1 in ev)
    byts = (raw.numel() * 4 + 2 * x.numel() * x.element_size() + a_out.numel() * 4
            + bias.numel() * 4 + A_log.numel() * 4)
    peaks, src = load_peaks()
    achieved = byts / (ms / 1e3) / 1e9
    # the forward fed by the discretisation: two launches (x_out and a written
    # and read back) against the one fused pass that never writes them
    front = {}
    if (not w.a_per_state and w.dtype == "bf16" and w.N == 128 and w.P == 64
            and w.chunk % 128 == 0):
        Bm = (torch.randn((w.B, w.T, w.G, w.N), generator=g) / w.N ** 0.5).to(dt).to(device)
        Cm = (torch.randn((w.B, w.T, w.G, w.N), generator=g) / w.N ** 0.5).to(dt).to(device)
        D = torch.randn((w.H,), generator=g).to(device)
        shape = ssd.shape_of(x, a_out, Bm, w.chunk)
        ws = ssd.alloc_workspace(shape, device)
        y = torch.empty_like(x)
        fin = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device=device)

        def two():
            ssd.discretize(raw, bias, A_log, x, a_out=a_out, x_out=x_out)
            ssd.forward(x_out, a_out, Bm, Cm, D, w.chunk, y=y, final_state=fin, workspace=ws,
                        path=ssd.PATH_FUSED)

        def one():
            ssd.forward_discretized(x, raw, bias, A_log, Bm, Cm, D, w.chunk, y=y, final_state=fin,
                                    workspace=ws)

        for name, fn in (("discretize_then_forward_ms", two), ("forward_discretized_ms", one)):
            for _ in range(args.warmup):
                scratch.fill_(1)
                fn()
            evs = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True))
                   for _ in range(args.steps)]
            torch.cuda.synchronize()
            for e0, e1 in evs:
                scratch.fill_(1)
                e0.record(st)
                fn()
                e1.record(st)
            torch.cuda.synchronize()
            front[name] = statistics.median(e0.elapsed_time(e1) for e0, e1 in evs)
        del Bm, Cm, ws, y, fin
    print(json.dumps({
        "metric": "SSD discretisation tokens/s (B*T per second)", "value": w.tokens / (ms / 1e3),
        "unit": "tokens/s", "ms_per_step": ms, "steps": args.steps, "warmup": args.warmup,
        "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name + "_discretize", "B": w.B, "T": w.T, "H": w.H, "P": w.P,
                   "a_per_state": w.a_per_state, "l2": "flushed (256 MB write) before every step"},
        "roofline": {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": achieved / peaks["hbm_gbs"], "algorithmic_bytes_per_launch": byts,
                     "kernel": "ssd_discretize", "peak_source": f"{src} (hbm_gbs)"},
        "front_end": front or None,
        "gpu_launches": args.steps}))
    return 0


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=10)
    ap.add_argument("--workload", default=DEFAULT_WORKLOAD, choices=list(WORKLOADS))
    ap.add_argument("--path", default="auto", choices=list(PATHS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--B", type=int, default=None, help="override the batch (profiling small cases)")
    ap.add_argument("--T", type=int, default=None, help="override the sequence length")
    ap.add_argument("--discretize", action="store_true",
                    help="time the discretisation front end (ssd_discretize) on the workload's "
                         "inputs instead of the forward; prints its own JSON line")
    ap.add_argument("--backward", action="store_true",
                    help="time the backward (ssd_backward, scalar decay) on the workload instead "
                         "of the forward; prints its own JSON line")
    ap.add_argument("--decode", action="store_true",
                    help="time the recurrent decode step (one token per chain) on the workload's "
                         "batch and heads instead of the forward; prints its own JSON line")
    args = ap.parse_args()

    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        return run_reference(args, rank, world)
    if args.warmup < 3:
        raise SystemExit("--warmup must be >= 3")

    torch.cuda.set_device(local)
    device = torch.device("cuda", local)
    if args.decode:
        return run_decode(args, device)
    if args.backward:
        return run_backward(args, device)
    if args.discretize:
        return run_discretize(args, device)
    dist = None
    if world > 1:
        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=300), device_id=device)

    w = WORKLOADS[args.workload]
    if args.B or args.T:
        w = w.scaled(B=args.B or w.B, T=args.T or w.T, name=w.name + f"_B{args.B or w.B}_T{args.T or w.T}")
    inp = generate(w, seed=rank_seed(w, rank))  # each rank: its own batch
    dev = {k: v.to(device) for k, v in inp.items()}
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    path = PATHS[args.path]
    if not ssd.path_supported(shape, path):
        raise SystemExit(f"path {args.path} does not serve workload {w.name}")
    path_used = args.path
    if path == ssd.PATH_AUTO:
        path_used = {ssd.PATH_FUSED: "fused", ssd.PATH_SPLIT: "split"}.get(ssd.auto_path(shape), "modular")
    ws = ssd.alloc_workspace(shape, device)
    y = torch.empty_like(dev["x"])
    fin = torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32, device=device)
    scratch = torch.empty(256 << 20, dtype=torch.uint8, device=device)

    def flush():
        scratch.fill_(1)

    def fwd():
        ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, y=y,
                    final_state=fin, workspace=ws, path=path)

    st = torch.cuda.current_stream()
    for _ in range(args.warmup):
        flush()
        fwd()
    torch.cuda.synchronize()
    code = ssd.device_status(ws)
    if code != ssd.SSD_OK:
        raise SystemExit(f"device status after warm-up: {ssd.status_string(code)}")

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    sampler = ClockSampler(local)
    if dist:
        dist.barrier()
    torch.cuda.synchronize()
    with sampler:
        for i in range(args.steps):
            flush()
            starts[i].record(st)
            fwd()
            ends[i].record(st)
        torch.cuda.synchronize()
    if dist:
        dist.barrier()
    code = ssd.device_status(ws)
    if code != ssd.SSD_OK:
        raise SystemExit(f"device status after timing: {ssd.status_string(code)}")
    step_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    stats = step_stats(step_ms)
    ms = max_over_ranks(stats["median"], dist, device)
    value = whole_job_rate(w.tokens, world, ms)

    # ---- dominant kernel: per-kernel split with events --------------------
    peaks, peak_src = load_peaks()
    flops, byts = algorithmic(w)
    t_roof = max(flops / (peaks["bf16_tflops"] * 1e12), byts / (peaks["hbm_gbs"] * 1e9))
    if path_used == "fused":
        split = {"fused": ms}
    elif path_used == "split":
        split = time_split_path(w, dev, flush, 11, ssd.split_pieces(shape))
    else:
        impl = ssd.IMPL_SIMT if path_used == "simt" else ssd.IMPL_AUTO
        split = time_steps_split(w, dev, flush, 11, impl)
    dom = max(split, key=split.get)
    dom_ms = split[dom]
    dom_bytes = kernel_bytes(w if path_used in ("fused", "split") else
                             step_workload(w, ssd.IMPL_SIMT if path_used == "simt" else ssd.IMPL_AUTO), dom)
    achieved = dom_bytes / (dom_ms / 1e3) / 1e9
    kernel_name = {"fused": "ssd_fused_kernel"}.get(dom, "ssd_" + dom)
    roofline = {"bound": "hbm", "achieved": achieved, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                "frac": achieved / peaks["hbm_gbs"], "traffic": traffic_record(kernel_name, w.name),
                "kernel": kernel_name, "algorithmic_bytes_per_launch": dom_bytes,
                "peak_source": f"{peak_src} (hbm_gbs)"}

    # ---- end to end through the host-buffer entry point -------------------
    e2e = None
    if not args.no_e2e:
        # Two streams, each with its own device buffer and host outputs, take
        # alternate steps, so one step's copies overlap the other's kernels (a
        # serving loop's double buffering); every step still copies all of its
        # inputs in and its y and final state out.
        pin = {k: v.pin_memory() for k, v in inp.items()}
        streams = [torch.cuda.Stream(device=device) for _ in range(2)]
        y_hs = [torch.empty_like(inp["x"]).pin_memory() for _ in range(2)]
        f_hs = [torch.empty((w.B, w.H, w.N, w.P), dtype=torch.float32).pin_memory() for _ in range(2)]
        bufs = [torch.empty(ssd.forward_host_bytes(shape), dtype=torch.uint8, device=device)
                for _ in range(2)]
        e2e_steps = max(4, min(args.steps, 20))

        def fwd_host(i):
            s_ = i % 2
            ssd.forward_host(shape, pin["x"], pin["a"], pin["Bm"], pin["Cm"], pin["D"], y_hs[s_],
                             f_hs[s_], bufs[s_], stream=streams[s_])

        for i in range(4):
            fwd_host(i)
        torch.cuda.synchronize()
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        if dist:
            dist.barrier()
        torch.cuda.synchronize()
        e0.record(st)
        for s_ in streams:
            s_.wait_event(e0)
        for i in range(e2e_steps):
            fwd_host(i)
        for s_ in streams:
            st.wait_stream(s_)
        e1.record(st)
        torch.cuda.synchronize()
        e_ms = max_over_ranks(e0.elapsed_time(e1) / e2e_steps, dist, device)
        h2d = sum(v.numel() * v.element_size() for v in inp.values())
        d2h = y_hs[0].numel() * y_hs[0].element_size() + f_hs[0].numel() * 4
        e2e = {"value": whole_job_rate(w.tokens, world, e_ms), "unit": "tokens/s", "h2d_bytes_per_step": h2d,
               "d2h_bytes_per_step": d2h, "ms_per_step": e_ms, "steps": e2e_steps,
               "api": "ssd_forward_host (pinned host buffers)",
               "streams": 2, "overlap": "alternate steps on two streams; a step's copies overlap the other's kernels"}
        del bufs

    # ---- CPU oracle baseline (rank 0, N = 1 only) -------------------------
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        cpu = oracle_sample(w, inp, 15.0, os.cpu_count() or 1)

    if rank == 0:
        launches = len(step_kernels(w, path_used)) * args.steps
        line = {
            "metric": "SSD forward tokens/s (B*T per second)", "value": value, "unit": "tokens/s",
            "n_gpus": world, "steps": args.steps, "warmup": args.warmup, "ms_per_step": ms,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": w.dtype,
            "data": "synthetic",
            "step_ms": {"median": ms, "p10": stats["p10"], "p90": stats["p90"], "mean": stats["mean"],
                        "note": "this rank's per-step device times; ms_per_step is the median "
                                "(the slowest rank's under torchrun)"},
            "config": {"workload": w.name, "B": w.B, "T": w.T, "H": w.H, "P": w.P, "N": w.N,
                       "G": w.G, "chunk": w.chunk, "a_per_state": w.a_per_state,
                       "global_batch": w.B * world, "seq_len": w.T,
                       "parallelism": f"independent batch per GPU x{world}", "path": path_used,
                       "l2": "flushed (256 MB write) before every timed step"},
            "roofline": roofline,
            "roofline_forward": {"t_roof_us": t_roof * 1e6, "t_us": ms * 1e3,
                                 "frac": t_roof / (ms / 1e3), "flops_alg": flops,
                                 "bytes_alg": byts, "bound": "hbm" if byts / peaks["hbm_gbs"] / 1e9 >=
                                 flops / peaks["bf16_tflops"] / 1e12 else "tensor",
                                 "peaks": {"hbm_gbs": peaks["hbm_gbs"],
                                           "bf16_tflops": peaks["bf16_tflops"], "source": peak_src}},
            "kernel_split_ms": split,
            "clocks": sampler.summary(),
            "e2e": e2e,
            "gpu_launches": launches,
            "cpu_baseline": cpu,
        }
        print(json.dumps(line))
    if dist:
        dist.barrier()
        dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
