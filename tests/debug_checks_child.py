"""Child process of tests/test_gpu_debug_checks.py: loads the index-checked
build (SSD_DEBUG_CHECKS=1 set by the parent), runs every entry point on tiny
in-bounds cases against the oracle, and prints one JSON line with the errors
and the check record; then turns on the switch that fails every check and
runs two kernels without device-side waits, printing the record again."""
from __future__ import annotations

import json
import os
import sys

import numpy as np
import torch

sys.path.insert(0, os.path.dirname(os.path.dirname(os.path.abspath(__file__))))

from oracle import ssd_oracle as O  # noqa: E402
from ssd_chunked_forward_b200 import ssd  # noqa: E402
from ssd_chunked_forward_b200.workloads import generate, small_case  # noqa: E402
from tests.gpu_helpers import rel_err, to_dev  # noqa: E402


def chains(y, fin):
    """[B,T,H,P] and [B,H,N,P] device outputs in the oracle's chain-major
    layout ([B*H,T,P], [B*H,N,P]), float64."""
    B, T, H, P = y.shape
    yc = y.float().permute(0, 2, 1, 3).reshape(B * H, T, P).cpu().numpy().astype(np.float64)
    fc = fin.reshape(B * H, fin.shape[2], fin.shape[3]).cpu().numpy().astype(np.float64)
    return yc, fc


def prob(inp):
    return O.Problem(*(inp[k].to(torch.float64).numpy() if inp[k] is not None else None
                       for k in ("x", "a", "Bm", "Cm", "D")))


def main():
    assert os.environ.get("SSD_DEBUG_CHECKS") == "1"
    ssd.load()
    out = {"debug_build": ssd.debug_build(), "errors": {}}
    ssd.debug_record()  # start from a clear record
    cases = {
        "fused_bf16": (small_case(B=2, T=384, H=4, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=301),
                       [ssd.PATH_FUSED, ssd.PATH_MODULAR]),
        "simt_f32": (small_case(B=1, T=150, H=3, P=24, N=20, G=1, chunk=64, dtype="f32", seed=302),
                     [ssd.PATH_AUTO]),
        "diag_bf16": (small_case(B=1, T=256, H=2, P=64, N=64, G=1, chunk=128, dtype="bf16", a_per_state=True,
                                 seed=303), [ssd.PATH_AUTO]),
        "diag_f32": (small_case(B=1, T=100, H=2, P=16, N=12, G=1, chunk=32, dtype="f32", a_per_state=True,
                                seed=304), [ssd.PATH_AUTO]),
    }
    for name, (w, paths) in cases.items():
        inp = generate(w)
        dev = to_dev(inp)
        ref = O.recurrence(prob(inp))
        for path in paths:
            y, fin = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=path)
            torch.cuda.synchronize()
            yc, fc = chains(y, fin)
            out["errors"][f"{name}_p{path}_y"] = rel_err(yc, ref["y"])
            out["errors"][f"{name}_p{path}_fin"] = rel_err(fc, ref["final"])
        # the backward on the same inputs
        g = torch.Generator().manual_seed(w.seed + 9)
        dy = torch.randn((w.B, w.T, w.H, w.P), generator=g).to(inp["x"].dtype)
        got = ssd.backward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], dy.cuda(), w.chunk)
        torch.cuda.synchronize()
        bref = O.backward(prob(inp), dy.to(torch.float64).numpy())
        for k in ("dx", "da", "dBm", "dCm", "dD"):
            out["errors"][f"{name}_bwd_{k}"] = rel_err(got[k].float().cpu().numpy().astype(np.float64), bref[k])
    # the long-sequence split path (segment states, their combination, the fused kernel over pieces)
    w = small_case(B=1, T=8192, H=2, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=305)
    inp = generate(w)
    dev = to_dev(inp)
    y, fin = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk, path=ssd.PATH_SPLIT)
    torch.cuda.synchronize()
    ref = O.recurrence(prob(inp))
    yc, fc = chains(y, fin)
    out["errors"]["split_y"] = rel_err(yc, ref["y"])
    out["errors"]["split_fin"] = rel_err(fc, ref["final"])
    # one decode step and the discretisation
    w = small_case(B=2, T=1, H=4, P=64, N=128, G=2, chunk=1, dtype="bf16", seed=306)
    inp = generate(w)
    dev = to_dev(inp)
    h0 = torch.randn((w.B, w.H, w.N, w.P), generator=torch.Generator().manual_seed(7))
    state = h0.cuda()
    y = ssd.decode_step(dev["x"][:, 0].contiguous(), dev["a"][:, 0].contiguous(), dev["Bm"][:, 0].contiguous(),
                        dev["Cm"][:, 0].contiguous(), dev["D"], state)
    torch.cuda.synchronize()
    ref = O.recurrence(prob(inp), initial=h0.to(torch.float64).numpy())
    out["errors"]["decode_y"] = rel_err(y.float().cpu().numpy().astype(np.float64),
                                        ref["y"].reshape(w.B, w.H, 1, w.P)[:, :, 0])
    raw = torch.randn((2, 33, 4), generator=torch.Generator().manual_seed(8)).cuda()
    A_log = torch.rand(4, generator=torch.Generator().manual_seed(9)).cuda()
    xx = torch.randn((2, 33, 4, 64), generator=torch.Generator().manual_seed(10)).to(torch.bfloat16).cuda()
    a_out, x_out = ssd.discretize(raw, None, A_log, xx)
    torch.cuda.synchronize()
    out["record"] = ssd.debug_record()
    # every check fails: the accesses are skipped and the first one recorded
    ssd.debug_fail_all(True)
    ssd.decode_step(dev["x"][:, 0].contiguous(), dev["a"][:, 0].contiguous(), dev["Bm"][:, 0].contiguous(),
                    dev["Cm"][:, 0].contiguous(), dev["D"], state)
    ssd.discretize(raw, None, A_log, xx, a_out=a_out, x_out=x_out)
    torch.cuda.synchronize()
    out["record_failing"] = ssd.debug_record()
    ssd.debug_fail_all(False)
    print(json.dumps(out))


if __name__ == "__main__":
    main()
