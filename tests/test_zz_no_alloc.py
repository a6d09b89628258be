"""ssd_forward_noalloc: the fused forward for callers that cannot allocate
device memory at call time (its scratch is a fixed array inside the library).
It must give the result of the regular ssd_forward, on two calls in a row
(the array keeps the previous call's contents, so the second call checks that
what must start at zero is cleared).  Collected last on purpose."""
from __future__ import annotations

import ctypes

import numpy as np
import pytest
import torch

from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.workloads import generate, small_case

pytestmark = pytest.mark.gpu

TOL = 2e-2  # bf16 inputs, fp32 accumulation


def _rel(a, b):
    a = a.float().cpu().numpy().astype(np.float64)
    b = b.float().cpu().numpy().astype(np.float64)
    return float(np.max(np.abs(a - b)) / max(np.max(np.abs(b)), 1e-30))


@pytest.mark.parametrize("w", [
    small_case(B=2, T=1024, H=8, P=64, N=128, G=2, chunk=256, dtype="bf16", seed=41),
    small_case(B=1, T=2048, H=16, P=64, N=128, G=1, chunk=128, dtype="bf16", seed=42),
], ids=["B2_T1024_H8_G2_Q256", "B1_T2048_H16_Q128"])
def test_noalloc_matches_forward_twice(w):
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ssd.load()
    dev = {k: v.cuda() for k, v in generate(w).items()}
    y_ref, f_ref = ssd.forward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], w.chunk)
    shape = ssd.shape_of(dev["x"], dev["a"], dev["Bm"], w.chunk)
    for call in range(2):
        y = torch.full_like(dev["x"], float("nan"))
        fin = torch.full((w.B, w.H, w.N, w.P), float("nan"), dtype=torch.float32, device="cuda")
        code = lib.ssd_forward_noalloc(ctypes.byref(shape), dev["x"].data_ptr(), dev["a"].data_ptr(),
                                       dev["Bm"].data_ptr(), dev["Cm"].data_ptr(), dev["D"].data_ptr(),
                                       y.data_ptr(), fin.data_ptr(),
                                       torch.cuda.current_stream().cuda_stream)
        assert code == ssd.SSD_OK, ssd.status_string(code)
        torch.cuda.synchronize()
        assert _rel(y, y_ref) <= TOL, f"call {call}: y"
        assert _rel(fin, f_ref) <= TOL, f"call {call}: final state"


def test_noalloc_rejects_too_many_chains():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    lib = ssd.load()
    shape = ssd.make_shape(B=8, T=256, H=64, P=64, G=1, N=128, chunk=256, dtype="bf16")  # 512 chains
    ok = 1 << 20  # aligned fake address; rejected before any use
    code = lib.ssd_forward_noalloc(ctypes.byref(shape), ok, ok, ok, ok, None, ok, None, None)
    assert code == ssd.SSD_ERR_WORKSPACE
