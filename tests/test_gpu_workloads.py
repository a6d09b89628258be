"""Full-size parity on the five measured workloads, in the launch
configuration bench.py times (SSD_PATH_AUTO).  The metric is
||y - y_ref||_inf / ||y_ref||_inf over the WHOLE output tensor (every batch
row, head, token and channel) and the same metric over the whole final
state, against the fp64 recurrence (O1) on the values the device received;
the oracle runs group by group and the comparison streams chain by chain."""
from __future__ import annotations

import pytest
import torch

from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.workloads import ORDER, WORKLOADS, generate
from tests.gpu_helpers import run_forward, to_dev, tol_for, whole_tensor_parity

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load()


@pytest.mark.parametrize("name", ORDER)
def test_workload_parity(name):
    w = WORKLOADS[name]
    inp = generate(w)
    dev = to_dev(inp)
    y, fin = run_forward(w, dev)
    y, fin = y.cpu(), fin.cpu()
    del dev
    torch.cuda.empty_cache()
    tol = tol_for(w)
    ey, ef, ymax = whole_tensor_parity(inp, y, fin)
    print(f"{name}: whole-tensor y rel err {ey:.3e} (max|y_ref| {ymax:.3g}), "
          f"final rel err {ef:.3e} (tol {tol})")
    assert ey <= tol, f"{name}: y rel err {ey:.3e} > {tol}"
    assert ef <= tol, f"{name}: final-state rel err {ef:.3e} > {tol}"
