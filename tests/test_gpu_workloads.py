"""Full-size parity on the five measured workloads, in the launch
configuration bench.py times (SSD_PATH_AUTO).  The oracle runs the fp64
recurrence over whole (batch, head) chains chosen to cover first, middle and
last heads and batches (every chain of the tiny fp32 workload); the metric is
||y - y_ref||_inf / ||y_ref||_inf over those chains, and the same on the final
state."""
from __future__ import annotations

import pytest
import torch

from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.workloads import WORKLOADS, generate
from tests.gpu_helpers import parity_on_chains, run_forward, to_dev, tol_for

pytestmark = pytest.mark.gpu

SAMPLES = {
    "tiny_f32": None,  # all chains
    "mamba2_130m": [(0, 0), (3, 11), (7, 23)],
    "mamba2_2p7b": [(0, 0), (1, 40), (3, 79)],
    "long_seq": [(0, 0), (0, 17), (0, 31)],
    "diag_ssm": [(0, 0), (2, 7), (3, 15)],
}
# tokens of the chain the oracle replays for y (the final state always uses a
# whole chain); long_seq replays 2^16 tokens = 256 chunks for y
T_END = {"long_seq": 65536}


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load()


@pytest.mark.parametrize("name", list(WORKLOADS))
def test_workload_parity(name):
    w = WORKLOADS[name]
    inp = generate(w)
    dev = to_dev(inp)
    y, fin = run_forward(w, dev)
    del dev
    chains = SAMPLES[name] or [(b, h) for b in range(w.B) for h in range(w.H)]
    tol = tol_for(w)
    t_end = T_END.get(name)
    ey, ef = parity_on_chains(inp, y, fin, chains, t_end=t_end)
    assert ey <= tol, f"{name}: y rel err {ey:.3e} > {tol}"
    if ef is None:  # y was compared on a prefix; compare one whole chain's final state
        _, ef = parity_on_chains(inp, y, fin, chains[-1:], t_end=None)
    assert ef <= tol, f"{name}: final-state rel err {ef:.3e} > {tol}"
    print(f"{name}: y rel err {ey:.3e}, final rel err {ef:.3e} (tol {tol})")
