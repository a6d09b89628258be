"""The autograd wrapper on the GPU with the library's kernels: a loss on y
and on the final state back-propagates to the same gradients that
ssd_backward gives directly (the wrapper adds no arithmetic)."""
import pytest
import torch

from ssd_chunked_forward_b200 import ssd
from ssd_chunked_forward_b200.autograd import ssd_autograd
from ssd_chunked_forward_b200.workloads import generate, small_case

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _cuda():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    ssd.load()


@pytest.mark.parametrize("w", [
    small_case(B=2, T=512, H=4, P=64, N=128, G=1, chunk=256, dtype="bf16", seed=121),
    small_case(B=1, T=200, H=2, P=16, N=24, G=2, chunk=64, dtype="f32", a_per_state=True, seed=122),
], ids=["scalar_bf16", "per_state_f32"])
def test_autograd_matches_backward(w):
    dev = {k: v.cuda() for k, v in generate(w).items()}
    g = torch.Generator().manual_seed(w.seed + 5)
    wy = torch.randn(dev["x"].shape, generator=g).to(dev["x"].dtype).cuda()
    wf = torch.randn((w.B, w.H, w.N, w.P), generator=g).cuda()
    h0 = torch.randn((w.B, w.H, w.N, w.P), generator=g).cuda()
    leaves = {k: dev[k].clone().requires_grad_() for k in ("x", "a", "Bm", "Cm", "D")}
    h0l = h0.clone().requires_grad_()
    y, fin = ssd_autograd(leaves["x"], leaves["a"], leaves["Bm"], leaves["Cm"], leaves["D"], w.chunk, h0l)
    loss = (y.float() * wy.float()).sum() + (fin * wf).sum()
    loss.backward()
    ref = ssd.backward(dev["x"], dev["a"], dev["Bm"], dev["Cm"], dev["D"], wy, w.chunk, dfinal=wf,
                       initial_state=h0)
    torch.cuda.synchronize()
    for k, name in (("x", "dx"), ("a", "da"), ("Bm", "dBm"), ("Cm", "dCm"), ("D", "dD")):
        assert torch.equal(leaves[k].grad, ref[name]), k
    assert torch.equal(h0l.grad, ref["dinit"])
