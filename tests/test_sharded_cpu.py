"""Sequence-sharded forward on CPU: two gloo ranks each hold half of the
sequence; the fp64 oracle stands in for the library's per-segment kernels, so
what is tested here is the orchestration and the collective (the library's
own kernels for the same steps are tested on the GPU)."""
import json
import os
import socket
import sys

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _free_port() -> int:
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _problem(per_state):
    rng = np.random.default_rng(101 + per_state)
    B, T, H, P, G, N = 2, 24, 2, 3, 1, 4
    x = rng.standard_normal((B, T, H, P))
    a = -rng.uniform(0, 0.6, size=(B, T, H, N) if per_state else (B, T, H))
    Bm = rng.standard_normal((B, T, G, N)) / 2
    Cm = rng.standard_normal((B, T, G, N)) / 2
    D = rng.standard_normal(H)
    h0 = rng.standard_normal((B, H, N, P))
    return x, a, Bm, Cm, D, h0


def _oracle_ops():
    from oracle import ssd_oracle as O
    from ssd_chunked_forward_b200.sharded import SegmentOps

    def forward(x, a, Bm, Cm, D, chunk, init):
        prob = O.Problem(x.numpy(), a.numpy(), Bm.numpy(), Cm.numpy(), D.numpy())
        B, T, H, P = x.shape
        N = Bm.shape[3]
        r = O.recurrence(prob, initial=None if init is None else init.numpy())
        y = r["y"].reshape(B, H, T, P).transpose(0, 2, 1, 3)
        return torch.from_numpy(np.ascontiguousarray(y)), torch.from_numpy(r["final"].reshape(B, H, N, P))

    def segment_state(x, a, Bm, chunk):
        # the segment's final state from zero (y not needed) and its total decay
        B, T, H, P = x.shape
        N = Bm.shape[3]
        Cz = np.zeros(Bm.shape)
        r = O.recurrence(O.Problem(x.numpy(), a.numpy(), Bm.numpy(), Cz, None), want_y=False)
        return torch.from_numpy(r["final"].reshape(B, H, N, P)), a.sum(dim=1)

    def state_combine(finals, totals, h0):
        S = finals.shape[0]
        h = torch.zeros_like(finals[0]) if h0 is None else h0.clone()
        out = [h]
        for s in range(S):
            e = torch.exp(totals[s])
            e = e[..., None, None] if totals.dim() == 3 else e[..., None]
            h = e * h + finals[s]
            out.append(h)
        return torch.stack(out)

    def backward(x, a, Bm, Cm, D, dy, chunk, dfinal, init):
        prob = O.Problem(x.numpy(), a.numpy(), Bm.numpy(), Cm.numpy(), D.numpy())
        r = O.backward(prob, dy.numpy(), dfinal=None if dfinal is None else dfinal.numpy(),
                       initial=None if init is None else init.numpy())
        return {k: torch.from_numpy(np.ascontiguousarray(r[k]))
                for k in ("dx", "da", "dBm", "dCm", "dD", "dinit")}

    return SegmentOps(forward=forward, segment_state=segment_state, state_combine=state_combine,
                      backward=backward)


def _rank_main(rank, world, port, out_dir, per_state, with_init):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    from ssd_chunked_forward_b200.sharded import sequence_sharded_forward

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    x, a, Bm, Cm, D, h0 = (torch.from_numpy(v) for v in _problem(per_state))
    T = x.shape[1]
    sl = slice(rank * T // world, (rank + 1) * T // world)
    seg = lambda t: t[:, sl].contiguous()
    y, fin = sequence_sharded_forward(seg(x), seg(a), seg(Bm), seg(Cm), D, 0, ops=_oracle_ops(),
                                      initial_state=h0 if with_init else None)
    dist.barrier()
    dist.destroy_process_group()
    np.save(os.path.join(out_dir, f"y{rank}.npy"), y.numpy())
    np.save(os.path.join(out_dir, f"f{rank}.npy"), fin.numpy())


@pytest.mark.timeout(300)
@pytest.mark.parametrize("per_state,with_init", [(False, False), (True, True)])
def test_two_rank_sequence_sharding(tmp_path, per_state, with_init):
    from oracle import ssd_oracle as O
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path), per_state, with_init), nprocs=world,
             join=True)
    x, a, Bm, Cm, D, h0 = _problem(per_state)
    B, T, H, P = x.shape
    N = Bm.shape[3]
    full = O.recurrence(O.Problem(x, a, Bm, Cm, D), initial=h0 if with_init else None)
    y_full = full["y"].reshape(B, H, T, P).transpose(0, 2, 1, 3)
    y = np.concatenate([np.load(tmp_path / f"y{r}.npy") for r in range(world)], axis=1)
    assert np.max(np.abs(y - y_full)) <= 1e-12 * np.max(np.abs(y_full))
    for r in range(world):  # every rank holds the whole sequence's final state
        f = np.load(tmp_path / f"f{r}.npy")
        assert np.max(np.abs(f - full["final"].reshape(B, H, N, P))) <= 1e-12 * np.max(np.abs(f))


def _bwd_rank_main(rank, world, port, out_dir, per_state, with_init, with_dfinal):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    import datetime
    from ssd_chunked_forward_b200.sharded import sequence_sharded_backward

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    x, a, Bm, Cm, D, h0 = (torch.from_numpy(v) for v in _problem(per_state))
    dy, dfin = (torch.from_numpy(v) for v in _bwd_extras(per_state))
    T = x.shape[1]
    sl = slice(rank * T // world, (rank + 1) * T // world)
    seg = lambda t: t[:, sl].contiguous()
    g = sequence_sharded_backward(seg(x), seg(a), seg(Bm), seg(Cm), D, seg(dy), 0, ops=_oracle_ops(),
                                  initial_state=h0 if with_init else None,
                                  dfinal=dfin if with_dfinal else None)
    dist.barrier()
    dist.destroy_process_group()
    for k, v in g.items():
        np.save(os.path.join(out_dir, f"{k}{rank}.npy"), v.numpy())


def _bwd_extras(per_state):
    rng = np.random.default_rng(211 + per_state)
    B, T, H, P, N = 2, 24, 2, 3, 4
    return rng.standard_normal((B, T, H, P)), rng.standard_normal((B, H, N, P))


@pytest.mark.timeout(300)
@pytest.mark.parametrize("world", [2, 3])
@pytest.mark.parametrize("per_state,with_init,with_dfinal",
                         [(False, False, False), (False, True, True), (True, True, True)])
def test_sequence_sharded_backward(tmp_path, world, per_state, with_init, with_dfinal):
    """The sharded backward (entering states forwards by one all-gather,
    entering-state adjoints backwards by another, dD summed by an all-reduce)
    equals the backward of the whole
    sequence: each rank's slice of dx, da, dB, dC, and dD and the initial
    state's gradient on every rank."""
    from oracle import ssd_oracle as O
    mp.spawn(_bwd_rank_main, args=(world, _free_port(), str(tmp_path), per_state, with_init, with_dfinal),
             nprocs=world, join=True)
    x, a, Bm, Cm, D, h0 = _problem(per_state)
    dy, dfin = _bwd_extras(per_state)
    ref = O.backward(O.Problem(x, a, Bm, Cm, D), dy, dfinal=dfin if with_dfinal else None,
                     initial=h0 if with_init else None)
    for k in ("dx", "da", "dBm", "dCm"):
        got = np.concatenate([np.load(tmp_path / f"{k}{r}.npy") for r in range(world)], axis=1)
        assert np.max(np.abs(got - ref[k])) <= 1e-12 * np.max(np.abs(ref[k])), k
    for r in range(world):
        for k in ("dD", "dinit"):
            got = np.load(tmp_path / f"{k}{r}.npy")
            assert np.max(np.abs(got - ref[k])) <= 1e-12 * max(1.0, np.max(np.abs(ref[k]))), (k, r)

