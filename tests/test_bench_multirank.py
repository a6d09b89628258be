"""Multi-rank logic of bench.py on CPU: world size 2 over gloo.

Under torchrun every rank times its own batch and the slowest rank sets the
step time; these tests run that host logic (seeding, max over ranks, the
whole-job rate, and the reference arm's rank-0-only rule) as two gloo
processes on 127.0.0.1, with no GPU.
"""
import io
import json
import os
import socket
import sys
from contextlib import redirect_stdout
from types import SimpleNamespace

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


def _rank_main(rank, world, port, out_dir):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank),
                      WORLD_SIZE=str(world))
    import datetime

    import bench
    from ssd_chunked_forward_b200.workloads import WORKLOADS, generate

    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=60))
    res = {}
    # each rank its own batch
    w = WORKLOADS["mamba2_130m"].scaled(B=1, T=256, H=2)
    inp = generate(w, seed=bench.rank_seed(w, rank))
    sums = [torch.zeros(1, dtype=torch.float64) for _ in range(world)]
    dist.all_gather(sums, inp["x"].double().sum().reshape(1))
    res["x_sums"] = [float(t) for t in sums]
    # the slowest rank's time, on every rank
    ms = 1.0 + 0.5 * rank
    res["max_ms"] = bench.max_over_ranks(ms, dist, "cpu")
    res["rate"] = bench.whole_job_rate(w.tokens, world, res["max_ms"])
    res["tokens"] = w.tokens
    # the reference arm: rank 0 alone times the oracle and prints one line
    args = SimpleNamespace(workload="tiny_f32", steps=1, warmup=0)
    buf = io.StringIO()
    with redirect_stdout(buf):
        code = bench.run_reference(args, rank, world)
    res["ref_code"] = code
    res["ref_out"] = buf.getvalue()
    dist.barrier()
    dist.destroy_process_group()
    with open(os.path.join(out_dir, f"rank{rank}.json"), "w") as f:
        json.dump(res, f)


@pytest.mark.timeout(300)
def test_two_rank_bench_logic(tmp_path):
    world = 2
    mp.spawn(_rank_main, args=(world, _free_port(), str(tmp_path)), nprocs=world, join=True)
    r = [json.load(open(tmp_path / f"rank{i}.json")) for i in range(world)]
    # every rank saw both ranks' batches, and they differ
    assert r[0]["x_sums"] == r[1]["x_sums"]
    assert r[0]["x_sums"][0] != r[0]["x_sums"][1]
    # max over ranks reaches every rank
    assert r[0]["max_ms"] == r[1]["max_ms"] == 1.5
    # whole-job rate: all ranks' tokens over the slowest step
    assert r[0]["rate"] == pytest.approx(world * r[0]["tokens"] / 1.5e-3)
    # reference arm: rank 0 prints one JSON line; rank 1 exits 0 without output
    assert r[0]["ref_code"] == 0 and r[1]["ref_code"] == 0
    assert r[1]["ref_out"] == ""
    lines = [l for l in r[0]["ref_out"].splitlines() if l.strip()]
    assert len(lines) == 1
    line = json.loads(lines[0])
    assert line["impl"] == "reference" and line["n_gpus"] == world
    assert line["cpu_baseline"]["kind"] == "oracle" and line["value"] > 0


def test_single_process_helpers():
    import bench
    assert bench.max_over_ranks(3.25) == 3.25
    assert bench.whole_job_rate(1000, 4, 2.0) == pytest.approx(2.0e6)


def test_reference_arm_json_contract():
    """`bench.py --impl reference` (the oracle on host cores) prints one JSON
    line with the contract's keys, its own cpu_baseline and an e2e object
    with no host-device traffic."""
    import subprocess
    out = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                          "--workload", "tiny_f32", "--steps", "2", "--warmup", "3"],
                         capture_output=True, text=True, timeout=240, cwd=ROOT,
                         env={**os.environ, "WORLD_SIZE": "1", "RANK": "0"})
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e", "gpu_launches"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 2 and d["warmup"] == 3
    assert d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "tiny_f32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["cpu_baseline"]["cores"] >= 1 and d["cpu_baseline"]["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": d["unit"], "h2d_bytes_per_step": 0,
                        "d2h_bytes_per_step": 0}
