"""The committed DRAM-traffic records that bench.py puts in its roofline line.

Each record in profiles/traffic.json holds the read and written bytes of one
ncu capture of a kernel, with a hash of the kernel's source at capture time.
bench.py reports the figure only while the source is unchanged; these tests
check that every committed record belongs to the current source, adds up,
names a committed summary, and that an edited source turns the figure off.
"""
import hashlib
import json
import os
import shutil

import pytest

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
TRAFFIC = os.path.join(ROOT, "profiles", "traffic.json")


def _records():
    with open(TRAFFIC) as f:
        rec = json.load(f)
    return [(k, w, r) for k, per in rec.items() for w, r in per.items()]


@pytest.mark.parametrize("kernel,workload,rec", _records(), ids=lambda v: v if isinstance(v, str) else "")
def test_traffic_record_is_current(kernel, workload, rec):
    src = os.path.join(ROOT, rec["source"])
    assert os.path.exists(src), rec["source"]
    with open(src, "rb") as f:
        h = hashlib.sha256(f.read()).hexdigest()[:16]
    assert h == rec["source_sha256_16"], f"{kernel}/{workload}: the capture predates the current {rec['source']}"
    assert rec["read"] + rec["write"] == rec["bytes_per_launch"]
    assert rec["bytes_per_launch"] > 0
    assert os.path.exists(os.path.join(ROOT, rec["capture"])), rec["capture"]
    assert bench.traffic_record(kernel, workload) == rec["bytes_per_launch"]


def test_traffic_record_turns_off_after_a_source_edit(tmp_path, monkeypatch):
    kernel, workload, rec = _records()[0]
    os.makedirs(tmp_path / "profiles")
    shutil.copy(TRAFFIC, tmp_path / "profiles" / "traffic.json")
    dst = tmp_path / rec["source"]
    os.makedirs(dst.parent)
    shutil.copy(os.path.join(ROOT, rec["source"]), dst)
    monkeypatch.setattr(bench, "ROOT", str(tmp_path))
    assert bench.traffic_record(kernel, workload) == rec["bytes_per_launch"]
    with open(dst, "a") as f:
        f.write("\n// edited\n")
    assert bench.traffic_record(kernel, workload) is None
    assert bench.traffic_record(kernel, "no_such_workload") is None
    assert bench.traffic_record("no_such_kernel", workload) is None
