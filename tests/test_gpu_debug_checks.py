"""The index-checked debug build (libssd_debug.so, SSD_DEBUG_CHECKS=1) on the
GPU: every entry point on tiny in-bounds cases matches the oracle with no
failed check recorded, and the test switch that fails every check skips the
accesses and records where (no index is ever out of bounds, nothing traps).
The build runs in a child process because a process loads one library."""
from __future__ import annotations

import json
import os
import subprocess
import sys

import pytest
import torch

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


@pytest.fixture(scope="module")
def child_result():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    from ssd_chunked_forward_b200.build import build
    build(debug=True)
    env = dict(os.environ, SSD_DEBUG_CHECKS="1")
    res = subprocess.run([sys.executable, os.path.join(ROOT, "tests", "debug_checks_child.py")],
                         capture_output=True, text=True, env=env, cwd=ROOT, timeout=600)
    assert res.returncode == 0, res.stderr[-3000:]
    return json.loads(res.stdout.strip().splitlines()[-1])


def test_debug_build_loaded(child_result):
    assert child_result["debug_build"] is True


def test_debug_build_matches_oracle_without_failed_checks(child_result):
    errs = child_result["errors"]
    for k, e in errs.items():
        tol = 1e-4 if "f32" in k else 2e-2
        assert e <= tol, (k, e)
    assert child_result["record"] == [0, 0, 0, 0]


def test_failing_every_check_records_the_site(child_result):
    failed, line, block, thread = child_result["record_failing"]
    assert failed > 0 and line > 0 and block >= 0 and thread >= 0
