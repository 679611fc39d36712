"""The prefill's work decomposition, checked on the CPU: tests/c/unit_plan_check.cu
compiles the planner the kernel's warps call (prefill_plan.cuh) for the host
and enumerates every unit of 40 launches (one-shot, query-block pairs for odd
groups, chunk mode through the rolling buffer, sinks, packed batches in head
pairs and in query-block pairs, the
last-wave and half-wave single-head splits, one head per unit for short
odd-group launches, pairs of query blocks split into
their blocks in a short last wave, windows whose edge falls on a
tile's first key), then 160 seeded random launches whose SM count is drawn too
(3 to 148 SMs, so every mode triggers at small sizes).  The persistent blocks
must take every unit exactly once,
each query row of each head must be computed exactly once,
by a unit of its KV head, and the unit's key tiles must hold exactly the row's
keys (window, sinks, buffer slots), tiles marked clean needing no mask."""
import os
import shutil
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "tests", "c", "unit_plan_check.cu")


@pytest.mark.skipif(shutil.which("nvcc") is None, reason="nvcc not on PATH")
def test_every_row_once_and_exactly_its_keys(tmp_path):
    exe = str(tmp_path / "unit_plan_check")
    subprocess.run(["nvcc", "-std=c++17", "-O2", "-gencode", "arch=compute_100a,code=sm_100a", "-o", exe, SRC],
                   check=True, capture_output=True, text=True)
    r = subprocess.run([exe], capture_output=True, text=True, timeout=300)
    assert r.returncode == 0, r.stdout + r.stderr
    words = r.stdout.split()
    assert words[0] == "ok" and int(words[1]) == 40 and int(words[2]) > 1400000, r.stdout
    assert words[3:5] == ["(and", "157"], r.stdout          # seeded random launches (3 empty ones skipped)
