"""Host-side logic of bench.py, on the CPU: the clock-sample summary (median
under load, throttle reasons), traffic figures tied to the kernels' source
hashes, the peak table, and the reference arm's JSON line (the oracle timed on
a bounded sample; only rank 0 prints)."""
import json
import os
import subprocess
import sys

import bench

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _sampler_with(tmp_path, lines):
    s = bench.ClockSampler(0)
    s.path = str(tmp_path / "clocks.csv")
    with open(s.path, "w") as f:
        f.write("\n".join(lines) + "\n")
    s.proc = object()                       # stands for a running nvidia-smi
    return s


def test_clock_summary_median_under_load_and_reasons(tmp_path):
    lines = [
        "0, 1965, 1965, 120.0, 0x0, Not Active, Not Active, Not Active, Not Active",   # idle, ignored
        "0, 1800, 1965, 900.0, 0x4, Not Active, Not Active, Not Active, Active",
        "0, 1850, 1965, 950.0, 0x0, Not Active, Not Active, Not Active, Not Active",
        "0, 1700, 1965, 980.0, 0x4, Not Active, Not Active, Not Active, Active",
        "garbage line",
    ]
    out = _sampler_with(tmp_path, lines).summary()
    assert out["sm_mhz"] == 1800.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"]
    assert out["samples"] == 4 and out["samples_under_load"] == 3


def test_clock_summary_reports_thermal_and_hardware_slowdown(tmp_path):
    lines = ["0, 1400, 1965, 700.0, 0x48, Active, Not Active, Active, Not Active"]
    out = _sampler_with(tmp_path, lines).summary()
    assert out["reasons"] == ["hw_slowdown", "sw_thermal_slowdown"]


def test_clock_summary_without_nvidia_smi():
    s = bench.ClockSampler(0)
    assert s.summary()["reasons"] == ["nvidia-smi unavailable"]


def test_traffic_only_for_current_kernel_sources(monkeypatch):
    d = json.load(open(os.path.join(ROOT, "profiles", "dram_traffic.json")))
    for kernel in bench.KERNEL_SOURCES:
        assert kernel in d
        if d[kernel]["source_hash"] == bench.kernel_source_hash(kernel):
            assert bench.ncu_traffic(kernel) == d[kernel]["bytes_per_launch"]
    monkeypatch.setattr(bench, "kernel_source_hash", lambda kernel: "0" * 16)
    for kernel in bench.KERNEL_SOURCES:
        assert bench.ncu_traffic(kernel) is None


def test_peaks_come_from_the_measured_table():
    p = bench.load_peaks()
    if os.path.exists(os.path.join(ROOT, "MEASURED_PEAKS.json")):
        m = json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))
        assert p["source"] == "measured" and p["hbm_gbs"] == m["hbm_gbs"] and p["bf16"] == m["bf16_tflops"]
    else:
        assert p["source"] == "fallback" and p["hbm_gbs"] == 6650.0


def _run_reference(env_extra):
    env = dict(os.environ, OMP_NUM_THREADS="4", **env_extra)
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                           "--steps", "1", "--warmup", "3", "--cpu-seconds", "1"],
                          capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)


def test_reference_arm_prints_one_contract_line():
    r = _run_reference({})
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [x for x in r.stdout.splitlines() if x.startswith("{")]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
                "scaling", "vs_baseline", "dtype", "data", "config", "cpu_baseline", "e2e"):
        assert key in d, key
    assert d["impl"] == "reference" and d["metric"] == bench.METRIC and d["unit"] == "TFLOP/s"
    assert d["value"] > 0 and d["steps"] == 1 and d["warmup"] == 3 and d["higher_is_better"] is True
    assert d["config"]["workload"] and d["vs_baseline"] is None
    # the same workload description as the native arm's line
    from sliding_window_gqa_prefill_b200 import workloads as wl
    assert d["config"] == bench.bench_config(wl.HEADLINE_PREFILL, 1)
    cb = d["cpu_baseline"]
    assert cb["kind"] == "oracle" and cb["value"] == d["value"] and cb["cores"] == 4 and cb["sample"]
    assert d["e2e"] == {"value": d["value"], "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}


def test_reference_arm_other_ranks_do_no_work():
    r = _run_reference({"RANK": "1", "WORLD_SIZE": "2"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_log_rows_one_per_measured_part(tmp_path):
    """--log appends the result line, then one JSON row per part (decode,
    chunked, rooflines, e2e, CPU baseline, each extra and sweep point), each
    carrying the workload config; a second run appends."""
    res = {"metric": "m", "value": 1.0, "config": {"workload": "w", "seeds": {"prefill": 1005}},
           "clocks": {"sm_mhz": 1900.0}, "decode": {"tokens_per_s": 3.0},
           "chunked": {"tflops": 2.0}, "roofline": {"frac": 0.9}, "e2e": {"value": 0.5},
           "cpu_baseline": {"value": 0.02, "check_of_timed_output": {"max_abs": 0.01}},
           "extras": {"a": {"tflops": 4.0}}, "sweep": {"N4096_W1024": {"tflops": 5.0}, "ratio": 2.1}}
    path = tmp_path / "log.jsonl"
    bench.write_log(str(path), res)
    rows = [json.loads(line) for line in path.read_text().splitlines()]
    assert rows[0] == res
    parts = [r["part"] for r in rows[1:]]
    assert parts == ["decode", "chunked", "roofline", "e2e", "cpu_baseline", "extras.a", "sweep.N4096_W1024",
                     "sweep.ratio"]
    assert all(r["config"] == res["config"] and r["impl"] == "native" for r in rows[1:])
    assert rows[-1]["value"] == 2.1 and rows[2]["tflops"] == 2.0
    bench.write_log(str(path), res)
    assert len(path.read_text().splitlines()) == 2 * len(rows)


def test_decode_launch_count_follows_the_split_policy():
    """bench.py counts one decode kernel per call for windows of one or four
    splits (merged on chip) and two otherwise; the split count is read back
    from the workspace size."""
    import sliding_window_gqa_prefill_b200 as swa
    swa.build()
    assert bench.decode_splits(swa, 64, 32, 8, 128, 4096) == 4
    assert bench.decode_splits(swa, 2, 32, 8, 128, 4096) == 16
    assert bench.decode_splits(swa, 1, 32, 8, 128, 100) == 1
    assert [bench.decode_kernels_per_call(n) for n in (1, 2, 4, 8, 16)] == [1, 2, 1, 2, 2]
