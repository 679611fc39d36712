#!/usr/bin/env python
"""Benchmark of the sliding-window GQA attention path on B200.

One step = one pass of the whole path over synthetic Mistral-7B-shaped inputs:
  1. one-shot prefill, B=2, N=16384, W=4096, 32 query / 8 KV heads, D=128
     (1% of key rows scaled x8) -- the headline workload;
  2. chunked prefill of a 16384-token prompt in 4 chunks of 4096 through a
     4096-slot rolling buffer (attention + buffer write per chunk), B=1;
  3. batched decode: 128 steps of (append one token, attend) for B=64
     sequences at positions drawn from [1, 32768], replayed as one CUDA graph.
`value` is the useful (unmasked) prefill TFLOP/s of part 1; parts 2 and 3
are reported beside it.  Inputs (0.4 GB prefill, 1 GB decode cache) are larger
than the 126 MB L2, so no flush is needed between steps.

Multi-GPU: one process per GPU (torchrun); every rank runs the same
independent workload (the path has no exchange step: replicas, weak
scaling); times are the max over ranks.

`--impl reference` times the fp64 CPU oracle (the only reference this path
has) on a bounded row sample of the same workload.
"""
from __future__ import annotations

import argparse
import hashlib
import itertools
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "SWA prefill useful TFLOP/s @N=16K,W=4K; decode tokens/s @B=64 (frac. of roofline)"


def parse_args(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=10)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["native", "reference"], default="native")
    ap.add_argument("--no-cpu-baseline", action="store_true", help="skip the oracle timing leg")
    ap.add_argument("--cpu-seconds", type=float, default=12.0, help="target oracle sample time")
    ap.add_argument("--log", default=None,
                    help="also append the result, and one row per measured part, as JSON lines to this file")
    ap.add_argument("--ncu-case", choices=["prefill", "prefill_b2", "chunk", "decode", "decode_w8k", "mixed"], default=None,
                    help="run a reduced case of one kernel three times for an ncu capture (no timing)")
    return ap.parse_args(argv)


def load_peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        d = json.load(open(p))
        return dict(hbm_gbs=float(d["hbm_gbs"]), bf16=float(d["bf16_tflops"]),
                    bf16_sustained=float(d.get("bf16_tflops_sustained", d["bf16_tflops"])),
                    source="measured")
    return dict(hbm_gbs=6650.0, bf16=1590.0, bf16_sustained=1400.0, source="fallback")


# the sources each kernel is built from (its launch code is in swa_api.cu)
KERNEL_SOURCES = {
    "swa_prefill_kernel<128>": ("device_common.cuh", "prefill_plan.cuh", "prefill_kernel.cuh", "swa_api.cu"),
    "swa_decode_kernel<128,4>": ("device_common.cuh", "decode_kernel.cuh", "swa_api.cu"),
}


def kernel_source_hash(kernel: str) -> str:
    h = hashlib.sha256()
    for f in KERNEL_SOURCES[kernel]:
        h.update(open(os.path.join(ROOT, "sliding_window_gqa_prefill_b200", "csrc", f), "rb").read())
    return h.hexdigest()[:16]


def ncu_traffic(kernel: str):
    """DRAM bytes per launch from the committed ncu summary, if it was taken on
    the current sources of that kernel (else None)."""
    p = os.path.join(ROOT, "profiles", "dram_traffic.json")
    if not os.path.exists(p):
        return None
    d = json.load(open(p))
    e = d.get(kernel)
    if not e or e.get("source_hash") != kernel_source_hash(kernel):
        return None
    return e.get("bytes_per_launch")


# ---------------------------------------------------------------- clocks sampler

class ClockSampler:
    FIELDS = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, index: int):
        self.index = index
        self.proc = None
        self.path = os.path.join("/tmp", f"swa_clocks_{os.getpid()}.csv")

    def __enter__(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "200"],
                stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append(dict(sm=float(parts[1]), smax=float(parts[2]), power=float(parts[3]),
                                 hw=parts[5], hwt=parts[6], swt=parts[7], pcap=parts[8]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        smax = max(r["smax"] for r in rows)
        load = [r for r in rows if r["power"] > 250.0] or rows
        reasons = set()
        for r in load:
            for key, name in (("hw", "hw_slowdown"), ("hwt", "hw_thermal_slowdown"),
                              ("swt", "sw_thermal_slowdown"), ("pcap", "sw_power_cap")):
                if r[key].lower() == "active":
                    reasons.add(name)
        return {"sm_mhz": statistics.median(r["sm"] for r in load), "sm_max_mhz": smax,
                "reasons": sorted(reasons), "samples": len(rows), "samples_under_load": len(load)}


# ---------------------------------------------------------------- distributed helpers

def dist_setup(gpus: int):
    import torch
    import torch.distributed as dist
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        import datetime
        torch.cuda.set_device(local)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", local))
    else:
        torch.cuda.set_device(0)
    return rank, world, local


def max_over_ranks(x: float, world: int, device: str = "cuda") -> float:
    """Maximum of a per-rank scalar (a time) over all ranks."""
    if world == 1:
        return x
    import torch
    import torch.distributed as dist
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def weak_scaling_rate(units_per_rank: float, world: int, max_seconds: float) -> float:
    """Whole-job throughput: every rank processes the same units; the job
    takes as long as its slowest rank."""
    return units_per_rank * world / max_seconds


def decode_splits(swa, B: int, Hq: int, Hkv: int, D: int, W: int) -> int:
    """Splits per window of a swa_decode call, read back from its workspace
    size (rows = B * Hq * splits of D floats, 256-byte padded, then one (m, l)
    pair per row)."""
    n = swa.swa_decode_workspace_size(B, Hq, Hkv, D, W)
    for splits in range(1, 4097):
        rows = B * Hq * splits
        if (rows * D * 4 + 255) // 256 * 256 + rows * 8 == n:
            return splits
    raise RuntimeError("decode workspace size matches no split count")


def decode_kernels_per_call(splits: int) -> int:
    """Kernels one swa_decode call (no sinks) launches: the split-KV kernel,
    plus the split merge unless the window is one split or exactly four
    (merged on chip by the four blocks of a cluster)."""
    return 1 if splits in (1, 4) else 2


def barrier(world: int):
    if world > 1:
        import torch.distributed as dist
        dist.barrier()


def bench_config(hp, world: int) -> dict:
    """The workload description both arms print (native and reference)."""
    from sliding_window_gqa_prefill_b200 import workloads as wl
    return {
        "workload": hp.name,
        "B": hp.B, "N": hp.N, "W": hp.W, "Hq": hp.Hq, "Hkv": hp.Hkv, "D": hp.D,
        "seeds": {"prefill": hp.seed, "chunked": wl.CHUNKED_16K.seed, "decode": wl.DECODE_B64.seed},
        "parallelism": f"replicas{world}" if world > 1 else "single",
        "l2": "inputs larger than L2 (prefill q/k/v/out 640 MB, decode cache 1 GB); no flush",
        "step": "one-shot prefill + 4-chunk prefill (N=16384) + 128 decode steps (B=64, graph)",
    }


# nominal B200 figures (datasheet, dense): fractions against them are reported
# beside the ones against the measured peaks, which are the roofline
NOMINAL_HBM_GBS = 8000.0
NOMINAL_BF16_TFLOPS = 2250.0


# ---------------------------------------------------------------- CPU oracle sample

_ORACLE_CACHE = {}


def cpu_oracle_sample(target_s: float, gpu_out=None):
    """Time the fp64 oracle on a row sample of the headline prefill workload.

    Returns (TFLOP/s, seconds, rows, threads, check): with gpu_out (the GPU's
    output of the same seeded workload, [B, N, Hq, D]) check holds the error
    of the GPU's rows against the oracle's on the sampled rows, else None."""
    import numpy as np
    import oracle
    from sliding_window_gqa_prefill_b200 import workloads as wl
    w = wl.HEADLINE_PREFILL
    if "inputs" not in _ORACLE_CACHE:
        q, k, v = wl.prefill_inputs(w)
        _ORACLE_CACHE["inputs"] = tuple(t.float().numpy().astype(np.float64) for t in (q, k, v))
    qn, kn, vn = _ORACLE_CACHE["inputs"]
    rng = np.random.default_rng(0)
    # rows past the first window: each sees exactly W keys
    pool = rng.permutation(np.arange(w.W, w.N))
    threads = int(os.environ.get("OMP_NUM_THREADS", os.cpu_count() or 1))
    done, t_total, used = 0, 0.0, 0
    batch = 8
    err_max, err_sum, err_n = 0.0, 0.0, 0
    while t_total < target_s and used + batch <= pool.size:
        rows = pool[used:used + batch]
        t0 = time.perf_counter()
        ref = oracle.swa_prefill(qn, kn, vn, w.W, w.scale, rows=rows)
        dt = time.perf_counter() - t0
        if gpu_out is not None:            # outside the timed region
            got = gpu_out[:, rows.tolist()].float().cpu().numpy().astype(np.float64)
            err = np.abs(got - ref)
            err_max = max(err_max, float(err.max()))
            err_sum += float(err.sum())
            err_n += err.size
        t_total += dt
        used += batch
        done += batch
        remaining = target_s - t_total
        if dt > 0 and remaining > 0:
            batch = int(min(max(8, batch * min(4.0, remaining / dt)), pool.size - used))
            if batch <= 0:
                break
    flops = 4.0 * w.B * w.Hq * w.D * w.W * done
    check = None
    if gpu_out is not None and err_n:
        check = {"rows": done, "max_abs": err_max, "mean_abs": err_sum / err_n, "bar": [2e-2, 2e-3],
                 "within_bar": err_max <= 2e-2 and err_sum / err_n <= 2e-3}
    return flops / t_total / 1e12, t_total, done, threads, check


# ---------------------------------------------------------------- native GPU run

def run_native(args):
    import torch
    import sliding_window_gqa_prefill_b200 as swa
    from sliding_window_gqa_prefill_b200 import workloads as wl

    rank, world, local = dist_setup(args.gpus)
    swa.build()
    swa.lib()
    peaks = load_peaks()
    dev = torch.device("cuda", torch.cuda.current_device())
    stream = torch.cuda.current_stream()

    # ---- inputs, resident in HBM before timing
    hp = wl.HEADLINE_PREFILL
    q_cpu, k_cpu, v_cpu = wl.prefill_inputs(hp)
    q, k, v = q_cpu.to(dev), k_cpu.to(dev), v_cpu.to(dev)
    out = torch.empty_like(q)
    pf_flops = wl.useful_flops(hp.B, hp.N, hp.W, hp.Hq, hp.D)

    cw = wl.CHUNKED_16K
    cq, ck, cv = (t.to(dev) for t in wl.chunked_inputs(cw))
    c_chunks = [(cq[:, s:s + cw.C].contiguous(), ck[:, s:s + cw.C].contiguous(),
                 cv[:, s:s + cw.C].contiguous()) for s in range(0, cw.N, cw.C)]
    c_start = [torch.full((cw.B,), s, dtype=torch.int32, device=dev) for s in range(0, cw.N, cw.C)]
    c_kc = torch.zeros(cw.B, cw.W, cw.Hkv, cw.D, dtype=torch.bfloat16, device=dev)
    c_vc = torch.zeros_like(c_kc)
    c_outs = [torch.empty_like(a) for a, _, _ in c_chunks]
    c_flops = wl.useful_flops(cw.B, cw.N, cw.W, cw.Hq, cw.D)

    dw = wl.DECODE_B64
    dd = wl.decode_inputs(dw)
    d_kc, d_vc = dd["k_cache"].to(dev), dd["v_cache"].to(dev)
    d_q = dd["q"].to(dev)
    d_kn = dd["k_new"].to(dev).unsqueeze(2).contiguous()      # [steps, B, 1, Hkv, D]
    d_vn = dd["v_new"].to(dev).unsqueeze(2).contiguous()
    pos_table = (dd["pos0"].unsqueeze(0) + torch.arange(dw.steps, dtype=torch.int32).unsqueeze(1)).to(torch.int32)
    d_pos = pos_table.to(dev).contiguous()                     # [steps, B]
    d_out = torch.empty(dw.steps, dw.B, dw.Hq, dw.D, dtype=torch.bfloat16, device=dev)
    ws_bytes = swa.swa_decode_workspace_size(dw.B, dw.Hq, dw.Hkv, dw.D, dw.W)
    d_ws = torch.empty(ws_bytes, dtype=torch.uint8, device=dev)
    L = torch.clamp(pos_table.to(torch.int64) + 1, max=dw.W)   # keys read per (step, sequence)
    kv_bytes = int(L.sum().item()) * dw.Hkv * dw.D * 2 * 2     # K and V rows read, all steps
    other_bytes = dw.steps * dw.B * (2 * dw.Hq * dw.D * 2 + 2 * 2 * dw.Hkv * dw.D * 2)  # q, out, append r+w

    # events around every swa_decode call (split-KV kernel + split merge) are
    # captured into the graph, so each replay re-records them on the launch stream
    dec_ev = [(torch.cuda.Event(enable_timing=True, external=True),
               torch.cuda.Event(enable_timing=True, external=True))
              for _ in range(dw.steps)]

    def decode_all(with_events=False):
        for s in range(dw.steps):
            swa.swa_cache_append(d_kn[s], d_vn[s], d_kc, d_vc, d_pos[s])
            if with_events:
                dec_ev[s][0].record()
            swa.swa_decode(d_q[s], d_kc, d_vc, d_pos[s], dw.scale, out=d_out[s], workspace=d_ws)
            if with_events:
                dec_ev[s][1].record()

    # ---- capture the 128 decode steps in one graph
    decode_all()
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        decode_all(with_events=True)
    torch.cuda.synchronize()

    def step(ev=None):
        if ev:
            ev[0].record()
        swa.swa_prefill(q, k, v, hp.W, hp.scale, out=out)
        if ev:
            ev[1].record()
        for (a, b, c), st, o in zip(c_chunks, c_start, c_outs):
            swa.swa_prefill_chunk(a, b, c, c_kc, c_vc, st, cw.W, cw.scale, out=o)
        if ev:
            ev[2].record()
        graph.replay()
        if ev:
            ev[3].record()

    for _ in range(args.warmup):
        step()
    torch.cuda.synchronize()
    assert swa.swa_get_device_status() == swa.SWA_OK

    evs = [[torch.cuda.Event(enable_timing=True) for _ in range(4)] for _ in range(args.steps)]
    barrier(world)
    torch.cuda.synchronize()
    with ClockSampler(dev.index) as clk:
        t_start = torch.cuda.Event(enable_timing=True)
        t_end = torch.cuda.Event(enable_timing=True)
        t_start.record()
        for i in range(args.steps):
            step(evs[i])
        t_end.record()
        torch.cuda.synchronize()
    barrier(world)
    status = swa.swa_get_device_status()
    # decode launches of the last timed replay (128 calls)
    dec_call_ms = sum(a.elapsed_time(b) for a, b in dec_ev)
    pf_ms = [e[0].elapsed_time(e[1]) for e in evs]
    ch_ms = [e[1].elapsed_time(e[2]) for e in evs]
    de_ms = [e[2].elapsed_time(e[3]) for e in evs]
    total_ms = t_start.elapsed_time(t_end)

    pf_total = max_over_ranks(sum(pf_ms), world)
    ch_total = max_over_ranks(sum(ch_ms), world)
    de_total = max_over_ranks(sum(de_ms), world)
    step_total = max_over_ranks(total_ms, world)

    value = weak_scaling_rate(pf_flops * args.steps, world, pf_total * 1e-3) / 1e12
    pf_avg_ms = pf_total / args.steps
    achieved = pf_flops / (pf_avg_ms * 1e-3) / 1e12
    chunk_tflops = weak_scaling_rate(c_flops * args.steps, world, ch_total * 1e-3) / 1e12
    dec_tok_s = weak_scaling_rate(dw.B * dw.steps * args.steps, world, de_total * 1e-3)
    dec_gbs = (kv_bytes + other_bytes) / ((de_total / args.steps) * 1e-3) / 1e9
    dec_kv_gbs = kv_bytes / ((de_total / args.steps) * 1e-3) / 1e9
    # roofline of the dominant launch (decode: split-KV kernel and its merge), bytes
    # it must move per call (K/V rows in the window, q in, out back) over the
    # event-timed duration of the calls
    dec_call_ms = max_over_ranks(dec_call_ms, world)
    dec_call_bytes = kv_bytes + dw.steps * dw.B * 2 * dw.Hq * dw.D * 2
    dec_call_gbs = dec_call_bytes / (dec_call_ms * 1e-3) / 1e9

    # ---- end to end through the public API with host buffers.  Per sequence,
    # the host->device copies, the prefill and the device->host copy of the
    # output run on three streams (two sets of device buffers, alternating by
    # step), so the copies of one sequence overlap the other's work, as a
    # serving loop would run them; every byte still crosses PCIe every step.
    hq, hk, hv = q_cpu.pin_memory(), k_cpu.pin_memory(), v_cpu.pin_memory()
    hout = torch.empty(out.shape, dtype=out.dtype, pin_memory=True)
    bufs = [(torch.empty_like(q), torch.empty_like(k), torch.empty_like(v), torch.empty_like(out))
            for _ in range(2)]
    s_cmp = torch.cuda.current_stream(dev)
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    evk = [(kind, x, b) for kind in ("in", "cmp", "out") for x in range(2) for b in range(hp.B)]
    ev = {key: torch.cuda.Event() for key in evk}
    for e in ev.values():
        e.record(s_cmp)                       # every wait below has an event to wait on
    torch.cuda.synchronize()

    def e2e_step(i):
        x = i % 2
        dq, dk, dv, do = bufs[x]
        for b in range(hp.B):
            with torch.cuda.stream(s_in):
                s_in.wait_event(ev[("cmp", x, b)])          # the prefill two steps back has read them
                dq[b].copy_(hq[b], non_blocking=True)
                dk[b].copy_(hk[b], non_blocking=True)
                dv[b].copy_(hv[b], non_blocking=True)
                ev[("in", x, b)].record(s_in)
            s_cmp.wait_event(ev[("in", x, b)])
            s_cmp.wait_event(ev[("out", x, b)])             # its output two steps back is copied out
            swa.swa_prefill(dq[b:b + 1], dk[b:b + 1], dv[b:b + 1], hp.W, hp.scale, out=do[b:b + 1])
            ev[("cmp", x, b)].record(s_cmp)
            with torch.cuda.stream(s_out):
                s_out.wait_event(ev[("cmp", x, b)])
                hout[b].copy_(do[b], non_blocking=True)
                ev[("out", x, b)].record(s_out)

    for i in range(max(1, args.warmup)):
        e2e_step(i)
    torch.cuda.synchronize()
    barrier(world)
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    e0.record(s_in)
    for i in range(args.steps):
        e2e_step(i)
    e1.record(s_out)                          # after the last copy out, which follows all the work
    torch.cuda.synchronize()
    e2e_ms = max_over_ranks(e0.elapsed_time(e1), world)
    e2e_value = weak_scaling_rate(pf_flops * args.steps, world, e2e_ms * 1e-3) / 1e12
    h2d = (hq.numel() + hk.numel() + hv.numel()) * 2
    d2h = hout.numel() * 2
    # the copy bound of that loop: the same bytes moved by plain copies, each
    # direction alone and both at once (pinned host memory, two streams)
    pcie = measure_pcie(dev, h2d, d2h, world)
    pcie["frac_of_both_at_once"] = pcie["both_ms"] / (e2e_ms / args.steps)

    # per step: the one-shot prefill, attention + append per chunk, and per
    # decode step the append and the decode kernels (at B=64 the 4096-key
    # window is 4 splits of 1024 keys, merged in a cluster: no merge launch)
    dec_splits = decode_splits(swa, dw.B, dw.Hq, dw.Hkv, dw.D, dw.W)
    launches_per_step = 1 + len(c_chunks) * 2 + dw.steps * (1 + decode_kernels_per_call(dec_splits))

    # ---- the widened rows, timed on their own (CUDA events, after the step)
    extras = measure_extras(swa, wl, dev, q, k, v, hp, dd, dw, max(3, args.steps // 2), world)
    sweep = measure_sweep(swa, wl, dev, max(3, args.steps // 2), world)

    result = None
    if rank == 0:
        cpu = None
        if not args.no_cpu_baseline and world == 1:
            tf, secs, rows, thr, check = cpu_oracle_sample(args.cpu_seconds, gpu_out=out)
            cpu = {"value": tf, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                   "sample": f"{rows} query rows x B={hp.B} x {hp.Hq} heads of the headline prefill "
                             f"(each row W={hp.W} keys), fp64, {secs:.1f} s"}
            if check is not None:       # the timed step's own output on the sampled rows
                cpu["check_of_timed_output"] = check
        traffic = ncu_traffic("swa_prefill_kernel<128>")
        result = {
            "metric": METRIC,
            "value": value,
            "unit": "TFLOP/s",
            "n_gpus": world,
            "steps": args.steps,
            "warmup": args.warmup,
            "ms_per_step": step_total / args.steps,
            "higher_is_better": True,
            "scaling": "weak",
            "vs_baseline": None,
            "dtype": "bf16",
            "data": "synthetic",
            "config": bench_config(hp, world),
            "roofline": {
                "bound": "hbm",
                "kernel": ("swa_decode (swa_decode_kernel<128,4>, its 4 splits merged in a cluster)"
                           if decode_kernels_per_call(dec_splits) == 1 and dec_splits == 4 else
                           "swa_decode (swa_decode_kernel<128,4> + swa_decode_combine_kernel<128,4>)"),
                "splits_per_window": dec_splits,
                "why_this_kernel": "largest share of the step's GPU time (ncu launch list and events)",
                "achieved": dec_call_gbs,
                "peak": peaks["hbm_gbs"],
                "unit": "GB/s",
                "frac": dec_call_gbs / peaks["hbm_gbs"],
                "peak_kind": f"HBM copy ({peaks['source']})",
                "frac_nominal": dec_call_gbs / NOMINAL_HBM_GBS,
                "nominal_peak": NOMINAL_HBM_GBS,
                "traffic": ncu_traffic("swa_decode_kernel<128,4>"),
                "algorithmic_bytes_per_launch": dec_call_bytes / dw.steps,
                "avg_launch_us": dec_call_ms * 1e3 / dw.steps,
            },
            "roofline_prefill": {
                "bound": "tensor",
                "kernel": "swa_prefill_kernel<128>",
                "achieved": achieved,
                "peak": peaks["bf16"],
                "unit": "TFLOP/s",
                "frac": achieved / peaks["bf16"],
                "peak_kind": f"bf16 dense burst ({peaks['source']})",
                "frac_of_sustained": achieved / peaks["bf16_sustained"],
                "frac_nominal": achieved / NOMINAL_BF16_TFLOPS,
                "nominal_peak": NOMINAL_BF16_TFLOPS,
                "traffic": traffic,
                "algorithmic_flops_per_launch": pf_flops,
            },
            "decode": {
                "workload": dw.name,
                "tokens_per_s": dec_tok_s,
                "ms_per_128_steps": de_total / args.steps,
                "roofline": {
                    "bound": "hbm",
                    "achieved": dec_gbs,
                    "achieved_kv_only": dec_kv_gbs,
                    "peak": peaks["hbm_gbs"],
                    "unit": "GB/s",
                    "frac": dec_gbs / peaks["hbm_gbs"],
                    "frac_kv_only": dec_kv_gbs / peaks["hbm_gbs"],
                    "bytes_per_128_steps": kv_bytes + other_bytes,
                    "traffic": ncu_traffic("swa_decode_kernel<128,4>"),
                },
            },
            "chunked": {"workload": cw.name, "tflops": chunk_tflops,
                        "ms": ch_total / args.steps,
                        "frac": chunk_tflops / world / peaks["bf16"]},
            "e2e": {"value": e2e_value, "unit": "TFLOP/s", "h2d_bytes_per_step": h2d,
                    "d2h_bytes_per_step": d2h, "ms_per_step": e2e_ms / args.steps, "copy_bound": pcie},
            "extras": extras,
            "sweep": sweep,
            "gpu_launches": launches_per_step * args.steps,
            "clocks": clk.summary(),
            "device_status": status,
        }
        if cpu is not None:
            result["cpu_baseline"] = cpu
    del graph
    if world > 1:
        import torch.distributed as dist
        dist.destroy_process_group()
    return result


def measure_pcie(dev, h2d_bytes: int, d2h_bytes: int, world: int) -> dict:
    """Plain copies of the end-to-end step's bytes between pinned host memory
    and the device: host->device alone, device->host alone, and both at once
    on two streams (median of 5 each, CUDA events, max over ranks)."""
    import torch
    hin = torch.empty(h2d_bytes, dtype=torch.uint8, pin_memory=True)
    din = torch.empty(h2d_bytes, dtype=torch.uint8, device=dev)
    dout = torch.empty(d2h_bytes, dtype=torch.uint8, device=dev)
    hout = torch.empty(d2h_bytes, dtype=torch.uint8, pin_memory=True)
    s1, s2 = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    cur = torch.cuda.current_stream(dev)

    def both():
        s1.wait_stream(cur)
        s2.wait_stream(cur)
        with torch.cuda.stream(s1):
            din.copy_(hin, non_blocking=True)
        with torch.cuda.stream(s2):
            hout.copy_(dout, non_blocking=True)
        cur.wait_stream(s1)
        cur.wait_stream(s2)

    t_in = max_over_ranks(_time_ms(lambda: din.copy_(hin, non_blocking=True), 5), world)
    t_out = max_over_ranks(_time_ms(lambda: hout.copy_(dout, non_blocking=True), 5), world)
    t_both = max_over_ranks(_time_ms(both, 5), world)
    return {"h2d_gbs": h2d_bytes / t_in / 1e6, "d2h_gbs": d2h_bytes / t_out / 1e6, "both_ms": t_both,
            "note": "frac_of_both_at_once = time of the step's bytes copied both ways at once / e2e time per step"}


def _time_ms(fn, iters: int) -> float:
    """Median CUDA-event time of fn() on the current stream, after one warm-up."""
    import torch
    fn()
    ts = []
    for _ in range(iters):
        a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        a.record()
        fn()
        b.record()
        b.synchronize()
        ts.append(a.elapsed_time(b))
    return statistics.median(ts)


def measure_sweep(swa, wl, dev, iters, world):
    """The long-prefill sweep (B=2, 32/8 heads, D=128): N in {4K, 8K, 16K, 32K}
    x W in {1024, 4096}, plus the dense-causal control W = N; useful TFLOP/s
    and ms per launch (CUDA events, median).  The inputs are the seeded
    ``workloads.sweep_point`` draws (1% of key rows x8), the same tensors the
    parity tests compare with the oracle at every point.  Also the time ratio
    of dense causal to W=4096 at N=16K, the pages' "about 2x faster at 16K"
    setting."""
    import torch
    res = {}
    for N in wl.SWEEP_N:
        w0 = wl.sweep_point(N, 4096)
        q, k, v = (t.to(dev) for t in wl.prefill_inputs(w0))
        out = torch.empty_like(q)
        for W in sorted(set(wl.SWEEP_W) | {N}):
            w = wl.sweep_point(N, W)
            ms = max_over_ranks(_time_ms(lambda: swa.swa_prefill(q, k, v, w.W, w.scale, out=out), iters), world)
            tf = wl.useful_flops(w.B, N, W, w.Hq, w.D) / (ms * 1e-3) / 1e12
            res[f"N{N}_W{W}" + ("_dense" if W == N else "")] = {"tflops": tf, "ms": ms}
        del q, k, v, out
    res["dense_over_swa_time_N16384_W4096"] = res["N16384_W16384_dense"]["ms"] / res["N16384_W4096"]["ms"]
    return res


def measure_extras(swa, wl, dev, q, k, v, hp, dd, dw, iters, world):
    """RoPE-fused prefill and decode, attention sinks, and a mixed
    variable-length launch (pre-fill chunks and decode tokens together), on the
    headline shapes; each reported with its useful work rate."""
    import torch
    theta, S = 10000.0, 4
    res = {}
    out = torch.empty_like(q)
    kr = k.clone()
    swa.swa_rope(kr, torch.zeros(hp.B, dtype=torch.int32, device=dev), theta)
    flops = wl.useful_flops(hp.B, hp.N, hp.W, hp.Hq, hp.D)
    ms = max_over_ranks(_time_ms(lambda: swa.swa_prefill(q, kr, v, hp.W, hp.scale, out=out, rope_theta=theta),
                                 iters), world)
    res["prefill_rope_q_fused"] = {"tflops": flops / ms / 1e9, "ms": ms,
                                   "note": "q rotated in shared memory after its TMA load; k pre-rotated"}
    sink_pairs = sum(max(0, min(S, i - hp.W + 1)) for i in range(hp.N))   # sink keys outside the window
    sflops = flops + 4 * hp.B * hp.Hq * hp.D * sink_pairs
    ms = max_over_ranks(_time_ms(lambda: swa.swa_prefill_sinks(q, k, v, hp.W, S, hp.scale, out=out), iters), world)
    res["prefill_sinks4"] = {"tflops": sflops / ms / 1e9, "ms": ms}
    # the same prompt (sequence 0) pre-filled in chunks of W with 4 sinks
    C = hp.W
    cqs = [(q[:1, s0:s0 + C].contiguous(), k[:1, s0:s0 + C].contiguous(), v[:1, s0:s0 + C].contiguous())
           for s0 in range(0, hp.N, C)]
    cst = [torch.full((1,), s0, dtype=torch.int32, device=dev) for s0 in range(0, hp.N, C)]
    ckc = torch.zeros(1, hp.W, hp.Hkv, hp.D, dtype=torch.bfloat16, device=dev)
    cvc = torch.zeros_like(ckc)
    cks = torch.zeros(1, S, hp.Hkv, hp.D, dtype=torch.bfloat16, device=dev)
    cvs = torch.zeros_like(cks)
    couts = [torch.empty_like(a) for a, _, _ in cqs]

    def chunks_sinks():
        for (a, b_, c), st, o in zip(cqs, cst, couts):
            swa.swa_prefill_chunk_sinks(a, b_, c, ckc, cvc, cks, cvs, st, hp.W, hp.scale, out=o)

    ms = max_over_ranks(_time_ms(chunks_sinks, iters), world)
    res["chunked_sinks4_B1"] = {"tflops": sflops / hp.B / ms / 1e9, "ms": ms, "chunks": len(cqs)}
    # decode with fused RoPE and with sinks: one step at B=64 (append + decode)
    kc, vc = dd["k_cache"].to(dev), dd["v_cache"].to(dev)
    ks = torch.zeros(dw.B, S, dw.Hkv, dw.D, dtype=torch.bfloat16, device=dev)
    vs = torch.zeros_like(ks)
    qd = dd["q"][0].to(dev)
    kn = dd["k_new"][0].to(dev).unsqueeze(1).contiguous()
    vn = dd["v_new"][0].to(dev).unsqueeze(1).contiguous()
    pos = dd["pos0"].to(dev)
    od = torch.empty_like(qd)
    ws = torch.empty(max(256, swa.swa_decode_workspace_size(dw.B, dw.Hq, dw.Hkv, dw.D, dw.W + S)),
                     dtype=torch.uint8, device=dev)

    def dec_rope():
        swa.swa_cache_append(kn, vn, kc, vc, pos, rope_theta=theta)
        swa.swa_decode(qd, kc, vc, pos, dw.scale, out=od, workspace=ws, rope_theta=theta)

    def dec_sinks():
        swa.swa_cache_append_sinks(kn, vn, kc, vc, ks, vs, pos)
        swa.swa_decode_sinks(qd, kc, vc, ks, vs, pos, dw.scale, out=od, workspace=ws)

    # timed as the decode of the step runs: 16 steps (the same position each
    # time) captured in one CUDA graph and replayed
    reps = 16
    for name, fn in (("decode_rope_step", dec_rope), ("decode_sinks4_step", dec_sinks)):
        fn()
        torch.cuda.synchronize()
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            for _ in range(reps):
                fn()
        ms = max_over_ranks(_time_ms(graph.replay, iters), world) / reps
        del graph
        res[name] = {"tokens_per_s": dw.B * world / (ms * 1e-3), "us": ms * 1e3,
                     "note": "append + decode (+ split merge) per step, replayed from a 16-step CUDA graph"}
    # mixed launch: 4 sequences pre-fill a 4096-token chunk, 60 decode one token
    nseq, nchunk, C = 64, 4, 4096
    lens = [C] * nchunk + [1] * (nseq - nchunk)
    total = sum(lens)
    cu = torch.tensor([0] + list(itertools.accumulate(lens)), dtype=torch.int32, device=dev)
    start = pos[:nseq].clone()
    qm = wl.random_bf16((total, hp.Hq, hp.D), 7001).to(dev)
    km = wl.random_bf16((total, hp.Hkv, hp.D), 7002).to(dev)
    vm = wl.random_bf16((total, hp.Hkv, hp.D), 7003).to(dev)
    om = torch.empty_like(qm)
    kcm, vcm = kc[:nseq].contiguous(), vc[:nseq].contiguous()
    ms = max_over_ranks(_time_ms(lambda: swa.swa_prefill_chunk_varlen(qm, km, vm, kcm, vcm, start, cu, dw.W,
                                                                       hp.scale, out=om), iters), world)
    # useful pairs: each chunk row sees min(W, s0 + t + 1) keys; each decode row min(W, s0 + 1)
    pairs = 0
    s0 = start.cpu().tolist()
    for b, n in enumerate(lens):
        pairs += sum(min(dw.W, s0[b] + t + 1) for t in range(n))
    res["varlen_mixed_4x4096_plus_60_decode"] = {"tflops": 4 * hp.Hq * hp.D * pairs * world / ms / 1e9,
                                                 "ms": ms, "tokens": total}
    return res


def run_reference(args):
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return None
    from sliding_window_gqa_prefill_b200 import workloads as wl
    hp = wl.HEADLINE_PREFILL
    per_step = max(1.0, min(args.cpu_seconds, 150.0 / max(1, args.steps + args.warmup)))
    for _ in range(args.warmup):
        cpu_oracle_sample(per_step / 4)  # warm-up
    vals, secs, rows_total, thr = [], 0.0, 0, 1
    for _ in range(args.steps):
        tf, s, rows, thr, _ = cpu_oracle_sample(per_step)
        vals.append(tf)
        secs += s
        rows_total += rows
    value = statistics.median(vals)
    sample = (f"{rows_total // max(1, args.steps)} query rows per step x B={hp.B} x {hp.Hq} heads of "
              f"the headline prefill (W={hp.W} keys each), fp64 oracle")
    return {
        "impl": "reference",
        "metric": METRIC,
        "value": value,
        "unit": "TFLOP/s",
        "n_gpus": int(os.environ.get("WORLD_SIZE", "1")),
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": secs / max(1, args.steps) * 1e3,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        "dtype": "f64",
        "data": "synthetic",
        "config": bench_config(hp, int(os.environ.get("WORLD_SIZE", "1"))),
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": thr, "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }


def run_ncu_case(case: str) -> None:
    """Launches for ncu captures, each repeated so a capture can skip warm-up
    launches: `prefill_b2` the headline prefill at its benchmark size (671 MB
    on the device), `prefill` half of it (B=1, same per-unit structure),
    `chunk` the benchmark's chunked prefill (4 x attention + append), `decode`
    a reduced decode (B=16, a quarter of the batch, positions from the same
    distribution, still above L2; 4 splits per window, merged in a cluster),
    `decode_w8k` the same batch with an 8192-slot buffer (8 splits per
    window, so the split merge kernel runs), `mixed` the benchmark's mixed packed call
    (4 chunks of 4096 and 60 decode tokens over the decode workload's 1 GB of
    buffers; its decode tokens run in the decode kernel's cluster mode).
    Prints the algorithmic bytes per launch so a capture's DRAM traffic can be
    compared with (or scaled to) the benchmark's launch."""
    import dataclasses
    import torch
    import sliding_window_gqa_prefill_b200 as swa
    from sliding_window_gqa_prefill_b200 import workloads as wl
    swa.lib()
    if case in ("prefill", "prefill_b2"):
        w = wl.HEADLINE_PREFILL if case == "prefill_b2" else dataclasses.replace(wl.HEADLINE_PREFILL, B=1)
        q, k, v = (t.cuda() for t in wl.prefill_inputs(w))
        for _ in range(3):
            swa.swa_prefill(q, k, v, w.W, w.scale)
        alg = (q.numel() + k.numel() + v.numel() + q.numel()) * 2
        print(f"ncu case {case} {w.name} B={w.B}: algorithmic bytes per launch {alg}, "
              f"useful FLOPs {wl.useful_flops(w.B, w.N, w.W, w.Hq, w.D)}")
    elif case == "chunk":
        # the benchmark's chunked prefill as it runs (B=1, 4 chunks of 4096
        # through a 4096-slot buffer): per chunk one attention launch, then the
        # append launch of 4096 rows; the 4th chunk reads a full buffer
        w = wl.CHUNKED_16K
        q, k, v = (t.cuda() for t in wl.chunked_inputs(w))
        kc = torch.zeros(w.B, w.W, w.Hkv, w.D, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        for s0 in range(0, w.N, w.C):
            st = torch.full((w.B,), s0, dtype=torch.int32, device="cuda")
            swa.swa_prefill_chunk(q[:, s0:s0 + w.C].contiguous(), k[:, s0:s0 + w.C].contiguous(),
                                  v[:, s0:s0 + w.C].contiguous(), kc, vc, st, w.W, w.scale)
        rows = w.B * w.C
        alg_attn = rows * (w.Hq * 2 + w.Hkv * 2 * 2) * w.D * 2 + 2 * w.B * w.W * w.Hkv * w.D * 2
        alg_append = 2 * 2 * rows * w.Hkv * w.D * 2
        print(f"ncu case chunk {w.name}: 4th chunk attention algorithmic bytes {alg_attn} (q, k, v, out of "
              f"the chunk + full K/V buffer), useful FLOPs "
              f"{wl.useful_flops(w.B, w.N, w.W, w.Hq, w.D) - wl.useful_flops(w.B, w.N - w.C, w.W, w.Hq, w.D)}; "
              f"append of {w.C} rows algorithmic bytes {alg_append} (k, v read and written)")
    elif case == "mixed":
        import itertools
        hp, dw = wl.HEADLINE_PREFILL, wl.DECODE_B64
        d = wl.decode_inputs(dataclasses.replace(dw, steps=1))
        kc, vc = d["k_cache"].cuda(), d["v_cache"].cuda()
        lens = [4096] * 4 + [1] * 60
        total = sum(lens)
        cu = torch.tensor([0] + list(itertools.accumulate(lens)), dtype=torch.int32, device="cuda")
        start = d["pos0"].cuda()
        qm = wl.random_bf16((total, hp.Hq, hp.D), 7001).cuda()
        km = wl.random_bf16((total, hp.Hkv, hp.D), 7002).cuda()
        vm = wl.random_bf16((total, hp.Hkv, hp.D), 7003).cuda()
        om = torch.empty_like(qm)
        for _ in range(3):
            swa.swa_prefill_chunk_varlen(qm, km, vm, kc, vc, start, cu, dw.W, hp.scale, out=om)
        keys = sum(min(int(p) + 1, dw.W) for p in d["pos0"][4:])
        alg = keys * dw.Hkv * dw.D * 2 * 2 + 60 * hp.Hq * hp.D * 2 * 2
        print(f"ncu case mixed: decode-token launch algorithmic bytes {alg} (K/V rows in the 60 windows, "
              f"the own rows included, + q + out rows)")
    else:
        w = dataclasses.replace(wl.DECODE_B64, B=16, steps=1, W=8192 if case == "decode_w8k" else wl.DECODE_B64.W)
        d = wl.decode_inputs(w)
        kc, vc, pos = d["k_cache"].cuda(), d["v_cache"].cuda(), d["pos0"].cuda()
        q = d["q"][0].cuda().contiguous()
        ws = torch.empty(swa.swa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.W), dtype=torch.uint8,
                         device="cuda")
        for _ in range(3):
            swa.swa_decode(q, kc, vc, pos, w.scale, workspace=ws)
        keys = sum(min(int(p) + 1, w.W) for p in d["pos0"])
        alg = keys * w.Hkv * w.D * 2 * 2 + q.numel() * 2 * 2
        print(f"ncu case {case} B=16 W={w.W}: algorithmic bytes per launch {alg} (K/V rows in the window "
              f"+ q + out), {decode_splits(swa, w.B, w.Hq, w.Hkv, w.D, w.W)} splits per window")
    torch.cuda.synchronize()
    if swa.swa_get_device_status() != 0:
        raise SystemExit("device status not OK")


def main(argv=None):
    args = parse_args(argv)
    if args.ncu_case:
        run_ncu_case(args.ncu_case)
        return
    os.environ.setdefault("OMP_NUM_THREADS", str(os.cpu_count() or 1))
    if args.impl == "reference":
        res = run_reference(args)
    else:
        res = run_native(args)
    if res is not None:
        print(json.dumps(res), flush=True)
        if args.log:
            write_log(args.log, res)


def write_log(path: str, res: dict) -> None:
    """Append the result line, then one row per measured part (each with the
    workload config, so that rows stand alone), as JSON lines."""
    rows = [res]
    base = {"impl": res.get("impl", "native"), "config": res.get("config"), "clocks": res.get("clocks")}
    for part in ("decode", "chunked", "roofline", "roofline_prefill", "e2e", "cpu_baseline"):
        if isinstance(res.get(part), dict):
            rows.append({"part": part, **base, **res[part]})
    for group in ("extras", "sweep"):
        for name, val in (res.get(group) or {}).items():
            rows.append({"part": f"{group}.{name}", **base,
                         **(val if isinstance(val, dict) else {"value": val})})
    with open(path, "a") as f:
        for r in rows:
            f.write(json.dumps(r) + "\n")


if __name__ == "__main__":
    main()
