"""Parity at the full sizes of the five workloads, in the launch configuration
the benchmark times, against the fp64 oracle on the same seeded inputs.

* Mistral one-shot prefill (B=1, N=8192, W=4096): every output row.
* Chunked prefill (N=16384 in 4 chunks of 4096 through a 4096-slot buffer):
  every output row against one-shot SWA, final cache bit for bit.
* Batched decode (B=64, W=4096, positions uniform on [1, 32768]): all 128
  steps, replayed from one CUDA graph as the benchmark runs them; every
  written cache slot bit for bit.
* Long-prefill sweep (B=2, N in {4K, 8K, 16K, 32K} x W in {1024, 4096, N},
  1% of key rows x8): on the inputs ``bench.py`` times (``workloads.sweep_point``),
  rows at the window and tile edges, the last row, and the rows of outlier
  keys.

Bar: max-abs 2e-2, mean-abs 2e-3 on bf16 outputs; caches bit-exact.  The
workloads: "Methods" (Table 1 shapes) and "Pre-fill + Chunking" of the
"Mistral 7B -- Sliding Window Attention" summary; section 3.2 of the manon006
review (16K tokens, W=4096) for the sweep.
"""
import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    swa.build()
    swa.lib()
    yield
    assert swa.swa_get_device_status() == swa.SWA_OK


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(got: np.ndarray, ref: np.ndarray, what: str):
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"


def test_mistral_8k_prefill_every_row(oracle_mod):
    """B=1, N=8192, W=4096, 32/8 heads, D=128: the whole output."""
    w = wl.MISTRAL_PREFILL_8K
    q, k, v = wl.prefill_inputs(w)
    out = swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), w.W, w.scale)
    got = f64(out)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), w.W, w.scale)
    assert_close(got, ref, "mistral 8k, every row")


def test_chunked_16k_every_row_and_cache(oracle_mod):
    """N=16384 in 4 chunks of 4096 through the 4096-slot buffer, as the
    benchmark launches them: every output row against one-shot SWA; the
    final buffer holds positions 12288..16383 at slot p mod 4096."""
    w = wl.CHUNKED_16K
    q, k, v = wl.chunked_inputs(w)
    qg, kg, vg = q.cuda(), k.cuda(), v.cuda()
    kc = torch.zeros(w.B, w.W, w.Hkv, w.D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for s0 in range(0, w.N, w.C):
        st = torch.full((w.B,), s0, dtype=torch.int32, device="cuda")
        outs.append(swa.swa_prefill_chunk(qg[:, s0:s0 + w.C].contiguous(), kg[:, s0:s0 + w.C].contiguous(),
                                          vg[:, s0:s0 + w.C].contiguous(), kc, vc, st, w.W, w.scale))
    got = f64(torch.cat(outs, dim=1))
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), w.W, w.scale)
    assert_close(got, ref, "chunked 16k, every row")
    assert torch.equal(kc.cpu(), k[:, w.N - w.W:]) and torch.equal(vc.cpu(), v[:, w.N - w.W:])


def test_decode_b64_all_128_steps(oracle_mod):
    """B=64 sequences at positions uniform on [1, 32768], W=4096, 32/8 heads:
    all 128 steps (append, then attend) captured in one CUDA graph and
    replayed, as the benchmark runs them, against the oracle's rolling buffer
    step by step; the final caches agree bit for bit (the 128 positions of a
    sequence take 128 distinct slots, so every written slot is checked)."""
    w = wl.DECODE_B64
    d = wl.decode_inputs(w)
    kg, vg = d["k_cache"].cuda(), d["v_cache"].cuda()
    ws = torch.empty(swa.swa_decode_workspace_size(w.B, w.Hq, w.Hkv, w.D, w.W), dtype=torch.uint8,
                     device="cuda")
    outs = torch.empty(w.steps, w.B, w.Hq, w.D, dtype=torch.bfloat16, device="cuda")
    kn = d["k_new"].unsqueeze(2).cuda()             # [steps, B, 1, Hkv, D]
    vn = d["v_new"].unsqueeze(2).cuda()
    qs = d["q"].cuda()
    pos_table = (d["pos0"].unsqueeze(0) + torch.arange(w.steps, dtype=torch.int32).unsqueeze(1)).to(torch.int32)
    pg = pos_table.cuda().contiguous()              # [steps, B]
    k0, v0 = kg.clone(), vg.clone()

    def steps():
        for s in range(w.steps):
            swa.swa_cache_append(kn[s], vn[s], kg, vg, pg[s])
            swa.swa_decode(qs[s], kg, vg, pg[s], w.scale, out=outs[s], workspace=ws)

    steps()                                         # eager once (warms up), then restore the caches
    kg.copy_(k0)
    vg.copy_(v0)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        steps()
    kg.copy_(k0)                                    # capture does not run the kernels, but be explicit
    vg.copy_(v0)
    outs.zero_()
    graph.replay()
    torch.cuda.synchronize()
    del graph
    sp = oracle_mod.slot_positions(d["pos0"].numpy(), w.W)
    kr, vr = f64(d["k_cache"]), f64(d["v_cache"])
    for s in range(w.steps):
        pos = pos_table[s]
        oracle_mod.cache_append(kr, vr, sp, f64(d["k_new"][s].unsqueeze(1)), f64(d["v_new"][s].unsqueeze(1)),
                                pos.numpy())
        ref = oracle_mod.swa_decode(f64(d["q"][s]), kr, vr, sp, pos.numpy(), w.W, w.scale)
        assert_close(f64(outs[s]), ref, f"decode B64 step {s}")
    assert np.array_equal(f64(kg), kr) and np.array_equal(f64(vg), vr)


# ------------------------------------------------------------------ long-prefill sweep

_inputs_cache = {}


def _sweep_inputs(N):
    """Seeded CPU inputs of a sweep point (one set per N: the seed does not
    depend on W), kept for the W values of the same N only."""
    if N not in _inputs_cache:
        _inputs_cache.clear()
        _inputs_cache[N] = wl.prefill_inputs(wl.sweep_point(N, 4096))
    return _inputs_cache[N]


def _sweep_rows(w, k_cpu):
    """Rows at the window and tile edges, the last rows, a few random ones, and
    the positions of outlier keys (where a query sees its own outlier key)."""
    N, W = w.N, w.W
    rows = {0, 1, 126, 127, 128, 129, N - 129, N - 128, N - 1, N - 2}
    for e in (W - 2, W - 1, W, W + 1, W + 127, W + 128, 2 * W - 1, 2 * W):
        rows.add(e)
    rng = np.random.default_rng(N + 31 * W)
    rows |= set(int(x) for x in rng.integers(0, N, 16))
    norms = k_cpu.float().norm(dim=-1).amax(dim=(0, 2))          # per position, over b and heads
    out_pos = torch.nonzero(norms > 4 * float(np.sqrt(w.D))).flatten().tolist()
    assert out_pos, "outlier rows expected"
    rows |= set(rng.choice(out_pos, size=min(8, len(out_pos)), replace=False).tolist())
    return sorted(r for r in rows if 0 <= r < N)


SWEEP = [(N, W) for N in wl.SWEEP_N for W in sorted({1024, 4096, N})]


@pytest.mark.parametrize("N,W", SWEEP)
def test_sweep_point_against_oracle(oracle_mod, N, W):
    """Every point of the long-prefill sweep, on the inputs the benchmark
    times: B=2, 32/8 heads, D=128, 1% of key rows x8; W = N is the dense
    causal control."""
    w = wl.sweep_point(N, W)
    q, k, v = _sweep_inputs(N)
    out = swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), w.W, w.scale)
    rows = _sweep_rows(w, k)
    got = f64(out[:, rows])
    del out
    ref = oracle_mod.swa_prefill(q.float().numpy(), k.float().numpy(), v.float().numpy(), w.W, w.scale,
                                 rows=rows)
    assert_close(got, ref, f"sweep N{N} W{W} ({len(rows)} rows, all heads)")
