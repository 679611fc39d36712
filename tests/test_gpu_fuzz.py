"""Seeded random shapes on the CUDA path against the fp64 oracle: one-shot
prefill, chunked prefill and decode over batch sizes, ragged lengths, group
sizes 1..8 (including odd), head dims 64 and 128, windows not aligned to the
128-key tiles, chunk lengths and decode positions around the buffer wrap.
Same bar as the hand-picked cases: max-abs 2e-2, mean-abs 2e-3, caches bit
for bit."""
import math

import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu
MAX_ABS, MEAN_ABS = 2e-2, 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    swa.build()
    swa.lib()
    yield
    assert swa.swa_get_device_status() == swa.SWA_OK


def f64(t):
    return t.detach().float().cpu().numpy().astype(np.float64)


def close(got, ref, what):
    g = f64(got)
    assert np.isfinite(g).all(), what
    err = np.abs(g - ref)
    assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (what, err.max(), err.mean())


def _heads(rng):
    Hkv = int(rng.choice([1, 2, 3, 4]))
    G = int(rng.choice([1, 2, 3, 4, 8]))
    return Hkv * G, Hkv, int(rng.choice([64, 128]))


@pytest.mark.parametrize("case", range(10))
def test_fuzz_prefill(oracle_mod, case):
    rng = np.random.default_rng(9000 + case)
    B = int(rng.integers(1, 4))
    N = int(rng.integers(1, 700))
    W = int(rng.integers(1, N + 60))
    Hq, Hkv, D = _heads(rng)
    seed = 9100 + 10 * case
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    out = swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), W, scale)
    torch.cuda.synchronize()
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale)
    close(out, ref, f"prefill B{B} N{N} W{W} H{Hq}/{Hkv} D{D}")


@pytest.mark.parametrize("case", range(8))
def test_fuzz_chunked(oracle_mod, case):
    rng = np.random.default_rng(9500 + case)
    B = int(rng.integers(1, 3))
    W = int(rng.integers(16, 400))
    C = int(rng.integers(1, W + 1))
    N = int(rng.integers(C, 3 * W + 2))
    Hq, Hkv, D = _heads(rng)
    seed = 9600 + 10 * case
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for s0 in range(0, N, C):
        e = min(N, s0 + C)
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        outs.append(swa.swa_prefill_chunk(q[:, s0:e].cuda().contiguous(), k[:, s0:e].cuda().contiguous(),
                                          v[:, s0:e].cuda().contiguous(), kc, vc, st, W, scale))
    torch.cuda.synchronize()
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale)
    close(torch.cat([o.cpu() for o in outs], dim=1), ref, f"chunked B{B} N{N} C{C} W{W} H{Hq}/{Hkv} D{D}")
    for slot in range(min(W, N)):
        p = slot + ((N - 1 - slot) // W) * W
        assert torch.equal(kc[:, slot].cpu(), k[:, p]) and torch.equal(vc[:, slot].cpu(), v[:, p]), slot


@pytest.mark.parametrize("case", range(8))
def test_fuzz_decode(oracle_mod, case):
    rng = np.random.default_rng(9800 + case)
    B = int(rng.integers(1, 6))
    W = int(rng.integers(8, 2500))
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    Hq, D = Hkv * G, int(rng.choice([64, 128]))
    seed = 9900 + 10 * case
    kc = wl.random_bf16((B, W, Hkv, D), seed)
    vc = wl.random_bf16((B, W, Hkv, D), seed + 1)
    pos0 = rng.integers(0, 3 * W, size=B).astype(np.int32)
    # slot s holds the latest position < pos0 with that slot (every slot written)
    sp = oracle_mod.slot_positions(pos0, W)
    kr, vr = f64(kc), f64(vc)
    kg, vg = kc.cuda(), vc.cuda()
    scale = 1.0 / math.sqrt(D)
    for s in range(3):
        q = wl.random_bf16((B, Hq, D), seed + 10 + s)
        kn = wl.random_bf16((B, 1, Hkv, D), seed + 20 + s)
        vn = wl.random_bf16((B, 1, Hkv, D), seed + 30 + s)
        pos = torch.from_numpy(pos0 + s)
        swa.swa_cache_append(kn.cuda(), vn.cuda(), kg, vg, pos.cuda())
        out = swa.swa_decode(q.cuda(), kg, vg, pos.cuda(), scale)
        torch.cuda.synchronize()
        oracle_mod.cache_append(kr, vr, sp, f64(kn), f64(vn), pos.numpy())
        ref = oracle_mod.swa_decode(f64(q), kr, vr, sp, pos.numpy(), W, scale)
        close(out.cpu(), ref, f"decode B{B} W{W} H{Hq}/{Hkv} D{D} step {s}")
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)
