"""Variable-length batches in one launch against the fp64 oracle run per
sequence: packed one-shot prefill, and a mixed call in which some sequences
pre-fill a chunk (through their rolling buffer), some decode one token, one
chunk is longer than the window and one sequence is empty."""
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


@pytest.mark.parametrize("lens,Hq,Hkv,D,W", [([300, 1, 0, 1000, 129], 8, 2, 128, 256),
                                            ([64, 700, 5], 6, 2, 64, 100)])
def test_prefill_varlen_matches_per_sequence_oracle(oracle_mod, lens, Hq, Hkv, D, W):
    total = sum(lens)
    cu = torch.tensor([0] + list(np.cumsum(lens)), dtype=torch.int32)
    q = wl.random_bf16((total, Hq, D), 81)
    k = wl.random_bf16((total, Hkv, D), 82)
    v = wl.random_bf16((total, Hkv, D), 83)
    scale = 1 / math.sqrt(D)
    out = swa.swa_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu.cuda(), W, scale)
    torch.cuda.synchronize()
    out = out.cpu()
    for b, n in enumerate(lens):
        if n == 0:
            continue
        s, e = int(cu[b]), int(cu[b + 1])
        ref = oracle_mod.swa_prefill(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None], W, scale)
        close(out[s:e], ref[0], f"varlen seq {b} (n={n})")


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (6, 2), (6, 1)])   # group sizes 4, 3 and 6
def test_mixed_chunks_and_decode_in_one_launch(oracle_mod, Hq, Hkv):
    D, W = 128, 256
    scale = 1 / math.sqrt(D)
    # per sequence: history length already in the buffer, tokens in this call
    hist = [1000, 7000, 0, 300, 50]
    now = [500, 1, 300, 0, 1]
    B = len(hist)
    rng_seed = 90
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16)
    vc = torch.zeros_like(kc)
    kref, vref = f64(kc), f64(vc)
    sp = np.full((B, W), -1, np.int32)
    # fill each buffer with its history through the oracle's write rule
    for b in range(B):
        if hist[b] == 0:
            continue
        kh = wl.random_bf16((1, hist[b], Hkv, D), rng_seed + b)
        vh = wl.random_bf16((1, hist[b], Hkv, D), rng_seed + 50 + b)
        kb, vb, spb = kref[b:b + 1].copy(), vref[b:b + 1].copy(), sp[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, spb, f64(kh), f64(vh), [0])
        kref[b], vref[b], sp[b] = kb[0], vb[0], spb[0]
    kc = torch.from_numpy(kref).to(torch.bfloat16)
    vc = torch.from_numpy(vref).to(torch.bfloat16)
    total = sum(now)
    cu = np.array([0] + list(np.cumsum(now)), np.int32)
    q = wl.random_bf16((total, Hq, D), 95)
    k = wl.random_bf16((total, Hkv, D), 96)
    v = wl.random_bf16((total, Hkv, D), 97)
    kg, vg = kc.cuda(), vc.cuda()
    start = torch.tensor(hist, dtype=torch.int32)
    out = swa.swa_prefill_chunk_varlen(q.cuda(), k.cuda(), v.cuda(), kg, vg, start.cuda(),
                                       torch.from_numpy(cu).cuda(), W, scale)
    torch.cuda.synchronize()
    out = out.cpu()
    for b in range(B):
        s, e = int(cu[b]), int(cu[b + 1])
        if e == s:
            continue
        ref = oracle_mod.swa_chunk(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None],
                                   kref[b:b + 1], vref[b:b + 1], sp[b:b + 1], [hist[b]], W, scale)
        close(out[s:e], ref[0], f"mixed seq {b} (history {hist[b]}, tokens {e - s})")
        kb, vb = kref[b:b + 1].copy(), vref[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, sp[b:b + 1].copy(), f64(k[s:e])[None], f64(v[s:e])[None], [hist[b]])
        kref[b], vref[b] = kb[0], vb[0]
    assert np.array_equal(f64(kg.cpu()), kref) and np.array_equal(f64(vg.cpu()), vref)
