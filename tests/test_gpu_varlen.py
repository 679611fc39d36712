"""Variable-length batches in one launch against the fp64 oracle run per
sequence: packed one-shot prefill, and mixed calls in which some sequences
pre-fill a chunk (through their rolling buffer), some decode one token, one
chunk is longer than the window and one sequence is empty.  The one-token
sequences go to the decode kernel (group sizes above 8 as several groups of
up to 8 heads on the same K/V head, 16 here)."""
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
                                            ([64, 700, 5], 6, 2, 64, 100),
                                            # odd groups at two waves of units: pairs of query blocks
                                            ([700, 600, 1, 1200], 32, 32, 128, 500),
                                            ([1000, 1, 1299], 24, 8, 64, 383)])
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


def _mixed(oracle_mod, hist, now, Hq, Hkv, D, W, seed):
    """One swa_prefill_chunk_varlen call: sequence b has hist[b] positions in
    its buffer (written through the oracle's write rule) and now[b] tokens in
    the call; every output row against the oracle's chunk attention, then the
    buffers bit for bit against the oracle's write."""
    scale = 1 / math.sqrt(D)
    B = len(hist)
    kref = np.zeros((B, W, Hkv, D))
    vref = np.zeros_like(kref)
    sp = np.full((B, W), -1, np.int32)
    for b in range(B):
        n = min(hist[b], W)                  # older positions would be overwritten
        if n == 0:
            continue
        kh = wl.random_bf16((1, n, Hkv, D), seed + b)
        vh = wl.random_bf16((1, n, Hkv, D), seed + 500 + b)
        kb, vb, spb = kref[b:b + 1].copy(), vref[b:b + 1].copy(), sp[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, spb, f64(kh), f64(vh), [hist[b] - n])
        kref[b], vref[b], sp[b] = kb[0], vb[0], spb[0]
    kg = torch.from_numpy(kref).to(torch.bfloat16).cuda()
    vg = torch.from_numpy(vref).to(torch.bfloat16).cuda()
    total = sum(now)
    cu = np.array([0] + list(np.cumsum(now)), np.int32)
    q = wl.random_bf16((total, Hq, D), seed + 1001)
    k = wl.random_bf16((total, Hkv, D), seed + 1002)
    v = wl.random_bf16((total, Hkv, D), seed + 1003)
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


@pytest.mark.parametrize("Hq,Hkv", [(8, 2), (6, 2), (6, 1), (16, 1)])   # group sizes 4, 3, 6 and 16
def test_mixed_chunks_and_decode_in_one_launch(oracle_mod, Hq, Hkv):
    # per sequence: history length already in the buffer, tokens in this call
    _mixed(oracle_mod, [1000, 7000, 0, 300, 50], [500, 1, 300, 0, 1], Hq, Hkv, 128, 256, 90)


@pytest.mark.parametrize("Hq,Hkv,hist,now", [
    (24, 8, [0, 5000, 100, 9], [1000, 1, 1298, 1]),      # groups of 3, 352 head-pair units: block pairs
    (32, 32, [2000, 0, 7], [800, 900, 1]),               # one head per KV head
])
def test_mixed_batch_in_pairs_of_query_blocks(oracle_mod, Hq, Hkv, hist, now):
    """A packed chunk batch with an odd group and at least two waves of units
    takes units of two consecutive query blocks of one head (prefix sums of
    256-row pairs per sequence); its one-row sequences still go to the decode
    kernel."""
    _mixed(oracle_mod, hist, now, Hq, Hkv, 128, 1024, 95)


@pytest.mark.parametrize("G", [1, 2, 3, 4, 5, 6, 7, 8, 12])
@pytest.mark.parametrize("D", [64, 128])
def test_decode_tokens_of_a_packed_batch(oracle_mod, G, D):
    """Length-1 sequences of a chunk batch at positions around the buffer
    edges (first token, just below the window, the wrap, far past it): with
    every group size they are decoded by the decode kernel, which
    takes the token's own key and value from the packed rows (its slot still
    holds position p - W, or nothing, until the write after the attention);
    two chunks and an empty sequence share the launch."""
    W = 300
    hist = [0, 1, W - 2, W - 1, W, W + 1, 2 * W - 1, 5000, 700, 0, 37]
    now = [1, 1, 1, 1, 1, 1, 1, 1, 130, 0, 200]
    _mixed(oracle_mod, hist, now, 2 * G, 2, D, W, 300 + 10 * G + D)


def test_mixed_call_replays_from_a_cuda_graph():
    """A serving loop captures the mixed call (decode clusters, attention
    kernel, buffer write) in a CUDA graph: one replay gives the eager call's
    outputs and buffers bit for bit."""
    Hq, Hkv, D, W = 8, 2, 128, 256
    hist = [0, 300, 9000, 40, 700]
    now = [130, 1, 1, 1, 200]
    B, total = len(hist), sum(now)
    cu = torch.tensor([0] + list(np.cumsum(now)), dtype=torch.int32).cuda()
    start = torch.tensor(hist, dtype=torch.int32).cuda()
    q = wl.random_bf16((total, Hq, D), 501).cuda()
    k = wl.random_bf16((total, Hkv, D), 502).cuda()
    v = wl.random_bf16((total, Hkv, D), 503).cuda()
    kc0 = wl.random_bf16((B, W, Hkv, D), 504).cuda()
    vc0 = wl.random_bf16((B, W, Hkv, D), 505).cuda()
    kc, vc = kc0.clone(), vc0.clone()
    ref = swa.swa_prefill_chunk_varlen(q, k, v, kc, vc, start, cu, W, 0.09)
    torch.cuda.synchronize()
    kg, vg = kc0.clone(), vc0.clone()
    out = torch.empty_like(q)
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        swa.swa_prefill_chunk_varlen(q, k, v, kg, vg, start, cu, W, 0.09, out=out)
    kg.copy_(kc0)
    vg.copy_(vc0)
    graph.replay()
    torch.cuda.synchronize()
    del graph
    assert torch.equal(out, ref) and torch.equal(kg, kc) and torch.equal(vg, vc)
