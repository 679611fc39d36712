"""Attention sinks on the CUDA path against the fp64 oracle: one-shot prefill
with the first S positions kept beside each window, and streaming decode with
a W-slot rolling buffer plus an S-slot sink buffer."""
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


@pytest.mark.parametrize("B,N,Hq,Hkv,D,W,S", [(1, 900, 8, 2, 128, 256, 4), (2, 500, 4, 4, 64, 64, 4),
                                              (1, 400, 6, 2, 128, 100, 130), (1, 300, 8, 2, 128, 512, 4)])
def test_prefill_with_sinks(oracle_mod, B, N, Hq, Hkv, D, W, S):
    q = wl.random_bf16((B, N, Hq, D), 101)
    k = wl.random_bf16((B, N, Hkv, D), 102)
    v = wl.random_bf16((B, N, Hkv, D), 103)
    scale = 1 / math.sqrt(D)
    out = swa.swa_prefill_sinks(q.cuda(), k.cuda(), v.cuda(), W, S, scale)
    torch.cuda.synchronize()
    ref = oracle_mod.swa_prefill_sinks(f64(q), f64(k), f64(v), W, S, scale)
    close(out, ref, f"prefill sinks W{W} S{S}")


@pytest.mark.parametrize("W,S,D", [(64, 4, 128), (600, 4, 128), (100, 8, 64)])
def test_streaming_decode_with_sinks(oracle_mod, W, S, D):
    """Append + decode one token at a time for sequences that run past the
    window: every step equals the oracle; the sink buffer ends up holding the
    first S positions, bit for bit."""
    B, Hq, Hkv = 2, 8, 2
    steps = W + S + 20
    q = wl.random_bf16((steps, B, Hq, D), 104)
    k = wl.random_bf16((steps, B, Hkv, D), 105)
    v = wl.random_bf16((steps, B, Hkv, D), 106)
    scale = 1 / math.sqrt(D)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ks = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vs = torch.zeros_like(ks)
    kr, vr = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    ksr, vsr = np.zeros((B, S, Hkv, D)), np.zeros((B, S, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    check = set(range(0, steps, 7)) | {W - 1, W, W + S - 1, W + S, steps - 1}
    for p in range(steps):
        pos = torch.full((B,), p, dtype=torch.int32)
        kn, vn = k[p].unsqueeze(1).cuda(), v[p].unsqueeze(1).cuda()
        swa.swa_cache_append_sinks(kn, vn, kc, vc, ks, vs, pos.cuda())
        out = swa.swa_decode_sinks(q[p].cuda(), kc, vc, ks, vs, pos.cuda(), scale)
        oracle_mod.cache_append(kr, vr, sp, f64(k[p].unsqueeze(1)), f64(v[p].unsqueeze(1)), pos.numpy())
        oracle_mod.sink_append(ksr, vsr, f64(k[p].unsqueeze(1)), f64(v[p].unsqueeze(1)), pos.numpy())
        if p in check:
            torch.cuda.synchronize()
            ref = oracle_mod.swa_decode_sinks(f64(q[p]), kr, vr, sp, ksr, vsr, pos.numpy(), W, scale)
            close(out.cpu(), ref, f"decode sinks step {p}")
    torch.cuda.synchronize()
    assert np.array_equal(f64(ks.cpu()), ksr) and np.array_equal(f64(ks.cpu()), f64(k[:S].permute(1, 0, 2, 3)))


@pytest.mark.parametrize("B,N,C,Hq,Hkv,D,W,S", [
    (1, 900, 256, 8, 2, 128, 256, 4),     # C = W
    (2, 700, 100, 4, 4, 64, 128, 8),      # C < W, MHA, D=64
    (1, 1000, 300, 6, 2, 128, 384, 130),  # two sink tiles, odd group
    (2, 2560, 1280, 16, 4, 128, 1536, 4),  # last wave split into single-head units, with a sink tile
    (1, 600, 200, 16, 1, 64, 256, 4),      # group of 16: decode as two groups of 8 on the same K/V head
    (2, 2600, 1280, 24, 8, 128, 1280, 4),  # groups of 3, 320 units: pairs of query blocks; a 40-row last chunk
    (1, 2560, 1280, 32, 32, 64, 1280, 130),  # one head per KV head in pairs of query blocks, two sink tiles
])
def test_chunked_prefill_with_sinks(oracle_mod, B, N, C, Hq, Hkv, D, W, S):
    """Chunks through the rolling buffer with the sink buffer: the outputs equal
    one-shot prefill with sinks over the whole prompt; afterwards the sink
    buffer holds positions 0..S-1 and the cache the last W positions, bit for
    bit; decode with sinks then continues the sequence."""
    q = wl.random_bf16((B, N + 2, Hq, D), 111)
    k = wl.random_bf16((B, N + 2, Hkv, D), 112)
    v = wl.random_bf16((B, N + 2, Hkv, D), 113)
    scale = 1 / math.sqrt(D)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    ks = torch.zeros(B, S, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vs = torch.zeros_like(ks)
    outs = []
    for s0 in range(0, N, C):
        e = min(N, s0 + C)
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        outs.append(swa.swa_prefill_chunk_sinks(q[:, s0:e].cuda().contiguous(), k[:, s0:e].cuda().contiguous(),
                                                v[:, s0:e].cuda().contiguous(), kc, vc, ks, vs, st, W, scale))
    torch.cuda.synchronize()
    ref = oracle_mod.swa_prefill_sinks(f64(q), f64(k), f64(v), W, S, scale)
    close(torch.cat([o.cpu() for o in outs], dim=1), ref[:, :N], f"chunked sinks W{W} S{S}")
    assert torch.equal(ks.cpu(), k[:, :S]) and torch.equal(vs.cpu(), v[:, :S])
    for slot in range(W):
        p = slot + ((N - 1 - slot) // W) * W
        assert torch.equal(kc[:, slot].cpu(), k[:, p]) and torch.equal(vc[:, slot].cpu(), v[:, p]), slot
    for p in (N, N + 1):
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        swa.swa_cache_append_sinks(k[:, p:p + 1].cuda().contiguous(), v[:, p:p + 1].cuda().contiguous(), kc, vc,
                                   ks, vs, pos)
        out = swa.swa_decode_sinks(q[:, p].cuda().contiguous(), kc, vc, ks, vs, pos, scale)
        torch.cuda.synchronize()
        close(out.cpu(), ref[:, p], f"decode with sinks after chunks at {p}")
