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


@pytest.mark.parametrize("case", range(16))
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


@pytest.mark.parametrize("case", range(12))
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


@pytest.mark.parametrize("case", range(12))
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


@pytest.mark.parametrize("G", list(range(1, 10)) + [11, 12, 16])
def test_fuzz_decode_every_group_size(oracle_mod, G):
    """Decode at each group size 1-9 and at 11, 12 and 16 (odd ones included:
    rows past the group in the MMA tile are zero; groups above 8 run as
    several groups of up to 8 heads on the same K/V head, 11 as 11 groups of
    one), with and without RoPE, random shapes and positions."""
    rng = np.random.default_rng(12400 + G)
    B = int(rng.integers(1, 5))
    W = int(rng.integers(8, 3000))
    Hkv = int(rng.choice([1, 2, 3]))
    Hq, D = Hkv * G, int(rng.choice([64, 128]))
    seed = 12500 + 10 * G
    kc = wl.random_bf16((B, W, Hkv, D), seed)
    vc = wl.random_bf16((B, W, Hkv, D), seed + 1)
    pos0 = rng.integers(0, 3 * W, size=B).astype(np.int32)
    sp = oracle_mod.slot_positions(pos0, W)
    kr, vr = f64(kc), f64(vc)
    kg, vg = kc.cuda(), vc.cuda()
    scale = 1.0 / math.sqrt(D)
    for s in range(2):
        q = wl.random_bf16((B, Hq, D), seed + 10 + s)
        kn = wl.random_bf16((B, 1, Hkv, D), seed + 20 + s)
        vn = wl.random_bf16((B, 1, Hkv, D), seed + 30 + s)
        pos = torch.from_numpy(pos0 + s)
        swa.swa_cache_append(kn.cuda(), vn.cuda(), kg, vg, pos.cuda())
        out = swa.swa_decode(q.cuda(), kg, vg, pos.cuda(), scale)
        out_r = swa.swa_decode(q.cuda(), kg, vg, pos.cuda(), scale, rope_theta=10000.0)
        torch.cuda.synchronize()
        oracle_mod.cache_append(kr, vr, sp, f64(kn), f64(vn), pos.numpy())
        ref = oracle_mod.swa_decode(f64(q), kr, vr, sp, pos.numpy(), W, scale)
        close(out.cpu(), ref, f"decode G={G} B{B} W{W} D{D} step {s}")
        qr = oracle_mod.rope(f64(q)[:, None], pos.numpy(), 10000.0)[:, 0]
        close(out_r.cpu(), oracle_mod.swa_decode(qr, kr, vr, sp, pos.numpy(), W, scale), f"decode RoPE G={G} step {s}")
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)


@pytest.mark.parametrize("case", range(6))
def test_fuzz_varlen(oracle_mod, case):
    """Packed batch of random lengths (zeros included): each sequence equals its own one-shot prefill."""
    rng = np.random.default_rng(10100 + case)
    lens = [int(x) for x in rng.integers(0, 600, size=int(rng.integers(1, 7)))]
    lens[int(rng.integers(0, len(lens)))] = max(1, lens[0])
    W = int(rng.integers(1, 650))
    Hq, Hkv, D = _heads(rng)
    total = sum(lens)
    cu = np.array([0] + list(np.cumsum(lens)), np.int32)
    seed = 10200 + 10 * case
    q = wl.random_bf16((total, Hq, D), seed)
    k = wl.random_bf16((total, Hkv, D), seed + 1)
    v = wl.random_bf16((total, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    out = swa.swa_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), torch.from_numpy(cu).cuda(), W, scale)
    torch.cuda.synchronize()
    out = out.cpu()
    for b, n in enumerate(lens):
        s, e = int(cu[b]), int(cu[b + 1])
        if n == 0:
            continue
        ref = oracle_mod.swa_prefill(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None], W, scale)
        close(out[s:e], ref[0], f"varlen seq {b} n{n} W{W} H{Hq}/{Hkv} D{D}")


@pytest.mark.parametrize("case", range(6))
def test_fuzz_mixed_chunk_varlen(oracle_mod, case):
    """One packed call continuing several sequences from random histories (decode-length pieces included)."""
    rng = np.random.default_rng(10500 + case)
    B = int(rng.integers(1, 6))
    W = int(rng.integers(8, 700))
    Hq, Hkv, D = _heads(rng)
    hist = [int(x) for x in rng.integers(0, 3 * W, size=B)]
    now = [int(x) for x in rng.integers(0, W + 1, size=B)]
    now[0] = max(now[0], 1)
    seed = 10600 + 10 * case
    kref = np.zeros((B, W, Hkv, D))
    vref = np.zeros_like(kref)
    sp = np.full((B, W), -1, np.int32)
    for b in range(B):
        if hist[b]:
            kh = f64(wl.random_bf16((1, hist[b], Hkv, D), seed + 100 + b))
            vh = f64(wl.random_bf16((1, hist[b], Hkv, D), seed + 200 + b))
            kb, vb, spb = kref[b:b + 1].copy(), vref[b:b + 1].copy(), sp[b:b + 1].copy()
            oracle_mod.cache_append(kb, vb, spb, kh[:, -W:], vh[:, -W:], [max(0, hist[b] - W)])
            kref[b], vref[b], sp[b] = kb[0], vb[0], spb[0]
    total = sum(now)
    cu = np.array([0] + list(np.cumsum(now)), np.int32)
    q = wl.random_bf16((total, Hq, D), seed)
    k = wl.random_bf16((total, Hkv, D), seed + 1)
    v = wl.random_bf16((total, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    kg = torch.from_numpy(kref).to(torch.bfloat16).cuda()
    vg = torch.from_numpy(vref).to(torch.bfloat16).cuda()
    out = swa.swa_prefill_chunk_varlen(q.cuda(), k.cuda(), v.cuda(), kg, vg,
                                       torch.tensor(hist, dtype=torch.int32).cuda(),
                                       torch.from_numpy(cu).cuda(), W, scale)
    torch.cuda.synchronize()
    out = out.cpu()
    for b in range(B):
        s, e = int(cu[b]), int(cu[b + 1])
        if e == s:
            continue
        ref = oracle_mod.swa_chunk(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None],
                                   kref[b:b + 1], vref[b:b + 1], sp[b:b + 1], [hist[b]], W, scale)
        close(out[s:e], ref[0], f"mixed seq {b} hist{hist[b]} n{e - s} W{W} H{Hq}/{Hkv} D{D}")
        kb, vb = kref[b:b + 1].copy(), vref[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, None, f64(k[s:e])[None], f64(v[s:e])[None], [hist[b]])
        kref[b], vref[b] = kb[0], vb[0]
    assert np.array_equal(f64(kg.cpu()), kref) and np.array_equal(f64(vg.cpu()), vref)


@pytest.mark.parametrize("case", range(6))
def test_fuzz_sinks(oracle_mod, case):
    """One-shot prefill with S sink positions; S below, inside and beyond the window and the sequence."""
    rng = np.random.default_rng(10900 + case)
    B = int(rng.integers(1, 3))
    N = int(rng.integers(1, 800))
    W = int(rng.integers(1, N + 40))
    S = int(rng.integers(0, N + 20))
    Hq, Hkv, D = _heads(rng)
    seed = 11000 + 10 * case
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    out = swa.swa_prefill_sinks(q.cuda(), k.cuda(), v.cuda(), W, S, scale)
    torch.cuda.synchronize()
    ref = oracle_mod.swa_prefill_sinks(f64(q), f64(k), f64(v), W, S, scale)
    close(out, ref, f"sinks B{B} N{N} W{W} S{S} H{Hq}/{Hkv} D{D}")


@pytest.mark.parametrize("case", range(6))
def test_fuzz_rope_sequence(oracle_mod, case):
    """RoPE: one-shot prefill with q rotated in the kernel, the same prompt in
    chunks, then two decode steps with the key rotated on its way into the
    cache; every output equals SWA on exactly rotated q and k."""
    rng = np.random.default_rng(11500 + case)
    B = int(rng.integers(1, 3))
    W = int(rng.integers(16, 500))
    C = int(rng.integers(1, W + 1))
    N = int(rng.integers(C, 3 * W))
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    Hq, D = Hkv * G, int(rng.choice([64, 128]))
    theta = float(rng.choice([10000.0, 1000000.0]))
    seed = 11600 + 10 * case
    q = wl.random_bf16((B, N + 2, Hq, D), seed)
    k = wl.random_bf16((B, N + 2, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N + 2, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    zero = torch.zeros(B, dtype=torch.int32, device="cuda")
    kr_dev = k[:, :N].cuda().contiguous()
    swa.swa_rope(kr_dev, zero, theta)
    one = swa.swa_prefill(q[:, :N].cuda().contiguous(), kr_dev, v[:, :N].cuda().contiguous(), W, scale,
                          rope_theta=theta)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for s0 in range(0, N, C):
        e = min(N, s0 + C)
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        kch = k[:, s0:e].cuda().contiguous()
        swa.swa_rope(kch, st, theta)
        outs.append(swa.swa_prefill_chunk(q[:, s0:e].cuda().contiguous(), kch, v[:, s0:e].cuda().contiguous(),
                                          kc, vc, st, W, scale, rope_theta=theta))
    dec = []
    for p in (N, N + 1):
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        swa.swa_cache_append(k[:, p:p + 1].cuda().contiguous(), v[:, p:p + 1].cuda().contiguous(), kc, vc, pos,
                             rope_theta=theta)
        dec.append(swa.swa_decode(q[:, p].cuda().contiguous(), kc, vc, pos, scale, rope_theta=theta))
    torch.cuda.synchronize()
    z = np.zeros(B, np.int32)
    ref = oracle_mod.swa_prefill(oracle_mod.rope(f64(q), z, theta), oracle_mod.rope(f64(k), z, theta), f64(v),
                                 W, scale)
    tag = f"rope B{B} N{N} C{C} W{W} H{Hq}/{Hkv} D{D} theta{theta:g}"
    close(one, ref[:, :N], "one-shot " + tag)
    close(torch.cat([o.cpu() for o in outs], dim=1), ref[:, :N], "chunked " + tag)
    for i, p in enumerate((N, N + 1)):
        close(dec[i].cpu(), ref[:, p], f"decode at {p} " + tag)


@pytest.mark.parametrize("case", range(6))
def test_fuzz_sinks_sequence(oracle_mod, case):
    """Sinks: the prompt in chunks through the rolling buffer and the sink
    buffer, then two decode steps with sinks; outputs equal one-shot prefill
    with sinks over the whole sequence, buffers bit for bit."""
    rng = np.random.default_rng(11800 + case)
    B = int(rng.integers(1, 3))
    W = int(rng.integers(8, 400))
    C = int(rng.integers(1, W + 1))
    N = int(rng.integers(C, 3 * W + 2))
    S = int(rng.integers(1, min(N, 300) + 1))
    Hkv = int(rng.choice([1, 2, 4]))
    G = int(rng.choice([1, 2, 4, 8]))
    Hq, D = Hkv * G, int(rng.choice([64, 128]))
    seed = 11900 + 10 * case
    q = wl.random_bf16((B, N + 2, Hq, D), seed)
    k = wl.random_bf16((B, N + 2, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N + 2, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
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
    tag = f"sinks B{B} N{N} C{C} W{W} S{S} H{Hq}/{Hkv} D{D}"
    close(torch.cat([o.cpu() for o in outs], dim=1), ref[:, :N], "chunked " + tag)
    assert torch.equal(ks.cpu(), k[:, :S]) and torch.equal(vs.cpu(), v[:, :S]), tag
    for p in (N, N + 1):
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        swa.swa_cache_append_sinks(k[:, p:p + 1].cuda().contiguous(), v[:, p:p + 1].cuda().contiguous(), kc, vc,
                                   ks, vs, pos)
        out = swa.swa_decode_sinks(q[:, p].cuda().contiguous(), kc, vc, ks, vs, pos, scale)
        torch.cuda.synchronize()
        close(out.cpu(), ref[:, p], f"decode at {p} " + tag)
    for slot in range(min(W, N + 2)):
        p = slot + ((N + 1 - slot) // W) * W
        assert torch.equal(kc[:, slot].cpu(), k[:, p]) and torch.equal(vc[:, slot].cpu(), v[:, p]), (tag, slot)
