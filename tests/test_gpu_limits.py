"""Limits of the entry points against the fp64 oracle: decode windows that
take more than 16 splits (the split merge's looped path, and the decode
clusters of a packed batch at 8192 keys per block), positions next to the
int32 maximum (chunk, append, decode, RoPE), and a packed batch of the most
sequences one launch takes (256), one past it rejected before any launch.

Bar: max-abs 2e-2, mean-abs 2e-3 on bf16 outputs; buffers bit-exact.
Pages: read and write steps of "Rolling Buffer KV Cache 동작 설명" (P1),
sections 3.3-3.4 and 4.1 of the manon006 review.
"""
import math

import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu
MAX_ABS, MEAN_ABS = 2e-2, 2e-3
INT32_MAX = 2 ** 31 - 1


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


def _filled_buffers(oracle_mod, B, W, Hkv, D, counts, seed):
    """Buffers holding each sequence's last min(count, W) positions, written
    through the oracle's write rule; returns (k, v, slot_pos) as float64 /
    int32 arrays."""
    kr = np.zeros((B, W, Hkv, D))
    vr = np.zeros_like(kr)
    sp = np.full((B, W), -1, np.int32)
    for b, c in enumerate(counts):
        n = min(int(c), W)
        if n == 0:
            continue
        kh = f64(wl.random_bf16((1, n, Hkv, D), seed + b))
        vh = f64(wl.random_bf16((1, n, Hkv, D), seed + 100 + b))
        kb, vb, sb = kr[b:b + 1].copy(), vr[b:b + 1].copy(), sp[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, sb, kh, vh, [int(c) - n])
        kr[b], vr[b], sp[b] = kb[0], vb[0], sb[0]
    return kr, vr, sp


@pytest.mark.parametrize("W,Hq,Hkv,D", [(20000, 8, 2, 128), (32768, 8, 2, 64), (20000, 4, 4, 128)])
def test_decode_beyond_16_splits(oracle_mod, W, Hq, Hkv, D):
    """21 to 43 splits (B=3 is a small batch: splits of 512-960 keys): the
    merge takes its looped path; the static-scratch entry point gives the
    same bits."""
    B = 3
    pos = np.array([W - 2, W + 5, 3 * W + 17], np.int32)
    kr, vr, sp = _filled_buffers(oracle_mod, B, W, Hkv, D, pos, 4000 + W)   # positions 0 .. pos-1
    q = wl.random_bf16((B, Hq, D), 4100)
    kn = wl.random_bf16((B, 1, Hkv, D), 4101)
    vn = wl.random_bf16((B, 1, Hkv, D), 4102)
    scale = 1 / math.sqrt(D)
    kg = torch.from_numpy(kr).to(torch.bfloat16).cuda()
    vg = torch.from_numpy(vr).to(torch.bfloat16).cuda()
    pg = torch.from_numpy(pos).cuda()
    swa.swa_cache_append(kn.cuda(), vn.cuda(), kg, vg, pg)
    out = swa.swa_decode(q.cuda(), kg, vg, pg, scale)
    out_na = torch.empty_like(out)
    swa.swa_decode_noalloc(q.cuda(), kg, vg, pg, scale, out_na)
    torch.cuda.synchronize()
    oracle_mod.cache_append(kr, vr, sp, f64(kn), f64(vn), pos)
    ref = oracle_mod.swa_decode(f64(q), kr, vr, sp, pos, W, scale)
    close(out.cpu(), ref, f"decode W={W}")
    assert torch.equal(out, out_na)
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)


def test_packed_decode_tokens_with_a_32k_window(oracle_mod):
    """Decode tokens of a packed chunk batch at W=32768: each 4-block cluster
    takes 8192 keys per block; a chunk shares the call."""
    W, Hq, Hkv, D = 32768, 8, 2, 128
    hist = [40000, 32767, 5, 70000]
    now = [1, 1, 1, 300]
    B = len(hist)
    kr, vr, sp = _filled_buffers(oracle_mod, B, W, Hkv, D, hist, 4200)
    total = sum(now)
    cu = np.array([0] + list(np.cumsum(now)), np.int32)
    q = wl.random_bf16((total, Hq, D), 4300)
    k = wl.random_bf16((total, Hkv, D), 4301)
    v = wl.random_bf16((total, Hkv, D), 4302)
    scale = 1 / math.sqrt(D)
    kg = torch.from_numpy(kr).to(torch.bfloat16).cuda()
    vg = torch.from_numpy(vr).to(torch.bfloat16).cuda()
    out = swa.swa_prefill_chunk_varlen(q.cuda(), k.cuda(), v.cuda(), kg, vg, torch.tensor(hist, dtype=torch.int32).cuda(),
                                       torch.from_numpy(cu).cuda(), W, scale)
    torch.cuda.synchronize()
    out = out.cpu()
    for b in range(B):
        s, e = int(cu[b]), int(cu[b + 1])
        ref = oracle_mod.swa_chunk(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None],
                                   kr[b:b + 1], vr[b:b + 1], sp[b:b + 1], [hist[b]], W, scale)
        close(out[s:e], ref[0], f"packed W=32768 seq {b}")
        kb, vb = kr[b:b + 1].copy(), vr[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, sp[b:b + 1].copy(), f64(k[s:e])[None], f64(v[s:e])[None], [hist[b]])
        kr[b], vr[b] = kb[0], vb[0]
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)


def test_positions_next_to_the_int32_maximum(oracle_mod):
    """A chunk ending 3 positions below 2^31 - 1, then decode steps up to
    2^31 - 2 (plain and with RoPE): slot arithmetic, window tests and rotation
    angles at the largest positions the int32 API carries."""
    B, Hq, Hkv, D, W, C = 2, 8, 2, 128, 512, 300
    s0 = INT32_MAX - 2 - C                       # chunk positions s0 .. INT32_MAX - 3
    kr, vr, sp = _filled_buffers(oracle_mod, B, W, Hkv, D, [s0, s0], 4400)
    q = wl.random_bf16((B, C + 2, Hq, D), 4500)
    k = wl.random_bf16((B, C + 2, Hkv, D), 4501)
    v = wl.random_bf16((B, C + 2, Hkv, D), 4502)
    scale = 1 / math.sqrt(D)
    kg = torch.from_numpy(kr).to(torch.bfloat16).cuda()
    vg = torch.from_numpy(vr).to(torch.bfloat16).cuda()
    st = torch.full((B,), s0, dtype=torch.int32).cuda()
    out = swa.swa_prefill_chunk(q[:, :C].cuda().contiguous(), k[:, :C].cuda().contiguous(),
                                v[:, :C].cuda().contiguous(), kg, vg, st, W, scale)
    torch.cuda.synchronize()
    ref = oracle_mod.swa_chunk(f64(q[:, :C]), f64(k[:, :C]), f64(v[:, :C]), kr, vr, sp, [s0, s0], W, scale)
    close(out.cpu(), ref, "chunk below 2^31")
    oracle_mod.cache_append(kr, vr, sp, f64(k[:, :C]), f64(v[:, :C]), [s0, s0])
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)
    for t in (C, C + 1):                          # positions INT32_MAX - 2, INT32_MAX - 1
        p = s0 + t
        pos = np.full(B, p, np.int32)
        pg = torch.from_numpy(pos).cuda()
        swa.swa_cache_append(k[:, t:t + 1].cuda().contiguous(), v[:, t:t + 1].cuda().contiguous(), kg, vg, pg)
        dec = swa.swa_decode(q[:, t].cuda().contiguous(), kg, vg, pg, scale)
        torch.cuda.synchronize()
        oracle_mod.cache_append(kr, vr, sp, f64(k[:, t:t + 1]), f64(v[:, t:t + 1]), pos)
        close(dec.cpu(), oracle_mod.swa_decode(f64(q[:, t]), kr, vr, sp, pos, W, scale), f"decode at {p}")
    # RoPE at the last position: q rotated in the decode kernel against the
    # oracle's rotation of q (the keys in the buffer are used as stored)
    pos = np.full(B, s0 + C + 1, np.int32)
    dec = swa.swa_decode(q[:, C + 1].cuda().contiguous(), kg, vg, torch.from_numpy(pos).cuda(), scale,
                         rope_theta=10000.0)
    torch.cuda.synchronize()
    qr = oracle_mod.rope(f64(q[:, C + 1:C + 2]), pos, 10000.0)[:, 0]
    close(dec.cpu(), oracle_mod.swa_decode(qr, kr, vr, sp, pos, W, scale), "decode with RoPE at 2^31 - 2")


def test_packed_batch_of_256_sequences(oracle_mod):
    """256 sequences (the most one packed launch takes): one-shot and chunk
    calls with lengths 0-5 (decode tokens among them) against the oracle per
    sequence; 257 sequences are rejected with SWA_ERR_UNSUPPORTED."""
    B, Hq, Hkv, D, W = 256, 8, 2, 64, 6
    rng = np.random.default_rng(4600)
    lens = rng.integers(0, 6, size=B)
    total = int(lens.sum())
    cu = np.concatenate([[0], np.cumsum(lens)]).astype(np.int32)
    q = wl.random_bf16((total, Hq, D), 4601)
    k = wl.random_bf16((total, Hkv, D), 4602)
    v = wl.random_bf16((total, Hkv, D), 4603)
    scale = 1 / math.sqrt(D)
    cug = torch.from_numpy(cu).cuda()
    out = swa.swa_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cug, W, scale)
    hist = rng.integers(0, 20, size=B).astype(np.int32)
    kr, vr, sp = _filled_buffers(oracle_mod, B, W, Hkv, D, hist, 4700)
    kg = torch.from_numpy(kr).to(torch.bfloat16).cuda()
    vg = torch.from_numpy(vr).to(torch.bfloat16).cuda()
    outc = swa.swa_prefill_chunk_varlen(q.cuda(), k.cuda(), v.cuda(), kg, vg, torch.from_numpy(hist).cuda(), cug,
                                        W, scale)
    torch.cuda.synchronize()
    out, outc = out.cpu(), outc.cpu()
    for b in range(B):
        s, e = int(cu[b]), int(cu[b + 1])
        if e == s:
            continue
        ref = oracle_mod.swa_prefill(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None], W, scale)
        close(out[s:e], ref[0], f"varlen seq {b}")
        refc = oracle_mod.swa_chunk(f64(q[s:e])[None], f64(k[s:e])[None], f64(v[s:e])[None],
                                    kr[b:b + 1], vr[b:b + 1], sp[b:b + 1], [int(hist[b])], W, scale)
        close(outc[s:e], refc[0], f"chunk varlen seq {b}")
        kb, vb = kr[b:b + 1].copy(), vr[b:b + 1].copy()
        oracle_mod.cache_append(kb, vb, sp[b:b + 1].copy(), f64(k[s:e])[None], f64(v[s:e])[None], [int(hist[b])])
        kr[b], vr[b] = kb[0], vb[0]
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)
    cu257 = torch.from_numpy(np.concatenate([cu, [cu[-1]]]).astype(np.int32)).cuda()
    with pytest.raises(swa.SwaError) as e:
        swa.swa_prefill_varlen(q.cuda(), k.cuda(), v.cuda(), cu257, W, scale)
    assert e.value.status == swa.SWA_ERR_UNSUPPORTED
