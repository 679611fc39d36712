"""Rotary position embedding on the CUDA path against the fp64 oracle.

The rotation itself is compared element by element: the GPU rotates in fp32
and rounds to bf16, so each element must lie within one bf16 rounding step
(2^-8 relative) of the exact fp64 rotation.  Attention with the rotation fused
into the Q load (prefill, chunked prefill, decode) and into the cache write
(append) is held to the same bar as the rest of the path (max-abs 2e-2,
mean-abs 2e-3 against the oracle run on exactly rotated inputs).
"""
import math

import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu

THETA = 10000.0
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


@pytest.mark.parametrize("B,T,H,D,pos", [(2, 33, 8, 128, [0, 31000]), (1, 5, 3, 64, [4095])])
def test_rope_kernel_within_one_rounding_step(oracle_mod, B, T, H, D, pos):
    x = wl.random_bf16((B, T, H, D), 61, scale=3.0)
    p = torch.tensor(pos, dtype=torch.int32)
    g = x.cuda()
    swa.swa_rope(g, p.cuda(), THETA)
    torch.cuda.synchronize()
    ref = oracle_mod.rope(f64(x), p.numpy(), THETA)
    got = f64(g)
    assert (np.abs(got - ref) <= np.abs(ref) * 2.0 ** -8 + 1e-6).all()
    exact_rounded = torch.from_numpy(ref).to(torch.bfloat16).float().numpy()
    assert (got == exact_rounded).mean() > 0.98


def test_cache_append_rope(oracle_mod):
    B, T, Hkv, D, W = 3, 7, 8, 128, 64
    kc = wl.random_bf16((B, W, Hkv, D), 62)
    vc = wl.random_bf16((B, W, Hkv, D), 63)
    kn = wl.random_bf16((B, T, Hkv, D), 64)
    vn = wl.random_bf16((B, T, Hkv, D), 65)
    pos = torch.tensor([5, 60, 20000], dtype=torch.int32)
    kg, vg = kc.cuda(), vc.cuda()
    swa.swa_cache_append(kn.cuda(), vn.cuda(), kg, vg, pos.cuda(), rope_theta=THETA)
    torch.cuda.synchronize()
    kr_exact = oracle_mod.rope(f64(kn), pos.numpy(), THETA)
    kref, vref = f64(kc), f64(vc)
    oracle_mod.cache_append(kref, vref, None, kr_exact, f64(vn), pos.numpy())
    got = f64(kg)
    assert (np.abs(got - kref) <= np.abs(kref) * 2.0 ** -8 + 1e-6).all()
    assert torch.equal(vg.cpu(), torch.from_numpy(vref).to(torch.bfloat16))   # values: plain copy


@pytest.mark.parametrize("B,N,Hq,Hkv,D,W", [(1, 700, 8, 2, 128, 256), (2, 300, 4, 4, 64, 64),
                                         (1, 400, 6, 2, 128, 100)])
def test_prefill_rope_fused_q(oracle_mod, B, N, Hq, Hkv, D, W):
    q = wl.random_bf16((B, N, Hq, D), 66)
    k = wl.random_bf16((B, N, Hkv, D), 67)
    v = wl.random_bf16((B, N, Hkv, D), 68)
    zero = torch.zeros(B, dtype=torch.int32)
    kg = k.cuda()
    swa.swa_rope(kg, zero.cuda(), THETA)
    out = swa.swa_prefill(q.cuda(), kg, v.cuda(), W, 1 / math.sqrt(D), rope_theta=THETA)
    torch.cuda.synchronize()
    qr = oracle_mod.rope(f64(q), zero.numpy(), THETA)
    kr = oracle_mod.rope(f64(k), zero.numpy(), THETA)
    ref = oracle_mod.swa_prefill(qr, kr, f64(v), W, 1 / math.sqrt(D))
    close(out, ref, "prefill rope")


@pytest.mark.parametrize("B,N,Hq,Hkv,D,W", [
    (1, 2304, 24, 8, 128, 600),      # groups of 3 in head pairs: 288 units, 70 blocks take a one-head unit first
    (1, 1300, 56, 8, 128, 700),      # groups of 7 in query-block pairs: 56 blocks start on the one-block pair
    (1, 1280, 24, 8, 64, 300),       # groups of 3, 160 units: 6 blocks take a one-head unit, then a pair (D=64)
])
def test_prefill_rope_second_q_tile_absent_then_present(oracle_mod, B, N, Hq, Hkv, D, W):
    """Persistent blocks whose unit has no second Q tile (the last head of an
    odd group, or a last query-block pair with one block) and whose next unit
    has one: the warpgroup that rotates tile 1 waits for that tile's own load
    and rotates it exactly once."""
    seed = 6900 + N + Hq
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N, Hkv, D), seed + 2)
    scale = 1 / math.sqrt(D)
    zero = np.zeros(B, np.int32)
    for _ in range(2):
        out = swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), W, scale, rope_theta=THETA)
        torch.cuda.synchronize()
        ref = oracle_mod.swa_prefill(oracle_mod.rope(f64(q), zero, THETA), f64(k), f64(v), W, scale)
        close(out, ref, f"prefill rope G={Hq // Hkv} N{N}")


@pytest.mark.parametrize("B,N,C,Hq,Hkv,D,W", [
    (2, 520, 200, 8, 2, 128, 256),
    (1, 2560, 1280, 32, 4, 64, 1280),    # 160 units: the last wave split into single-head units, G=8, D=64
    (1, 2560, 1280, 24, 8, 128, 1280),   # groups of 3: blocks that take a one-head unit, then a pair
])
def test_chunked_rope_then_decode_rope_continue_the_sequence(oracle_mod, B, N, C, Hq, Hkv, D, W):
    """Chunks with q rotated at load and keys rotated before the chunk call,
    then decode with the key rotated into the cache and q rotated in the
    kernel: every output equals one-shot SWA on exactly rotated q and k."""
    q = wl.random_bf16((B, N + 2, Hq, D), 69)
    k = wl.random_bf16((B, N + 2, Hkv, D), 70)
    v = wl.random_bf16((B, N + 2, Hkv, D), 71)
    scale = 1 / math.sqrt(D)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for s0 in range(0, N, C):
        e = min(N, s0 + C)
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        kch = k[:, s0:e].cuda().contiguous()
        swa.swa_rope(kch, st, THETA)
        outs.append(swa.swa_prefill_chunk(q[:, s0:e].cuda().contiguous(), kch, v[:, s0:e].cuda().contiguous(),
                                          kc, vc, st, W, scale, rope_theta=THETA))
    dec = []
    for p in (N, N + 1):
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        swa.swa_cache_append(k[:, p:p + 1].cuda().contiguous(), v[:, p:p + 1].cuda().contiguous(), kc, vc, pos,
                             rope_theta=THETA)
        dec.append(swa.swa_decode(q[:, p].cuda().contiguous(), kc, vc, pos, scale, rope_theta=THETA))
    torch.cuda.synchronize()
    zero = np.zeros(B, np.int32)
    qr = oracle_mod.rope(f64(q), zero, THETA)
    kr = oracle_mod.rope(f64(k), zero, THETA)
    ref = oracle_mod.swa_prefill(qr, kr, f64(v), W, scale)
    close(torch.cat([o.cpu() for o in outs], dim=1), ref[:, :N], "chunked rope")
    for i, p in enumerate((N, N + 1)):
        close(dec[i].cpu(), ref[:, p], f"decode rope at {p}")
