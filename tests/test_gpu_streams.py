"""Determinism, and calls on several CUDA streams at once, as a serving
process issues them: every kernel is deterministic, so repeated calls and
work that overlaps on the GPU must give the same bits as the same calls run
one after another.

Two independent sequence sets, each with its own buffers and workspace:
set A pre-fills in chunks and decodes on stream 1, set B takes a mixed packed
call (chunks and decode tokens, the decode kernel's cluster mode) and a
one-shot prefill on stream 2; the streams are not ordered against each other.
"""
import math

import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available()
    swa.build()
    swa.lib()
    yield
    assert swa.swa_get_device_status() == swa.SWA_OK


def _set_a(seed):
    B, N, C, Hq, Hkv, D, W = 2, 1536, 512, 16, 4, 128, 512
    t = {"q": wl.random_bf16((B, N + 2, Hq, D), seed).cuda(), "k": wl.random_bf16((B, N + 2, Hkv, D), seed + 1).cuda(),
         "v": wl.random_bf16((B, N + 2, Hkv, D), seed + 2).cuda()}
    t["kc"] = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    t["vc"] = torch.zeros_like(t["kc"])
    t["ws"] = torch.empty(swa.swa_decode_workspace_size(B, Hq, Hkv, D, W), dtype=torch.uint8, device="cuda")
    t["outs"] = [torch.empty(B, C, Hq, D, dtype=torch.bfloat16, device="cuda") for _ in range(N // C)]
    t["dec"] = torch.empty(2, B, Hq, D, dtype=torch.bfloat16, device="cuda")
    t["st"] = [torch.full((B,), s0, dtype=torch.int32, device="cuda") for s0 in range(0, N, C)]
    t["pos"] = [torch.full((B,), p, dtype=torch.int32, device="cuda") for p in (N, N + 1)]
    t["shape"] = (B, N, C, Hq, Hkv, D, W)
    return t


def _run_a(t, stream):
    B, N, C, Hq, Hkv, D, W = t["shape"]
    scale = 1 / math.sqrt(D)
    with torch.cuda.stream(stream):
        for i, s0 in enumerate(range(0, N, C)):
            swa.swa_prefill_chunk(t["q"][:, s0:s0 + C].contiguous(), t["k"][:, s0:s0 + C].contiguous(),
                                  t["v"][:, s0:s0 + C].contiguous(), t["kc"], t["vc"], t["st"][i], W, scale,
                                  out=t["outs"][i])
        for j, p in enumerate((N, N + 1)):
            swa.swa_cache_append(t["k"][:, p:p + 1].contiguous(), t["v"][:, p:p + 1].contiguous(), t["kc"], t["vc"],
                                 t["pos"][j])
            swa.swa_decode(t["q"][:, p].contiguous(), t["kc"], t["vc"], t["pos"][j], scale, out=t["dec"][j],
                           workspace=t["ws"])


def _set_b(seed):
    Hq, Hkv, D, W = 8, 2, 128, 1024
    lens = [700, 1, 1, 0, 300, 1]
    hist = [2000, 5000, 3, 0, 90, 1023]
    total = sum(lens)
    t = {"q": wl.random_bf16((total, Hq, D), seed).cuda(), "k": wl.random_bf16((total, Hkv, D), seed + 1).cuda(),
         "v": wl.random_bf16((total, Hkv, D), seed + 2).cuda(),
         "kc": wl.random_bf16((len(lens), W, Hkv, D), seed + 3).cuda(),
         "vc": wl.random_bf16((len(lens), W, Hkv, D), seed + 4).cuda(),
         "cu": torch.tensor([0] + [sum(lens[:i + 1]) for i in range(len(lens))], dtype=torch.int32, device="cuda"),
         "start": torch.tensor(hist, dtype=torch.int32, device="cuda"),
         "pq": wl.random_bf16((1, 3000, 32, D), seed + 5).cuda(), "pk": wl.random_bf16((1, 3000, 8, D), seed + 6).cuda(),
         "pv": wl.random_bf16((1, 3000, 8, D), seed + 7).cuda()}
    t["out"] = torch.empty_like(t["q"])
    t["pout"] = torch.empty_like(t["pq"])
    t["W"] = W
    return t


def _run_b(t, stream):
    with torch.cuda.stream(stream):
        swa.swa_prefill_chunk_varlen(t["q"], t["k"], t["v"], t["kc"], t["vc"], t["start"], t["cu"], t["W"], 0.088,
                                     out=t["out"])
        swa.swa_prefill(t["pq"], t["pk"], t["pv"], 1024, 0.088, out=t["pout"])


def _snapshot(a, b):
    return [x.clone() for x in a["outs"]] + [a["dec"].clone(), a["kc"].clone(), a["vc"].clone(),
                                            b["out"].clone(), b["pout"].clone(), b["kc"].clone(), b["vc"].clone()]


def test_overlapping_streams_give_the_sequential_bits():
    s1, s2 = torch.cuda.Stream(), torch.cuda.Stream()
    a, b = _set_a(7100), _set_b(7200)
    kc_b0, vc_b0 = b["kc"].clone(), b["vc"].clone()
    torch.cuda.synchronize()                # inputs were copied on the default stream
    # one after the other
    _run_a(a, s1)
    s1.synchronize()
    _run_b(b, s2)
    s2.synchronize()
    ref = _snapshot(a, b)
    # again, both streams at once (fresh buffers, nothing ordering them)
    a2, b2 = _set_a(7100), _set_b(7200)
    b2["kc"].copy_(kc_b0)
    b2["vc"].copy_(vc_b0)
    torch.cuda.synchronize()
    for _ in range(3):                      # interleave the issue order too
        _run_b(b2, s2)
        _run_a(a2, s1)
        torch.cuda.synchronize()
        got = _snapshot(a2, b2)
        for x, y in zip(got, ref):
            assert torch.equal(x, y)
        a2, b2 = _set_a(7100), _set_b(7200)
        b2["kc"].copy_(kc_b0)
        b2["vc"].copy_(vc_b0)
        torch.cuda.synchronize()
    assert swa.swa_get_device_status() == swa.SWA_OK


def test_repeated_calls_are_bit_identical():
    """Every entry point is deterministic: the same inputs give the same bits
    on every call (the persistent prefill's schedule is static, the split
    merge has a fixed order), so results reproduce exactly."""
    B, N, Hq, Hkv, D, W = 2, 2000, 32, 8, 128, 1024
    q, k, v = (wl.random_bf16((B, N, h, D), 7300 + i).cuda() for i, h in enumerate((Hq, Hkv, Hkv)))
    first = swa.swa_prefill(q, k, v, W, 0.088)
    kc = wl.random_bf16((B, W, Hkv, D), 7310).cuda()
    vc = wl.random_bf16((B, W, Hkv, D), 7311).cuda()
    pos = torch.tensor([5000, 900], dtype=torch.int32, device="cuda")
    dec0 = swa.swa_decode(q[:, 0].contiguous(), kc, vc, pos, 0.088)
    kc2, vc2 = kc.clone(), vc.clone()
    st = torch.tensor([3000, 10], dtype=torch.int32, device="cuda")
    ch0 = swa.swa_prefill_chunk(q[:, :W].contiguous(), k[:, :W].contiguous(), v[:, :W].contiguous(), kc2, vc2, st,
                                W, 0.088)
    for _ in range(3):
        assert torch.equal(swa.swa_prefill(q, k, v, W, 0.088), first)
        assert torch.equal(swa.swa_decode(q[:, 0].contiguous(), kc, vc, pos, 0.088), dec0)
        kc3, vc3 = kc.clone(), vc.clone()
        ch = swa.swa_prefill_chunk(q[:, :W].contiguous(), k[:, :W].contiguous(), v[:, :W].contiguous(), kc3, vc3,
                                   st, W, 0.088)
        assert torch.equal(ch, ch0) and torch.equal(kc3, kc2) and torch.equal(vc3, vc2)
