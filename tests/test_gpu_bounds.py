"""The index-checked build (libswa_debug.so, compiled with SWA_BOUNDS_CHECK).

Its kernels check every global row, cache slot, sink slot, output row and TMA
start coordinate they compute against the extent of the tensor it indexes; a
failed check records SWA_ERR_INVALID_ARG and skips the access, with no trap.
Every entry point is run here on small edge-case shapes (ragged lengths,
windows off tile edges, odd head groups, D = 64 and 128, wrapped buffers,
split decode, sinks, rotary embedding, packed batches): no check may fire,
and the outputs and caches must equal, bit for bit, those of the normal
library on the same inputs (the checks change no arithmetic).
"""
import math

import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module", autouse=True)
def _libs():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    swa.build()
    swa.build(debug=True)
    swa.lib()
    with swa.bounds_checked():
        swa.lib()
        assert swa.swa_get_device_status() == swa.SWA_OK
    yield


def _both(fn):
    """fn() with the normal library, then with the index-checked one; the
    debug run must record no failed check.  Returns both results."""
    a = fn()
    torch.cuda.synchronize()
    assert swa.swa_get_device_status() == swa.SWA_OK
    with swa.bounds_checked():
        b = fn()
        torch.cuda.synchronize()
        assert swa.swa_get_device_status() == swa.SWA_OK, "an index check failed"
    return a, b


def _equal(a, b):
    if isinstance(a, (list, tuple)):
        assert len(a) == len(b)
        for x, y in zip(a, b):
            _equal(x, y)
    else:
        assert torch.equal(a, b)


def _r(shape, seed, scale=1.0):
    return wl.random_bf16(shape, seed, scale).cuda()


@pytest.mark.parametrize("B,N,Hq,Hkv,D,W,mode", [
    (1, 128, 2, 1, 128, 128, 0), (1, 300, 4, 2, 128, 64, 0), (2, 517, 8, 2, 128, 200, 0),
    (1, 640, 4, 4, 64, 1, 0), (1, 384, 6, 2, 64, 3, 0), (1, 450, 8, 1, 128, 1000, 0),
    (1, 257, 2, 2, 64, 129, 0), (1, 400, 4, 2, 128, 100, 1),
])
def test_prefill(B, N, Hq, Hkv, D, W, mode):
    q, k, v = _r((B, N, Hq, D), 1), _r((B, N, Hkv, D), 2), _r((B, N, Hkv, D), 3)
    _equal(*_both(lambda: swa.swa_prefill(q, k, v, W, 1 / math.sqrt(D), window_mode=mode)))


def test_prefill_sinks_and_rope():
    q, k, v = _r((2, 333, 8, 2 * 64), 4), _r((2, 333, 2, 128), 5), _r((2, 333, 2, 128), 6)
    _equal(*_both(lambda: swa.swa_prefill_sinks(q, k, v, 100, 4, 0.09)))
    _equal(*_both(lambda: swa.swa_prefill(q, k, v, 100, 0.09, rope_theta=10000.0)))


@pytest.mark.parametrize("B,N,C,Hq,Hkv,D,W", [
    (1, 512, 128, 4, 2, 128, 128), (2, 700, 96, 4, 2, 128, 256), (1, 600, 200, 8, 2, 64, 200),
    (1, 333, 45, 2, 1, 128, 100), (1, 1100, 300, 6, 2, 128, 384), (2, 2560, 1280, 16, 4, 128, 1536),
])
def test_chunked_prefill(B, N, C, Hq, Hkv, D, W):
    q, k, v = _r((B, N, Hq, D), 7), _r((B, N, Hkv, D), 8), _r((B, N, Hkv, D), 9)

    def run(sinks):
        kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
        vc = torch.zeros_like(kc)
        ks = torch.zeros(B, 4, Hkv, D, dtype=torch.bfloat16, device="cuda")
        vs = torch.zeros_like(ks)
        outs = []
        for s0 in range(0, N, C):
            e = min(N, s0 + C)
            st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
            a, b_, c = (t[:, s0:e].contiguous() for t in (q, k, v))
            if sinks:
                outs.append(swa.swa_prefill_chunk_sinks(a, b_, c, kc, vc, ks, vs, st, W, 0.1))
            else:
                outs.append(swa.swa_prefill_chunk(a, b_, c, kc, vc, st, W, 0.1))
        return outs + [kc, vc, ks, vs]

    _equal(*_both(lambda: run(False)))
    if C <= W and B * N < 4000:
        _equal(*_both(lambda: run(True)))


def test_packed_batches():
    lens = [0, 1, 130, 257, 1, 600]
    cu = torch.tensor([0] + [sum(lens[:i + 1]) for i in range(len(lens))], dtype=torch.int32, device="cuda")
    total = int(cu[-1])
    Hq, Hkv, D, W = 8, 2, 128, 256
    q, k, v = _r((total, Hq, D), 10), _r((total, Hkv, D), 11), _r((total, Hkv, D), 12)
    _equal(*_both(lambda: swa.swa_prefill_varlen(q, k, v, cu, W, 0.1)))
    B = len(lens)
    start = wl.random_positions(B, 0, 3 * W, 13).cuda()

    def chunk():
        kc = _r((B, W, Hkv, D), 14)
        vc = _r((B, W, Hkv, D), 15)
        o = swa.swa_prefill_chunk_varlen(q, k, v, kc, vc, start, cu, W, 0.1)
        return [o, kc, vc]

    _equal(*_both(chunk))


@pytest.mark.parametrize("B,Hq,Hkv,D,W,pos0", [
    (4, 32, 8, 128, 4096, [0, 1, 4094, 4095]), (3, 8, 2, 128, 4096, [4096, 8191, 30000]),
    (2, 4, 4, 64, 700, [10, 2000]), (2, 16, 2, 128, 1000, [999, 5]), (2, 4, 2, 64, 300, [299, 77]),
    (2, 8, 2, 128, 8192, [8191, 20000]), (1, 4, 1, 64, 5000, [4999]),
    (8, 32, 8, 128, 4096, [0, 1, 17, 63, 64, 4095, 4096, 9000]),   # 4 splits per window: merged in a cluster
])
def test_append_and_decode(B, Hq, Hkv, D, W, pos0):
    pos = torch.tensor(pos0, dtype=torch.int32, device="cuda")
    q = _r((B, Hq, D), 16)
    kn, vn = _r((B, 1, Hkv, D), 17), _r((B, 1, Hkv, D), 18)

    def run():
        kc, vc = _r((B, W, Hkv, D), 19), _r((B, W, Hkv, D), 20)
        ks, vs = _r((B, 4, Hkv, D), 21), _r((B, 4, Hkv, D), 22)
        swa.swa_cache_append(kn, vn, kc, vc, pos)
        o1 = swa.swa_decode(q, kc, vc, pos, 0.1)
        o2 = swa.swa_decode(q, kc, vc, pos, 0.1, rope_theta=10000.0)
        swa.swa_cache_append_sinks(kn, vn, kc, vc, ks, vs, pos)
        o3 = swa.swa_decode_sinks(q, kc, vc, ks, vs, pos, 0.1)
        swa.swa_cache_append(kn, vn, kc, vc, pos, rope_theta=10000.0)
        return [o1, o2, o3, kc, vc, ks, vs]

    _equal(*_both(run))
