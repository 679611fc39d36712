"""swa_decode_noalloc: decode for callers that cannot give the library scratch
memory (a plug-in whose host application owns all device memory, a serving
loop that cannot afford cudaMalloc's device-wide synchronisation, a caller
with a budget fixed at start-up).  It keeps its split partials in a scratch
array the library reserves statically per GPU, so it allocates nothing.

Checked through the C ABI against swa_decode (caller workspace) on two calls
in a row with different inputs, so stale contents left in the shared scratch
by the first call would show up in the second.  This file is collected last;
it also passes alone in a fresh process (the first call does the one-time
scratch address lookup).
"""
import ctypes
import math

import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


def _inputs(B, Hq, Hkv, D, W, seed):
    kc = wl.random_bf16((B, W, Hkv, D), seed).cuda()
    vc = wl.random_bf16((B, W, Hkv, D), seed + 1).cuda()
    q = wl.random_bf16((B, Hq, D), seed + 2).cuda()
    pos = wl.random_positions(B, 0, 3 * W, seed + 3).cuda()
    return q, kc, vc, pos


def test_noalloc_decode_matches_workspace_decode_twice():
    assert torch.cuda.is_available()
    swa.build()
    L = swa.lib()
    # W = 8192: 8 splits of 1024 keys per sequence, merged through the scratch
    B, Hq, Hkv, D, W = 16, 32, 8, 128, 8192
    assert swa.swa_decode_workspace_size(B, Hq, Hkv, D, W) > 0
    scale = 1.0 / math.sqrt(D)
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    for call, seed in enumerate((101, 202)):
        q, kc, vc, pos = _inputs(B, Hq, Hkv, D, W, seed)
        out_ref = torch.empty_like(q)
        out_new = torch.full_like(q, float("nan"))
        ws = torch.empty(swa.swa_decode_workspace_size(B, Hq, Hkv, D, W), dtype=torch.uint8, device="cuda")
        st = L.swa_decode(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), pos.data_ptr(), out_ref.data_ptr(),
                          B, Hq, Hkv, D, W, scale, ws.data_ptr(), ws.numel(), stream)
        assert st == swa.SWA_OK
        st = L.swa_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), pos.data_ptr(),
                                  out_new.data_ptr(), B, Hq, Hkv, D, W, scale, stream)
        assert st == swa.SWA_OK, f"call {call}: status {st}"
        torch.cuda.synchronize()
        # the same kernels on the same inputs: the same bits, whatever the
        # previous call left in the shared scratch
        assert torch.equal(out_new, out_ref), f"call {call}: differs from swa_decode"
        a = out_new.float().cpu().numpy()
        b = out_ref.float().cpu().numpy()
        assert np.isfinite(a).all(), f"call {call}: non-finite output"
        err = np.abs(a - b)
        assert err.max() <= MAX_ABS and err.mean() <= MEAN_ABS, (call, err.max(), err.mean())
    assert swa.swa_get_device_status() == swa.SWA_OK


def test_noalloc_rejects_sizes_beyond_its_scratch():
    swa.build()
    L = swa.lib()
    B, Hq, Hkv, D, W = 256, 32, 8, 128, 8192          # needs ~34 MB of partials
    assert swa.swa_decode_workspace_size(B, Hq, Hkv, D, W) > (16 << 20)
    st = L.swa_decode_noalloc(0x1000, 0x1000, 0x1000, 0x1000, 0x1000, B, Hq, Hkv, D, W, 0.1, None)
    assert st == swa.SWA_ERR_UNSUPPORTED


def test_noalloc_python_binding_matches_the_c_call():
    """The Python binding passes its arguments through unchanged: same bits as
    the raw C call on the same inputs."""
    swa.build()
    L = swa.lib()
    B, Hq, Hkv, D, W = 8, 32, 8, 128, 4096
    scale = 1.0 / math.sqrt(D)
    q, kc, vc, pos = _inputs(B, Hq, Hkv, D, W, 303)
    a = torch.empty_like(q)
    b = swa.swa_decode_noalloc(q, kc, vc, pos, scale, torch.empty_like(q))
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    st = L.swa_decode_noalloc(q.data_ptr(), kc.data_ptr(), vc.data_ptr(), pos.data_ptr(), a.data_ptr(),
                              B, Hq, Hkv, D, W, scale, stream)
    assert st == swa.SWA_OK
    torch.cuda.synchronize()
    assert torch.equal(a, b)
