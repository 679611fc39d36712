"""Checkpoint and resume of a sequence through its rolling buffer.

The rolling buffer (W slots, slot = position mod W) plus the next position is
the whole state a sequence carries from pre-fill into decode ("Pre-fill과의
상호작용" of the "Mistral 7B -- Sliding Window Attention" summary: decoding
continues from the buffer the pre-fill left).  Here a prompt is pre-filled in
four chunks; after chunk 1 the buffers and the next position are copied to the
host and saved; a fresh process (nothing shared but that file and the seeds
of the inputs) restores them, pre-fills chunks 2-3 and decodes 8 tokens.  Its
outputs and final buffers equal, bit for bit, those of the same work run
without interruption, and they match the fp64 oracle.
"""
import math
import os
import subprocess
import sys

import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
B, C, NCHUNK, Hq, Hkv, D, W, DEC = 2, 256, 4, 8, 2, 128, 512, 8
N = C * NCHUNK
SEED = 4242


def _inputs():
    """The prompt and the decoded tokens: positions 0 .. N+DEC-1."""
    q = wl.random_bf16((B, N + DEC, Hq, D), SEED)
    k = wl.random_bf16((B, N + DEC, Hkv, D), SEED + 1)
    v = wl.random_bf16((B, N + DEC, Hkv, D), SEED + 2)
    return q, k, v


def _run(q, k, v, kc, vc, chunks, decode_steps):
    """Pre-fill the given chunks, then decode_steps tokens after the prompt;
    returns the chunk outputs and the decode outputs (on the host)."""
    scale = 1.0 / math.sqrt(D)
    outs, decs = [], []
    for c in chunks:
        s0 = c * C
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        outs.append(swa.swa_prefill_chunk(q[:, s0:s0 + C].contiguous(), k[:, s0:s0 + C].contiguous(),
                                          v[:, s0:s0 + C].contiguous(), kc, vc, st, W, scale).cpu())
    for t in range(decode_steps):
        p = N + t
        pos = torch.full((B,), p, dtype=torch.int32, device="cuda")
        swa.swa_cache_append(k[:, p:p + 1].contiguous(), v[:, p:p + 1].contiguous(), kc, vc, pos)
        decs.append(swa.swa_decode(q[:, p].contiguous(), kc, vc, pos, scale).cpu())
    torch.cuda.synchronize()
    return outs, decs


_CHILD = r"""
import sys, torch
sys.path.insert(0, sys.argv[1])
import test_gpu_resume as t
import sliding_window_gqa_prefill_b200 as swa
swa.build()
ck = torch.load(sys.argv[2])
assert ck["next_pos"] == 2 * t.C
q, k, v = (x.cuda() for x in t._inputs())
kc, vc = ck["k_cache"].cuda(), ck["v_cache"].cuda()
outs, decs = t._run(q, k, v, kc, vc, [2, 3], t.DEC)
assert swa.swa_get_device_status() == swa.SWA_OK
torch.save({"outs": outs, "decs": decs, "k_cache": kc.cpu(), "v_cache": vc.cpu()}, sys.argv[3])
"""


def test_resume_in_a_fresh_process_is_bit_identical(oracle_mod, tmp_path):
    swa.build()
    q, k, v = (x.cuda() for x in _inputs())
    # uninterrupted
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs, decs = _run(q, k, v, kc, vc, range(NCHUNK), DEC)
    # interrupted after chunk 1: buffers and next position to the host, saved
    kc2 = torch.zeros_like(kc)
    vc2 = torch.zeros_like(kc)
    outs01, _ = _run(q, k, v, kc2, vc2, [0, 1], 0)
    ckpt = tmp_path / "ckpt.pt"
    torch.save({"k_cache": kc2.cpu(), "v_cache": vc2.cpu(), "next_pos": 2 * C}, ckpt)
    del kc2, vc2
    res = tmp_path / "resumed.pt"
    env = dict(os.environ, PYTHONPATH=os.pathsep.join([ROOT, os.environ.get("PYTHONPATH", "")]))
    r = subprocess.run([sys.executable, "-c", _CHILD, os.path.join(ROOT, "tests"), str(ckpt), str(res)],
                       capture_output=True, text=True, timeout=600, env=env, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-3000:]
    got = torch.load(res)
    for a, b in zip(outs01, outs[:2]):
        assert torch.equal(a, b)
    for i, (a, b) in enumerate(zip(got["outs"], outs[2:])):
        assert torch.equal(a, b), f"chunk {2 + i}"
    for i, (a, b) in enumerate(zip(got["decs"], decs)):
        assert torch.equal(a, b), f"decode step {i}"
    assert torch.equal(got["k_cache"], kc.cpu()) and torch.equal(got["v_cache"], vc.cpu())
    # and the resumed run is right: rows of one-shot SWA over the whole sequence
    f64 = lambda t: t.float().cpu().numpy().astype(np.float64)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, 1.0 / math.sqrt(D))
    gpu = np.concatenate([f64(o) for o in got["outs"]] + [f64(d).reshape(B, 1, Hq, D) for d in got["decs"]], 1)
    err = np.abs(gpu - ref[:, 2 * C:])
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
