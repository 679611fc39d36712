"""The README's usage example runs as written and its outputs agree with the
oracle (sampled rows of the one-shot prefill, the chunked prefill over the
same prompt, and the decode step)."""
import os
import re

import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu
ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_readme_example(oracle_mod):
    text = open(os.path.join(ROOT, "README.md")).read()
    code = re.search(r"```python\n(.*?)```", text, re.S).group(1)
    torch.manual_seed(0)
    env = {}
    exec(compile(code, "README.md", "exec"), env)
    torch.cuda.synchronize()
    f64 = lambda t: t.detach().float().cpu().numpy().astype(np.float64)
    q, k, v, W, D, N = env["q"], env["k"], env["v"], env["W"], env["D"], env["N"]
    scale = D ** -0.5
    rows = [0, 1, 127, W - 1, W, W + 1, N // 2, N - 1]
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale, rows=rows)
    err = np.abs(f64(env["out"][:, rows]) - ref)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
    # the cache holds the last W positions: N from the append, the rest from the prompt
    B = q.shape[0]
    kx = torch.cat([k.cpu(), env["k_new"].cpu()], dim=1)
    vx = torch.cat([v.cpu(), env["v_new"].cpu()], dim=1)
    last = [s + ((N - s) // W) * W for s in range(W)]
    kc_expect, vc_expect = kx[:, last].contiguous(), vx[:, last].contiguous()
    assert torch.equal(env["k_cache"].cpu(), kc_expect) and torch.equal(env["v_cache"].cpu(), vc_expect)
    pos = np.full(B, N, np.int32)
    sp = oracle_mod.slot_positions(pos + 1, W)
    ref_o = oracle_mod.swa_decode(f64(env["q_new"]), f64(kc_expect), f64(vc_expect), sp, pos, W, scale)
    err = np.abs(f64(env["o"]) - ref_o)
    assert err.max() <= 2e-2 and err.mean() <= 2e-3, (err.max(), err.mean())
