"""Receptive field of stacked sliding-window layers.

The pages: a token at layer k reaches k*W positions back through the stack
("Mistral 7B -- Sliding Window Attention" summary, section "Methods"; the
receptive-field simulator of "Mistral 7B: Engineering Extreme Efficiency in
LLMs", section 2, prints a span of 9 tokens for W = 3 and 3 layers, formula
Span = L x W).  With identity projections (q = k = v = the layer input) a
stack of L SWA layers is run on a sequence; one input position j is perturbed;
exactly the outputs at positions j .. j + L*lookback change, where lookback is
W under the i-W <= j <= i reading (the simulator's) and W-1 under the adopted
i-W < j <= i reading.  On the GPU every layer is also compared with the oracle
run on that layer's input.
"""
import numpy as np
import pytest
import torch

from sliding_window_gqa_prefill_b200 import workloads as wl


def _stack_oracle(oracle_mod, x, W, L, mode, scale=None):
    for _ in range(L):
        x = oracle_mod.swa_prefill(x, x, x, W, 1.0 / np.sqrt(x.shape[-1]) if scale is None else scale, mode=mode)
    return x


def _changed_positions(a, b):
    return sorted(set(np.nonzero(np.abs(a - b).reshape(a.shape[0], a.shape[1], -1).max(axis=(0, 2)) > 0)[0].tolist()))


@pytest.mark.parametrize("W,L,mode,span", [(3, 3, 1, 9), (3, 3, 0, 6), (5, 2, 0, 8), (4, 1, 1, 4)])
def test_oracle_stack_reach(oracle_mod, W, L, mode, span):
    """W=3, L=3 under the simulator's reading reaches exactly 9 positions back."""
    rng = np.random.default_rng(W * 10 + L)
    N, D, j = 40, 8, 11
    x = rng.standard_normal((1, N, 1, D))
    y = x.copy()
    y[0, j] += 5.0 * rng.standard_normal(D)
    a = _stack_oracle(oracle_mod, x, W, L, mode)
    b = _stack_oracle(oracle_mod, y, W, L, mode)
    assert _changed_positions(a, b) == list(range(j, j + span + 1))


def _gpu_stack(swa, t, W, L, mode, scale):
    """Run L layers on the GPU; return every layer's bf16 input and the output."""
    layers = [t]
    for _ in range(L):
        t = swa.swa_prefill(t, t, t, W, scale, window_mode=mode)
        layers.append(t)
    torch.cuda.synchronize()
    return layers


def _f64(t):
    return t.float().cpu().numpy().astype(np.float64)


@pytest.mark.gpu
@pytest.mark.parametrize("W,L,mode,span", [(3, 3, 1, 9), (3, 3, 0, 6), (5, 2, 0, 8), (130, 2, 0, 258)])
def test_gpu_stack_against_oracle(oracle_mod, W, L, mode, span):
    """The CUDA prefill stacked L times (bf16 between layers, identity
    projections): every layer equals the oracle run on that layer's bf16
    input (max-abs 2e-2, mean-abs 2e-3 on the unperturbed stack; scaled by
    the magnitude on the perturbed one), and the positions a perturbed input
    moves are exactly those the oracle's fp64 stack moves on the same inputs.
    For W = 3 and 5 every move survives bf16, so the set is compared whole: a
    window one key narrower or wider changes the reach by L positions and
    fails.  For W = 130 the farthest moves are below bf16 resolution, so the
    check is that nothing outside the reach moves and every move the oracle
    finds above 0.05 shows.  A small softmax scale (0.02) keeps the weights
    within a window comparable, so a move survives several layers instead of
    being swamped by each query's own key (q = k = v)."""
    import sliding_window_gqa_prefill_b200 as swa
    assert torch.cuda.is_available()
    swa.build()
    N, H, D, j = 600, 2, 64, 37
    x = wl.random_bf16((1, N, H, D), 77).cuda()
    y = x.clone()
    y[0, j] = (wl.random_bf16((H, D), 78) * 10).cuda()
    scale = 0.02
    lx, ly = _gpu_stack(swa, x, W, L, mode, scale), _gpu_stack(swa, y, W, L, mode, scale)
    for layers, rel in ((lx, False), (ly, True)):
        for i in range(L):
            ref = oracle_mod.swa_prefill(_f64(layers[i]), _f64(layers[i]), _f64(layers[i]), W, scale,
                                         mode=mode)
            got = _f64(layers[i + 1])
            err = np.abs(got - ref) / (np.maximum(1.0, np.abs(ref)) if rel else 1.0)
            assert np.isfinite(got).all()
            assert err.max() <= 2e-2 and err.mean() <= 2e-3, (W, L, mode, i, err.max(), err.mean())
    gpu_changed = _changed_positions(_f64(lx[-1]), _f64(ly[-1]))
    a = _stack_oracle(oracle_mod, _f64(x), W, L, mode, scale)
    b = _stack_oracle(oracle_mod, _f64(y), W, L, mode, scale)
    assert _changed_positions(a, b) == list(range(j, j + span + 1))
    if W <= 5:
        assert gpu_changed == list(range(j, j + span + 1)), gpu_changed
    else:
        assert gpu_changed and gpu_changed[0] == j and gpu_changed[-1] <= j + span, gpu_changed[-3:]
        big = np.nonzero(np.abs(a - b).reshape(N, -1).max(axis=1) > 0.05)[0].tolist()
        assert set(big) <= set(gpu_changed), sorted(set(big) - set(gpu_changed))[:5]
