"""Seeded synthetic workloads shaped like Mistral-7B attention (Table 1 of the
Mistral 7B paper: 32 query heads, 8 KV heads, head_dim 128, window 4096).

This module only draws random inputs and describes workload shapes.  It holds
none of the attention or rolling-buffer arithmetic: both the CUDA path and
the CPU oracle take their inputs from here and compute independently.

Every tensor is drawn on the CPU from ``torch.Generator().manual_seed(seed)``
as float32 N(0, 1) and, unless a workload says otherwise, rounded to bfloat16
(round-to-nearest-even, by torch's dtype conversion).
"""
from __future__ import annotations

import dataclasses
import math

import torch


@dataclasses.dataclass(frozen=True)
class Prefill:
    """One-shot prefill workload: q [B,N,Hq,D], k/v [B,N,Hkv,D]."""
    name: str
    B: int
    N: int
    W: int
    Hq: int
    Hkv: int
    D: int
    seed: int
    fp32_inputs: bool = False       # draw stays float32 (the kernels take bf16)
    outlier_frac: float = 0.0       # fraction of (b, n, kv-head) key rows scaled
    outlier_scale: float = 1.0

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


@dataclasses.dataclass(frozen=True)
class Chunked:
    """A prompt of N tokens pre-filled in chunks of C through a W-slot cache."""
    name: str
    B: int
    N: int
    C: int
    W: int
    Hq: int
    Hkv: int
    D: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


@dataclasses.dataclass(frozen=True)
class Decode:
    """Batched single-token decode against a full W-slot rolling cache."""
    name: str
    B: int
    W: int
    Hq: int
    Hkv: int
    D: int
    steps: int
    max_pos: int
    seed: int

    @property
    def scale(self) -> float:
        return 1.0 / math.sqrt(self.D)


# The workloads, named by what they are.
TINY = Prefill("tiny_prefill_B1_N256_W64_H4x2_D64", B=1, N=256, W=64, Hq=4, Hkv=2, D=64,
               seed=1001, fp32_inputs=True)
MISTRAL_PREFILL_8K = Prefill("mistral_prefill_B1_N8192_W4096", B=1, N=8192, W=4096, Hq=32, Hkv=8,
                             D=128, seed=1002)
CHUNKED_16K = Chunked("mistral_chunked_B1_N16384_C4096_W4096", B=1, N=16384, C=4096, W=4096,
                      Hq=32, Hkv=8, D=128, seed=1003)
DECODE_B64 = Decode("mistral_decode_B64_W4096_128steps", B=64, W=4096, Hq=32, Hkv=8, D=128,
                    steps=128, max_pos=32768, seed=1004)


def sweep_point(N: int, W: int) -> Prefill:
    """Long-prefill sweep point: B=2, bf16, 1% of key rows scaled by 8."""
    return Prefill(f"mistral_prefill_B2_N{N}_W{W}", B=2, N=N, W=W, Hq=32, Hkv=8, D=128,
                   seed=1005, outlier_frac=0.01, outlier_scale=8.0)


SWEEP_N = (4096, 8192, 16384, 32768)
SWEEP_W = (1024, 4096)
# The headline prefill workload: B=2, N=16384, W=4096.
HEADLINE_PREFILL = sweep_point(16384, 4096)


def _draw(gen: torch.Generator, shape, fp32: bool) -> torch.Tensor:
    x = torch.randn(*shape, generator=gen, dtype=torch.float32)
    return x if fp32 else x.to(torch.bfloat16)


def prefill_inputs(w: Prefill):
    """Return CPU tensors (q, k, v) for a prefill workload."""
    g = torch.Generator().manual_seed(w.seed)
    q = torch.randn(w.B, w.N, w.Hq, w.D, generator=g, dtype=torch.float32)
    k = torch.randn(w.B, w.N, w.Hkv, w.D, generator=g, dtype=torch.float32)
    v = torch.randn(w.B, w.N, w.Hkv, w.D, generator=g, dtype=torch.float32)
    if w.outlier_frac > 0.0:
        rows = w.B * w.N * w.Hkv
        n_out = max(1, int(round(rows * w.outlier_frac)))
        idx = torch.randperm(rows, generator=g)[:n_out]
        kf = k.view(rows, w.D)
        kf[idx] *= w.outlier_scale
    if not w.fp32_inputs:
        q, k, v = q.to(torch.bfloat16), k.to(torch.bfloat16), v.to(torch.bfloat16)
    return q, k, v


def chunked_inputs(w: Chunked):
    """Return CPU bf16 tensors (q, k, v) of the whole N-token prompt."""
    g = torch.Generator().manual_seed(w.seed)
    q = _draw(g, (w.B, w.N, w.Hq, w.D), False)
    k = _draw(g, (w.B, w.N, w.Hkv, w.D), False)
    v = _draw(g, (w.B, w.N, w.Hkv, w.D), False)
    return q, k, v


def decode_inputs(w: Decode):
    """Return a dict of CPU tensors for a decode workload.

    pos0      int32 [B]        position of each sequence's first new token,
                               uniform on [1, max_pos]
    k_cache   bf16 [B,W,Hkv,D] random initial cache contents (every slot drawn)
    v_cache   bf16 [B,W,Hkv,D]
    q         bf16 [steps,B,Hq,D]   per-step new queries
    k_new     bf16 [steps,B,Hkv,D]  per-step new keys
    v_new     bf16 [steps,B,Hkv,D]
    """
    g = torch.Generator().manual_seed(w.seed)
    pos0 = torch.randint(1, w.max_pos + 1, (w.B,), generator=g, dtype=torch.int64).to(torch.int32)
    k_cache = _draw(g, (w.B, w.W, w.Hkv, w.D), False)
    v_cache = _draw(g, (w.B, w.W, w.Hkv, w.D), False)
    q = _draw(g, (w.steps, w.B, w.Hq, w.D), False)
    k_new = _draw(g, (w.steps, w.B, w.Hkv, w.D), False)
    v_new = _draw(g, (w.steps, w.B, w.Hkv, w.D), False)
    return dict(pos0=pos0, k_cache=k_cache, v_cache=v_cache, q=q, k_new=k_new, v_new=v_new)


def random_bf16(shape, seed: int, scale: float = 1.0) -> torch.Tensor:
    """Generic seeded N(0, scale^2) bf16 CPU tensor (edge-case tests)."""
    g = torch.Generator().manual_seed(seed)
    return (torch.randn(*shape, generator=g, dtype=torch.float32) * scale).to(torch.bfloat16)


def random_positions(n: int, lo: int, hi: int, seed: int) -> torch.Tensor:
    """Seeded int32 positions uniform on [lo, hi]."""
    g = torch.Generator().manual_seed(seed)
    return torch.randint(lo, hi + 1, (n,), generator=g, dtype=torch.int64).to(torch.int32)


def useful_pairs(N: int, W: int) -> int:
    """Number of (query, key) pairs inside a causal window of W keys, per head.

    Counting only: sum over i of min(i+1, W).  Used for FLOP accounting."""
    full = max(0, N - W)
    ramp = min(N, W)
    return ramp * (ramp + 1) // 2 + full * W


def useful_flops(B: int, N: int, W: int, Hq: int, D: int) -> int:
    """Useful (unmasked) FLOPs of prefill: QK^T and PV, 2*D each per pair."""
    return 4 * B * Hq * D * useful_pairs(N, W)
