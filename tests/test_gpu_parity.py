"""Parity of the CUDA path (through the C ABI) with the fp64 CPU oracle.

Bar (from the method's accuracy target): bf16 outputs within max-abs 2e-2 and
mean-abs 2e-3 of the fp64 oracle run on the same bf16 inputs; rolling-buffer
cache contents bit-exact.  Small and edge cases compare every element; the
full-size workloads are in test_gpu_full_size.py.
"""
import math

import numpy as np
import pytest
import torch

import sliding_window_gqa_prefill_b200 as swa
from sliding_window_gqa_prefill_b200 import workloads as wl

pytestmark = pytest.mark.gpu

MAX_ABS = 2e-2
MEAN_ABS = 2e-3


@pytest.fixture(scope="module", autouse=True)
def _lib():
    assert torch.cuda.is_available(), "GPU tests need a CUDA device"
    swa.build()
    swa.lib()
    yield
    assert swa.swa_get_device_status() == swa.SWA_OK


def f64(t: torch.Tensor) -> np.ndarray:
    return t.detach().float().cpu().numpy().astype(np.float64)


def assert_close(gpu: torch.Tensor, ref: np.ndarray, what: str):
    got = f64(gpu)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert np.isfinite(got).all(), f"{what}: non-finite output"
    err = np.abs(got - ref)
    assert err.max() <= MAX_ABS, f"{what}: max-abs {err.max():.3e}"
    assert err.mean() <= MEAN_ABS, f"{what}: mean-abs {err.mean():.3e}"


def run_prefill(q, k, v, W, scale, mode=0):
    out = swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), W, scale, window_mode=mode)
    torch.cuda.synchronize()
    return out.cpu()


# ------------------------------------------------------------------ one-shot prefill

def test_tiny_workload_full(oracle_mod):
    """B=1, N=256, W=64, 4 query / 2 KV heads, D=64; fp32 draws rounded to bf16."""
    w = wl.TINY
    q, k, v = (t.to(torch.bfloat16) for t in wl.prefill_inputs(w))
    out = run_prefill(q, k, v, w.W, w.scale)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), w.W, w.scale)
    assert_close(out, ref, "tiny")
    # information only: distance to the oracle on the unrounded fp32 draws
    q32, k32, v32 = wl.prefill_inputs(w)
    ref32 = oracle_mod.swa_prefill(q32.numpy(), k32.numpy(), v32.numpy(), w.W, w.scale)
    print(f"tiny: max |gpu - oracle(fp32 inputs)| = {np.abs(f64(out) - ref32).max():.3e}")


CASES = [
    # B, N, Hq, Hkv, D, W
    (1, 128, 2, 1, 128, 128),      # one tile, dense
    (1, 300, 4, 2, 128, 64),       # ragged N, W < tile
    (2, 517, 8, 2, 128, 200),      # W not a multiple of 128, ragged tail, B=2
    (1, 640, 4, 4, 64, 1),         # W=1: output is v itself (MHA, D=64)
    (1, 384, 6, 2, 64, 3),         # group of 3 (odd: half-empty head pair)
    (1, 450, 8, 1, 128, 1000),     # W > N: dense causal, group 8
    (2, 1024, 8, 2, 128, 256),     # several full bands
    (1, 257, 2, 2, 64, 129),       # G=1, window one past a tile
]


@pytest.mark.parametrize("B,N,Hq,Hkv,D,W", CASES)
def test_prefill_edge_cases(oracle_mod, B, N, Hq, Hkv, D, W):
    seed = 7 * N + W
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    out = run_prefill(q, k, v, W, scale)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale)
    assert_close(out, ref, f"prefill B{B} N{N} H{Hq}/{Hkv} D{D} W{W}")


def test_prefill_inclusive_window_reading(oracle_mod):
    B, N, Hq, Hkv, D, W = 1, 400, 4, 2, 128, 100
    q = wl.random_bf16((B, N, Hq, D), 11)
    k = wl.random_bf16((B, N, Hkv, D), 12)
    v = wl.random_bf16((B, N, Hkv, D), 13)
    out = run_prefill(q, k, v, W, 0.1, mode=swa.SWA_WINDOW_INCL_LEFT)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, 0.1, mode=oracle_mod.WINDOW_INCL_LEFT)
    assert_close(out, ref, "inclusive window")


def test_prefill_large_logits_stable(oracle_mod):
    """Outlier keys (x8) and a large scale: the lazy-rescaled online softmax
    must stay finite and accurate."""
    B, N, Hq, Hkv, D, W = 1, 700, 4, 1, 128, 256
    q = wl.random_bf16((B, N, Hq, D), 21)
    k = wl.random_bf16((B, N, Hkv, D), 22)
    k[:, ::37] *= 8
    v = wl.random_bf16((B, N, Hkv, D), 23)
    out = run_prefill(q, k, v, W, 0.3)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, 0.3)
    assert_close(out, ref, "large logits")


def test_dense_control_equals_wide_window():
    """W >= N (dense causal control) gives the same bits for any W >= N."""
    B, N, Hq, Hkv, D = 2, 700, 8, 2, 128
    q = wl.random_bf16((B, N, Hq, D), 31)
    k = wl.random_bf16((B, N, Hkv, D), 32)
    v = wl.random_bf16((B, N, Hkv, D), 33)
    a = run_prefill(q, k, v, N, 0.09)
    b = run_prefill(q, k, v, 10 * N, 0.09)
    assert torch.equal(a, b)


@pytest.mark.parametrize("D", [64, 128])
def test_output_only_16_byte_aligned(D):
    """An output 16 but not 32 bytes aligned takes the 16-byte store path of the
    epilogue: same bits as a 32-byte aligned output, one-shot and chunked."""
    B, N, Hq, Hkv, W = 2, 300, 8, 2, 200
    q = wl.random_bf16((B, N, Hq, D), 41).cuda()
    k = wl.random_bf16((B, N, Hkv, D), 42).cuda()
    v = wl.random_bf16((B, N, Hkv, D), 43).cuda()
    n = B * N * Hq * D
    flat = torch.zeros(n + 16, dtype=torch.bfloat16, device="cuda")
    assert flat.data_ptr() % 32 == 0
    odd = flat[8:8 + n].view(B, N, Hq, D)            # 16 bytes past a 32-byte boundary
    ref = swa.swa_prefill(q, k, v, W, 0.1)
    swa.swa_prefill(q, k, v, W, 0.1, out=odd)
    torch.cuda.synchronize()
    assert torch.equal(odd, ref)
    assert not flat[:8].any() and not flat[8 + n:].any()
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    st = torch.zeros(B, dtype=torch.int32, device="cuda")
    ref_c = swa.swa_prefill_chunk(q[:, :150].contiguous(), k[:, :150].contiguous(), v[:, :150].contiguous(),
                                  kc.clone(), vc.clone(), st, W, 0.1)
    m = B * 150 * Hq * D
    odd_c = flat[8:8 + m].view(B, 150, Hq, D)
    swa.swa_prefill_chunk(q[:, :150].contiguous(), k[:, :150].contiguous(), v[:, :150].contiguous(),
                          kc, vc, st, W, 0.1, out=odd_c)
    torch.cuda.synchronize()
    assert torch.equal(odd_c, ref_c)


# ------------------------------------------------------------------ rolling buffer append

@pytest.mark.parametrize("B,T,Hkv,D,W", [(3, 1, 8, 128, 64), (2, 37, 2, 64, 50), (1, 64, 4, 128, 64),
                                         (4, 5, 8, 128, 4096)])
def test_cache_append_bit_exact(oracle_mod, B, T, Hkv, D, W):
    kc = wl.random_bf16((B, W, Hkv, D), 41)
    vc = wl.random_bf16((B, W, Hkv, D), 42)
    kn = wl.random_bf16((B, T, Hkv, D), 43)
    vn = wl.random_bf16((B, T, Hkv, D), 44)
    pos = wl.random_positions(B, 0, 3 * W, 45)
    kg, vg = kc.cuda(), vc.cuda()
    swa.swa_cache_append(kn.cuda(), vn.cuda(), kg, vg, pos.cuda())
    torch.cuda.synchronize()
    kr = kc.view(torch.int16).numpy().copy()
    vr = vc.view(torch.int16).numpy().copy()
    oracle_mod.cache_append(kr, vr, None, kn.view(torch.int16).numpy(), vn.view(torch.int16).numpy(), pos.numpy())
    assert np.array_equal(kg.cpu().view(torch.int16).numpy(), kr)
    assert np.array_equal(vg.cpu().view(torch.int16).numpy(), vr)


# ------------------------------------------------------------------ chunked prefill

def _chunked_case(oracle_mod, B, N, C, Hq, Hkv, D, W, seed, start=0):
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, Hkv, D), seed + 1)
    v = wl.random_bf16((B, N, Hkv, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    outs = []
    for s0 in range(start, N, C):
        e = min(N, s0 + C)
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        outs.append(swa.swa_prefill_chunk(q[:, s0:e].cuda().contiguous(), k[:, s0:e].cuda().contiguous(),
                                          v[:, s0:e].cuda().contiguous(), kc, vc, st, W, scale))
    torch.cuda.synchronize()
    return q, k, v, scale, torch.cat([o.cpu() for o in outs], dim=1), kc.cpu(), vc.cpu()


@pytest.mark.parametrize("B,N,C,Hq,Hkv,D,W", [
    (1, 512, 128, 4, 2, 128, 128),    # C = W aligned
    (2, 700, 96, 4, 2, 128, 256),     # C < W, unaligned starts
    (1, 600, 200, 8, 2, 64, 200),     # W not a multiple of 128, C = W
    (1, 333, 45, 2, 1, 128, 100),     # small ragged chunks
    (1, 1100, 300, 6, 2, 128, 384),   # odd group, wrap inside tiles
    (2, 2560, 1280, 16, 4, 128, 1536),  # 160 units: on 148 SMs the last 12 run as single-head units
    (1, 2560, 1280, 32, 16, 64, 1280),  # the same split with G=2, D=64, C=W
])
def test_chunked_prefill_matches_oracle(oracle_mod, B, N, C, Hq, Hkv, D, W):
    q, k, v, scale, out, kc, vc = _chunked_case(oracle_mod, B, N, C, Hq, Hkv, D, W, seed=N + C)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale)
    assert_close(out, ref, f"chunked N{N} C{C} W{W}")
    # cache: slot s holds the last position p < N with p mod W == s, bit for bit
    for s in range(min(W, N)):
        p = s + ((N - 1 - s) // W) * W
        assert torch.equal(kc[:, s], k[:, p]) and torch.equal(vc[:, s], v[:, p]), (s, p)


# ------------------------------------------------------------------ decode

def _decode_case(oracle_mod, B, Hq, Hkv, D, W, pos0, steps, seed):
    kc = wl.random_bf16((B, W, Hkv, D), seed)
    vc = wl.random_bf16((B, W, Hkv, D), seed + 1)
    qs = wl.random_bf16((steps, B, Hq, D), seed + 2)
    kn = wl.random_bf16((steps, B, Hkv, D), seed + 3)
    vn = wl.random_bf16((steps, B, Hkv, D), seed + 4)
    scale = 1.0 / math.sqrt(D)
    kg, vg = kc.cuda(), vc.cuda()
    pos0 = torch.as_tensor(pos0, dtype=torch.int32)
    sp = oracle_mod.slot_positions(pos0.numpy(), W)
    kr, vr = f64(kc), f64(vc)
    for s in range(steps):
        pos = (pos0 + s).to(torch.int32)
        pg = pos.cuda()
        swa.swa_cache_append(kn[s].unsqueeze(1).cuda(), vn[s].unsqueeze(1).cuda(), kg, vg, pg)
        out = swa.swa_decode(qs[s].cuda(), kg, vg, pg, scale)
        torch.cuda.synchronize()
        oracle_mod.cache_append(kr, vr, sp, f64(kn[s].unsqueeze(1)), f64(vn[s].unsqueeze(1)), pos.numpy())
        ref = oracle_mod.swa_decode(f64(qs[s]), kr, vr, sp, pos.numpy(), W, scale)
        assert_close(out.cpu(), ref, f"decode step {s}")
    assert np.array_equal(f64(kg.cpu()), kr) and np.array_equal(f64(vg.cpu()), vr)


@pytest.mark.parametrize("B,Hq,Hkv,D,W,pos0", [
    (4, 32, 8, 128, 4096, [0, 1, 4094, 4095]),          # partial buffer, last slot, first wrap
    (3, 8, 2, 128, 4096, [4096, 8191, 30000]),          # wrap points and deep positions
    (2, 4, 4, 64, 700, [10, 2000]),                     # G=1, W not a multiple of 16 keys per block
    (2, 16, 2, 128, 1000, [999, 5]),                    # G=8
    (2, 4, 2, 64, 300, [299, 77]),                      # G=2, single split
    (2, 8, 2, 128, 8192, [8191, 20000]),                # small batch: 32 splits of 256 keys, merged
    (1, 4, 1, 64, 5000, [4999]),                        # 20 splits of 256, the last one partial, G=4, D=64
])
def test_decode_edge_cases(oracle_mod, B, Hq, Hkv, D, W, pos0):
    _decode_case(oracle_mod, B, Hq, Hkv, D, W, pos0, steps=3, seed=B * W + D)


@pytest.mark.parametrize("B,Hq,Hkv,D,W,pos0", [
    (8, 32, 8, 128, 4096, [0, 1, 17, 63, 64, 4094, 4095, 9000]),  # 4 splits of 1024; short windows leave blocks empty
    (2, 4, 2, 64, 1000, [5, 30000]),                              # 4 splits of 256 (small batch), D=64
    (4, 96, 8, 128, 1024, [1023, 3, 5000, 700]),                  # group of 12: two groups of 6 per K/V head
])
def test_decode_windows_of_four_splits_merge_in_a_cluster(oracle_mod, B, Hq, Hkv, D, W, pos0):
    """A window cut into exactly 4 splits (the W=4096 decode at large batch) is
    merged on chip by the 4 blocks of a cluster: outputs against the oracle,
    plain and with RoPE on q, and the caller's workspace left as it was."""
    kc = wl.random_bf16((B, W, Hkv, D), 9100 + W)
    vc = wl.random_bf16((B, W, Hkv, D), 9101 + W)
    q = wl.random_bf16((B, Hq, D), 9102 + W)
    pos = torch.tensor(pos0, dtype=torch.int32)
    scale = 1.0 / math.sqrt(D)
    sp = oracle_mod.slot_positions((pos + 1).numpy(), W)     # the token at pos is already in the buffer
    need = swa.swa_decode_workspace_size(B, Hq, Hkv, D, W)
    assert need > 0
    ws = torch.full((need,), 0x5A, dtype=torch.uint8, device="cuda")
    kg, vg, pg = kc.cuda(), vc.cuda(), pos.cuda()
    out = swa.swa_decode(q.cuda(), kg, vg, pg, scale, workspace=ws)
    outr = swa.swa_decode(q.cuda(), kg, vg, pg, scale, workspace=ws, rope_theta=10000.0)
    torch.cuda.synchronize()
    assert bool((ws == 0x5A).all()), "the on-chip merge leaves the workspace untouched"
    ref = oracle_mod.swa_decode(f64(q), f64(kc), f64(vc), sp, pos.numpy(), W, scale)
    assert_close(out.cpu(), ref, f"4-split decode B{B} W{W} G{Hq // Hkv}")
    qr = oracle_mod.rope(f64(q)[:, None], pos.numpy(), 10000.0)[:, 0]
    refr = oracle_mod.swa_decode(qr, f64(kc), f64(vc), sp, pos.numpy(), W, scale)
    assert_close(outr.cpu(), refr, f"4-split decode RoPE B{B} W{W}")


def test_prefill_then_decode_continues_the_sequence(oracle_mod):
    """Chunked prefill leaves the buffer in the state decode continues from:
    decode at position N equals row N of one-shot SWA over N+1 tokens."""
    B, N, C, Hq, Hkv, D, W = 1, 600, 256, 8, 2, 128, 256
    q = wl.random_bf16((B, N + 1, Hq, D), 51)
    k = wl.random_bf16((B, N + 1, Hkv, D), 52)
    v = wl.random_bf16((B, N + 1, Hkv, D), 53)
    scale = 1.0 / math.sqrt(D)
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    for s0 in range(0, N, C):
        e = min(N, s0 + C)
        st = torch.full((B,), s0, dtype=torch.int32, device="cuda")
        swa.swa_prefill_chunk(q[:, s0:e].cuda().contiguous(), k[:, s0:e].cuda().contiguous(),
                              v[:, s0:e].cuda().contiguous(), kc, vc, st, W, scale)
    pos = torch.full((B,), N, dtype=torch.int32, device="cuda")
    swa.swa_cache_append(k[:, N:].cuda().contiguous(), v[:, N:].cuda().contiguous(), kc, vc, pos)
    out = swa.swa_decode(q[:, N].cuda().contiguous(), kc, vc, pos, scale)
    ref = oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale, rows=[N])
    assert_close(out.cpu(), ref[:, 0], "prefill -> decode")


# ------------------------------------------------------------------ FMA-pipe exponential

def test_polynomial_exp2_against_cuda_exp2():
    """The softmax's polynomial 2^x against CUDA's exp2f (torch.exp2) on the
    range it sees (x <= 8 after max subtraction), plus masked inputs."""
    x = torch.cat([torch.linspace(-126.0, 8.0, 1_000_003, device="cuda"),
                   torch.rand(1_000_000, device="cuda") * 20 - 12]).contiguous()
    y = swa.swa_selftest_exp2(x)
    ref = torch.exp2(x.double())
    rel = ((y.double() - ref).abs() / ref).max().item()
    # fit error 7.5e-5 plus fp32 rounding of coefficients and Horner steps;
    # P is stored in bf16 (relative step 2^-8), so 2e-4 is far below what matters
    assert rel < 2e-4, rel
    lo = torch.tensor([-126.5, -127.0, -200.0, -1e30, float("-inf")], device="cuda")
    ylo = swa.swa_selftest_exp2(lo)
    assert bool(((ylo >= 0) & (ylo <= 2.0 ** -125)).all()), ylo.tolist()


# ------------------------------------------------------------------ failure paths (no fault)

def test_timeout_path_reports_status_and_context_survives(oracle_mod):
    swa.swa_set_wait_limit_ns(2_000_000)            # 2 ms
    try:
        swa.swa_selftest_wait_timeout()
        assert swa.swa_get_device_status() == swa.SWA_ERR_TIMEOUT
    finally:
        swa.swa_set_wait_limit_ns(1_000_000_000)
    assert swa.swa_get_device_status() == swa.SWA_OK
    test_prefill_edge_cases(oracle_mod, 1, 300, 4, 2, 128, 64)


def test_negative_position_is_reported_not_faulted():
    B, W, Hkv, D = 2, 64, 2, 64
    kc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros_like(kc)
    kn = torch.ones(B, 1, Hkv, D, dtype=torch.bfloat16, device="cuda")
    pos = torch.tensor([-5, 3], dtype=torch.int32, device="cuda")
    swa.swa_cache_append(kn, kn, kc, vc, pos)
    assert swa.swa_get_device_status() == swa.SWA_ERR_INVALID_ARG
    assert kc[0].abs().sum().item() == 0 and kc[1, 3].abs().sum().item() > 0


def test_host_side_validation_errors():
    q = torch.zeros(1, 16, 4, 128, dtype=torch.bfloat16, device="cuda")
    k = torch.zeros(1, 16, 2, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(swa.SwaError) as e:
        swa.swa_prefill(q, k, k, 0, 0.1)             # W = 0
    assert e.value.status == swa.SWA_ERR_INVALID_ARG
    with pytest.raises(swa.SwaError) as e:
        swa.swa_prefill(q, k, k, 4, float("nan"))
    assert e.value.status == swa.SWA_ERR_INVALID_ARG
    q3 = torch.zeros(1, 16, 3, 128, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(swa.SwaError) as e:
        swa.swa_prefill(q3, k, k, 4, 0.1)            # Hq % Hkv != 0
    assert e.value.status == swa.SWA_ERR_INVALID_ARG
    q96 = torch.zeros(1, 16, 4, 96, dtype=torch.bfloat16, device="cuda")
    k96 = torch.zeros(1, 16, 2, 96, dtype=torch.bfloat16, device="cuda")
    with pytest.raises(swa.SwaError) as e:
        swa.swa_prefill(q96, k96, k96, 4, 0.1)       # head_dim 96
    assert e.value.status == swa.SWA_ERR_UNSUPPORTED


def test_decode_bindings_check_the_key_cache_shape():
    """The decode bindings take W and Hkv from k_cache and check its full
    shape, so an undersized or mismatched key cache is refused on the host
    before any launch could read past it."""
    B, Hq, Hkv, D, W = 4, 8, 2, 128, 64
    q = torch.zeros(B, Hq, D, dtype=torch.bfloat16, device="cuda")
    vc = torch.zeros(B, W, Hkv, D, dtype=torch.bfloat16, device="cuda")
    pos = torch.zeros(B, dtype=torch.int32, device="cuda")
    out = torch.empty_like(q)
    ks = torch.zeros(B, 4, Hkv, D, dtype=torch.bfloat16, device="cuda")
    bad = [torch.zeros(B - 1, W, Hkv, D, dtype=torch.bfloat16, device="cuda"),    # fewer sequences
           torch.zeros(B, W, Hkv, 64, dtype=torch.bfloat16, device="cuda")]       # head_dim differs from q's
    for kc in bad:
        with pytest.raises(ValueError):
            swa.swa_decode(q, kc, vc, pos, 0.1, out=out)
        with pytest.raises(ValueError):
            swa.swa_decode_noalloc(q, kc, vc, pos, 0.1, out)
        with pytest.raises(ValueError):
            swa.swa_decode_sinks(q, kc, vc, ks, ks, pos, 0.1, out=out)


# ------------------------------------------------------------------ one query head per KV head

@pytest.mark.parametrize("B,N,Hq,H,D,W", [
    (1, 1900, 32, 32, 128, 500),     # one head per KV head; 15 query blocks: the last pair holds one
    (2, 1280, 16, 16, 64, 300),      # D=64, an even number of blocks
    (1, 2048, 32, 32, 128, 3000),    # window wider than the sequence
    (1, 2560, 24, 8, 128, 600),      # groups of 3
    (1, 1700, 40, 8, 64, 450),       # groups of 5, ragged last pair, D=64
    (1, 1300, 56, 8, 128, 700),      # groups of 7
])
def test_odd_groups_in_units_of_two_query_blocks(oracle_mod, B, N, Hq, H, D, W):
    """Odd groups (1, 3, 5, 7 query heads per KV head) with at least two waves
    of units: a unit takes two consecutive 128-row query blocks of one head (key
    tiles of both bands, masked per row), plain, with RoPE on q and with
    sinks."""
    seed = 8000 + N + H
    q = wl.random_bf16((B, N, Hq, D), seed)
    k = wl.random_bf16((B, N, H, D), seed + 1)
    v = wl.random_bf16((B, N, H, D), seed + 2)
    scale = 1.0 / math.sqrt(D)
    out = run_prefill(q, k, v, W, scale)
    assert_close(out, oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale), f"G={Hq // H} B{B} N{N} D{D} W{W}")
    outr = swa.swa_prefill(q.cuda(), k.cuda(), v.cuda(), W, scale, rope_theta=10000.0)
    qr = oracle_mod.rope(f64(q), np.zeros(B, np.int32), 10000.0)
    assert_close(outr.cpu(), oracle_mod.swa_prefill(qr, f64(k), f64(v), W, scale), f"MHA RoPE N{N}")
    outs = swa.swa_prefill_sinks(q.cuda(), k.cuda(), v.cuda(), W, 4, scale)
    assert_close(outs.cpu(), oracle_mod.swa_prefill_sinks(f64(q), f64(k), f64(v), W, 4, scale), f"MHA sinks N{N}")


@pytest.mark.parametrize("B,Hq,H", [(1, 32, 32), (2, 24, 8)])
def test_odd_groups_chunked_in_units_of_two_query_blocks(oracle_mod, B, Hq, H):
    """Chunked prefill with groups of 1 and 3 (10 query blocks per chunk: 320
    head-pair units either way, so pairs of blocks): every row against
    one-shot SWA, the buffer bit for bit."""
    N, C, D, W = 2560, 1280, 128, 1280
    q, k, v, scale, out, kc, vc = _chunked_case(oracle_mod, B, N, C, Hq, H, D, W, seed=8100 + Hq)
    assert_close(out, oracle_mod.swa_prefill(f64(q), f64(k), f64(v), W, scale), f"G={Hq // H} chunked")
    for s in range(W):
        p = s + ((N - 1 - s) // W) * W
        assert torch.equal(kc[:, s], k[:, p]) and torch.equal(vc[:, s], v[:, p]), (s, p)
