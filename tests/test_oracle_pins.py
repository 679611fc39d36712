"""Pins of the fp64 CPU oracle to facts fixed outside the oracle itself.

Each test checks the oracle against one of: a value worked by hand from the
pages (tests/golden/), a closed form, a library routine (torch's
scaled_dot_product_attention in float64), an invariant the method must keep,
or brute force over explicit key sets.  No GPU is used.
"""
import math
import os

import numpy as np
import pytest
import torch

from sliding_window_gqa_prefill_b200 import workloads

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _rand(shape, seed, scale=1.0):
    return np.random.default_rng(seed).standard_normal(shape) * scale


def _sdpa(q, k, v, scale, mask=None, causal=False):
    """torch SDPA in float64 on [B, N, H, D] inputs with K/V heads already expanded."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)
    with torch.no_grad():
        o = torch.nn.functional.scaled_dot_product_attention(
            t(q), t(k), t(v), attn_mask=None if mask is None else torch.from_numpy(mask),
            is_causal=causal, scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


# ---------------------------------------------------------------- hand-worked examples

def test_golden_hand_example(oracle_mod):
    """Values worked by hand from the window definition (golden file)."""
    rows = [l.split() for l in open(os.path.join(GOLDEN, "swa_hand_example.txt"))
            if l.strip() and not l.startswith("#")]
    q = np.ones((1, 3, 1, 1))
    k = np.array([0.0, math.log(2.0), math.log(3.0)]).reshape(1, 3, 1, 1)
    v = np.array([1.0, 10.0, 100.0]).reshape(1, 3, 1, 1)
    assert len(rows) == 8
    for W, mode, row, expect in rows:
        out = oracle_mod.swa_prefill(q, k, v, int(W), 1.0, mode=int(mode))
        assert out[0, int(row), 0, 0] == pytest.approx(float(expect), rel=1e-13)


def test_golden_rolling_buffer_w4(oracle_mod):
    """slot = p mod W: ten positions written into W=4 slots (golden file)."""
    lines = [l.split() for l in open(os.path.join(GOLDEN, "rolling_buffer_w4.txt"))
             if l.strip() and not l.startswith("#")]
    assert lines[0] == ["W", "4"]
    W = 4
    kc = np.zeros((1, W, 1, 1), np.uint16)
    vc = np.zeros((1, W, 1, 1), np.uint16)
    sp = np.full((1, W), -1, np.int32)
    for row in lines[1:]:
        p = int(row[0])
        tok = np.full((1, 1, 1, 1), 1000 + p, np.uint16)
        oracle_mod.cache_append(kc, vc, sp, tok, tok + 1, [p])
        assert sp[0].tolist() == [int(x) for x in row[1:]]
        # the bytes stored follow the same map
        want = [1000 + x if x >= 0 else 0 for x in sp[0]]
        assert kc[0, :, 0, 0].tolist() == want
        assert vc[0, :, 0, 0].tolist() == [w + 1 if w else 0 for w in want]
    # the appends as a batch of T=10 tokens give the same final state
    kc2 = np.zeros_like(kc)
    sp2 = np.full((1, W), -1, np.int32)
    toks = (1000 + np.arange(10, dtype=np.uint16)).reshape(1, 10, 1, 1)
    oracle_mod.cache_append(kc2, kc2.copy(), sp2, toks, toks, [0])
    assert sp2[0].tolist() == [8, 9, 6, 7]
    assert kc2[0, :, 0, 0].tolist() == [1008, 1009, 1006, 1007]
    # simulated fill map agrees
    assert oracle_mod.slot_positions([10], 4)[0].tolist() == [8, 9, 6, 7]


# ---------------------------------------------------------------- brute force and library routines

@pytest.mark.parametrize("W", [1, 3, 7, 24, 64])
def test_brute_force_explicit_key_sets(oracle_mod, W):
    """Every row against a brute force over its key set, built as 'the last W
    positions at or before i' by sorting (not by the window inequality)."""
    B, N, Hq, Hkv, D = 2, 24, 4, 2, 8
    q, k, v = _rand((B, N, Hq, D), 1), _rand((B, N, Hkv, D), 2), _rand((B, N, Hkv, D), 3)
    scale = 0.37
    out = oracle_mod.swa_prefill(q, k, v, W, scale)
    G = Hq // Hkv
    for b in range(B):
        for i in range(N):
            keys = sorted(range(i + 1))[-W:]
            for h in range(Hq):
                g = h // G
                s = np.array([scale * float(q[b, i, h] @ k[b, j, g]) for j in keys])
                w = np.exp(s - s.max())
                w /= w.sum()
                ref = sum(wj * v[b, j, g] for wj, j in zip(w, keys))
                np.testing.assert_allclose(out[b, i, h], ref, rtol=1e-12, atol=1e-12)


@pytest.mark.parametrize("N,W", [(33, 33), (33, 40), (20, 1000)])
def test_wide_window_is_dense_causal_sdpa(oracle_mod, N, W):
    """W >= N reduces to dense causal attention: torch SDPA (is_causal) in fp64."""
    B, Hq, Hkv, D = 2, 8, 2, 16
    q, k, v = _rand((B, N, Hq, D), 4), _rand((B, N, Hkv, D), 5), _rand((B, N, Hkv, D), 6)
    scale = 1 / math.sqrt(D)
    out = oracle_mod.swa_prefill(q, k, v, W, scale)
    G = Hq // Hkv
    ref = _sdpa(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), scale, causal=True)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


@pytest.mark.parametrize("W", [1, 5, 16])
def test_window_matches_sdpa_with_boolean_mask(oracle_mod, W):
    """Banded attention equals torch SDPA (fp64) with a boolean band mask."""
    B, N, Hq, Hkv, D = 1, 40, 4, 1, 8
    q, k, v = _rand((B, N, Hq, D), 7), _rand((B, N, Hkv, D), 8), _rand((B, N, Hkv, D), 9)
    out = oracle_mod.swa_prefill(q, k, v, W, 0.5)
    i = np.arange(N)[:, None]
    j = np.arange(N)[None, :]
    mask = (j <= i) & (j > i - W)
    ref = _sdpa(q, np.repeat(k, Hq, 2), np.repeat(v, Hq, 2), 0.5, mask=mask)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


def test_gqa_equals_mha_with_repeated_kv_heads(oracle_mod):
    """GQA (32 query heads, 8 KV heads: group size 4) equals MHA with each
    KV head repeated 4 times in place (contiguous groups)."""
    B, N, Hq, Hkv, D, W = 1, 40, 32, 8, 8, 9
    q, k, v = _rand((B, N, Hq, D), 10), _rand((B, N, Hkv, D), 11), _rand((B, N, Hkv, D), 12)
    gqa = oracle_mod.swa_prefill(q, k, v, W, 0.3)
    mha = oracle_mod.swa_prefill(q, np.repeat(k, 4, axis=2), np.repeat(v, 4, axis=2), W, 0.3)
    np.testing.assert_array_equal(gqa, mha)
    # and a strided (h % Hkv) grouping would give a different answer
    strided = oracle_mod.swa_prefill(q, np.tile(k, (1, 1, 4, 1)), np.tile(v, (1, 1, 4, 1)), W, 0.3)
    assert np.abs(strided - gqa).max() > 1e-3


# ---------------------------------------------------------------- closed forms

def test_window_of_one_returns_own_value(oracle_mod):
    B, N, Hq, Hkv, D = 2, 17, 4, 2, 8
    q, k, v = _rand((B, N, Hq, D), 13), _rand((B, N, Hkv, D), 14), _rand((B, N, Hkv, D), 15)
    out = oracle_mod.swa_prefill(q, k, v, 1, 1.0)
    np.testing.assert_array_equal(out, np.repeat(v, 2, axis=2))


@pytest.mark.parametrize("W", [1, 4, 9, 30])
def test_constant_keys_average_the_window(oracle_mod, W):
    """Equal keys give equal weights: row i is the mean of V over
    positions max(0, i-W+1) .. i (pins the window size to W keys)."""
    B, N, Hq, Hkv, D = 1, 30, 2, 1, 4
    q = _rand((B, N, Hq, D), 16)
    k = np.broadcast_to(_rand((1, 1, 1, D), 17), (B, N, Hkv, D)).copy()
    v = _rand((B, N, Hkv, D), 18)
    out = oracle_mod.swa_prefill(q, k, v, W, 1.0)
    for i in range(N):
        lo = max(0, i - W + 1)
        np.testing.assert_allclose(out[0, i, 0], v[0, lo:i + 1, 0].mean(axis=0), rtol=1e-12, atol=1e-13)


def test_softmax_weights_sum_to_one(oracle_mod):
    """Values of all ones come back as ones (weights sum to 1 to 1e-12)."""
    B, N, Hq, Hkv, D = 1, 50, 4, 2, 8
    q, k = _rand((B, N, Hq, D), 19, 3.0), _rand((B, N, Hkv, D), 20, 3.0)
    out = oracle_mod.swa_prefill(q, k, np.ones((B, N, Hkv, D)), 7, 1.0)
    np.testing.assert_allclose(out, 1.0, atol=1e-12)


def test_inclusive_reading_is_one_more_key(oracle_mod):
    """The i-W <= j <= i reading with W equals i-W < j <= i with W+1."""
    B, N, Hq, Hkv, D = 1, 30, 4, 2, 8
    q, k, v = _rand((B, N, Hq, D), 21), _rand((B, N, Hkv, D), 22), _rand((B, N, Hkv, D), 23)
    a = oracle_mod.swa_prefill(q, k, v, 5, 0.4, mode=oracle_mod.WINDOW_INCL_LEFT)
    b = oracle_mod.swa_prefill(q, k, v, 6, 0.4, mode=oracle_mod.WINDOW_EXCL_LEFT)
    np.testing.assert_array_equal(a, b)


def test_row_sampling_matches_full(oracle_mod):
    B, N, Hq, Hkv, D = 2, 40, 4, 2, 8
    q, k, v = _rand((B, N, Hq, D), 24), _rand((B, N, Hkv, D), 25), _rand((B, N, Hkv, D), 26)
    full = oracle_mod.swa_prefill(q, k, v, 11, 0.3)
    rows = [0, 10, 11, 39, 5]
    part = oracle_mod.swa_prefill(q, k, v, 11, 0.3, rows=rows)
    np.testing.assert_array_equal(part, full[:, rows])


# ---------------------------------------------------------------- rolling buffer, chunking, decode

def _run_chunked(oracle_mod, q, k, v, W, C, scale, start=0):
    """Pre-fill a prompt chunk by chunk through a W-slot cache; returns
    (outputs, k_cache, v_cache, slot_pos)."""
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    kc = np.zeros((B, W, Hkv, D))
    vc = np.zeros((B, W, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    outs = []
    for s0 in range(start, N, C):
        e = min(N, s0 + C)
        st = np.full(B, s0, np.int32)
        outs.append(oracle_mod.swa_chunk(q[:, s0:e], k[:, s0:e], v[:, s0:e], kc, vc, sp, st, W, scale))
        oracle_mod.cache_append(kc, vc, sp, k[:, s0:e], v[:, s0:e], st)
    return np.concatenate(outs, axis=1), kc, vc, sp


@pytest.mark.parametrize("W,C", [(16, 16), (16, 8), (16, 5), (12, 1), (7, 7), (64, 64)])
def test_chunked_prefill_equals_one_shot(oracle_mod, W, C):
    B, N, Hq, Hkv, D = 2, 53, 4, 2, 8
    q, k, v = _rand((B, N, Hq, D), 27), _rand((B, N, Hkv, D), 28), _rand((B, N, Hkv, D), 29)
    one = oracle_mod.swa_prefill(q, k, v, W, 0.25)
    chunked, kc, vc, sp = _run_chunked(oracle_mod, q, k, v, W, C, 0.25)
    np.testing.assert_allclose(chunked, one, rtol=1e-12, atol=1e-13)
    # final buffer: slot s holds the last position p < N with p mod W == s
    for s in range(W):
        p = max(x for x in range(N) if x % W == s) if s < N else -1
        assert sp[0, s] == p
        if p >= 0:
            np.testing.assert_array_equal(kc[:, s], k[:, p])
            np.testing.assert_array_equal(vc[:, s], v[:, p])


def test_chunk_reads_cache_before_writing(oracle_mod):
    """With C = W the chunk overwrites every slot; attending after writing
    would lose the previous window and differ from one-shot."""
    B, N, Hq, Hkv, D, W = 1, 32, 2, 1, 4, 16
    q, k, v = _rand((B, N, Hq, D), 30), _rand((B, N, Hkv, D), 31), _rand((B, N, Hkv, D), 32)
    one = oracle_mod.swa_prefill(q, k, v, W, 0.5)
    kc, vc = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    oracle_mod.cache_append(kc, vc, sp, k[:, :16], v[:, :16], [0])
    oracle_mod.cache_append(kc, vc, sp, k[:, 16:], v[:, 16:], [16])     # write first (wrong order)
    wrong = oracle_mod.swa_chunk(q[:, 16:], k[:, 16:], v[:, 16:], kc, vc, sp, [16], W, 0.5)
    assert np.abs(wrong - one[:, 16:]).max() > 1e-3


def test_decode_equals_row_of_one_shot(oracle_mod):
    """Append position p, then decode == row p of one-shot SWA over the same
    token history (pos below, at and past the first wrap)."""
    B, N, Hq, Hkv, D, W = 1, 40, 4, 2, 8, 8
    q, k, v = _rand((B, N, Hq, D), 33), _rand((B, N, Hkv, D), 34), _rand((B, N, Hkv, D), 35)
    one = oracle_mod.swa_prefill(q, k, v, W, 0.3)
    kc, vc = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    for p in range(N):
        oracle_mod.cache_append(kc, vc, sp, k[:, p:p + 1], v[:, p:p + 1], [p])
        out = oracle_mod.swa_decode(q[:, p], kc, vc, sp, [p], W, 0.3)
        np.testing.assert_allclose(out, one[:, p], rtol=1e-12, atol=1e-13)


def test_decode_window_over_cache_never_needs_more_than_w_slots(oracle_mod):
    """Under i-W < j <= i every key a query needs is still in a W-slot buffer;
    under i-W <= j <= i the oldest needed key was overwritten by position i."""
    B, N, Hq, Hkv, D, W = 1, 20, 2, 1, 4, 5
    q, k, v = _rand((B, N, Hq, D), 36), _rand((B, N, Hkv, D), 37), _rand((B, N, Hkv, D), 38)
    incl = oracle_mod.swa_prefill(q, k, v, W, 0.3, mode=oracle_mod.WINDOW_INCL_LEFT)
    kc, vc = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    oracle_mod.cache_append(kc, vc, sp, k[:, :N], v[:, :N], [0])
    p = N - 1
    dec = oracle_mod.swa_decode(q[:, p], kc, vc, sp, [p], W, 0.3, mode=oracle_mod.WINDOW_INCL_LEFT)
    assert np.abs(dec - incl[:, p]).max() > 1e-3


def test_slot_positions_closed_form(oracle_mod):
    """Simulated writes of 0..n-1 leave slot s holding n-1-((n-1-s) mod W)."""
    W = 37
    counts = [0, 1, 5, 36, 37, 38, 100, 4096]
    sp = oracle_mod.slot_positions(counts, W)
    for b, n in enumerate(counts):
        for s in range(W):
            p = n - 1 - ((n - 1 - s) % W)
            assert sp[b, s] == (p if p >= 0 else -1)


def test_cache_memory_is_constant_and_8x_at_32k():
    """Cache bytes depend on W only; for a 32K-token sequence and W = 4096 a
    dense cache is 8x larger (the pages' 8x memory figure)."""
    B, Hkv, D, W, bytes_el = 1, 8, 128, 4096, 2
    rolling = B * W * Hkv * D * bytes_el * 2
    for N in (4096, 8192, 32768, 1 << 20):
        dense = B * N * Hkv * D * bytes_el * 2
        if N == 32768:
            assert dense / rolling == 8
    assert rolling == 16 * 2 ** 20


def test_useful_pair_counts():
    """Counting of unmasked pairs, against brute force and the closed forms
    used for FLOP accounting (N=16384, W=4096 vs dense: ratio 2.286, which
    the pages round to '~2x')."""
    for N, W in [(1, 1), (5, 2), (17, 17), (40, 7), (100, 300)]:
        brute = sum(1 for i in range(N) for j in range(N) if i - W < j <= i)
        assert workloads.useful_pairs(N, W) == brute
    assert workloads.useful_pairs(8192, 4096) == 25_167_872
    assert workloads.useful_pairs(16384, 4096) == 58_722_304
    assert workloads.useful_pairs(16384, 16384) == 134_225_920
    assert abs(134_225_920 / 58_722_304 - 2.286) < 1e-3
    assert workloads.useful_flops(2, 16384, 4096, 32, 128) == 1_924_212_457_472


# ---------------------------------------------------------------- rotary position embedding

def test_rope_position_zero_is_identity(oracle_mod):
    x = _rand((2, 1, 3, 16), 40)
    np.testing.assert_array_equal(oracle_mod.rope(x, [0, 0]), x)


def test_rope_closed_form_two_dims(oracle_mod):
    """D = 2: the single pair turns by p radians (theta^0 = 1)."""
    x = np.zeros((1, 5, 1, 2))
    x[..., 0] = 1.0
    y = oracle_mod.rope(x, [3])
    for t in range(5):
        np.testing.assert_allclose(y[0, t, 0], [np.cos(3 + t), np.sin(3 + t)], rtol=0, atol=1e-15)


def test_rope_matches_complex_multiplication(oracle_mod):
    """Brute force with numpy complex numbers: pair i is the complex number
    x[2i] + 1j*x[2i+1], multiplied by exp(1j * p * theta**(-2i/D))."""
    B, T, H, D = 2, 7, 3, 64
    x = _rand((B, T, H, D), 41)
    pos = [5, 31000]
    y = oracle_mod.rope(x, pos)
    c = x[..., 0::2] + 1j * x[..., 1::2]
    p = (np.asarray(pos)[:, None] + np.arange(T)[None, :]).astype(np.float64)
    ang = p[:, :, None, None] * (10000.0 ** (-np.arange(D // 2) * 2.0 / D))[None, None, None, :]
    z = c * np.exp(1j * ang)
    np.testing.assert_allclose(y[..., 0::2], z.real, rtol=0, atol=1e-9)
    np.testing.assert_allclose(y[..., 1::2], z.imag, rtol=0, atol=1e-9)


def test_rope_preserves_pair_norms_and_composes(oracle_mod):
    x = _rand((1, 4, 2, 32), 42)
    y = oracle_mod.rope(x, [100])
    n0 = x[..., 0::2] ** 2 + x[..., 1::2] ** 2
    n1 = y[..., 0::2] ** 2 + y[..., 1::2] ** 2
    np.testing.assert_allclose(n1, n0, rtol=1e-12)
    # rotating by a then by b equals rotating by a + b (one row: row t adds t twice)
    x1 = x[:, :1]
    z = oracle_mod.rope(oracle_mod.rope(x1, [100]), [250])
    np.testing.assert_allclose(z, oracle_mod.rope(x1, [350]), rtol=0, atol=1e-9)


def test_rope_scores_depend_on_relative_position_only(oracle_mod):
    """<R(p) q, R(p') k> is unchanged when both positions shift by the same c."""
    q = _rand((1, 1, 1, 128), 43)
    k = _rand((1, 1, 1, 128), 44)
    s1 = float(np.sum(oracle_mod.rope(q, [1000]) * oracle_mod.rope(k, [900])))
    s2 = float(np.sum(oracle_mod.rope(q, [1100 + 4096]) * oracle_mod.rope(k, [1000 + 4096])))
    assert abs(s1 - s2) < 1e-8


# ---------------------------------------------------------------- attention sinks

def test_sinks_zero_is_plain_window(oracle_mod):
    B, N, Hq, Hkv, D = 1, 40, 4, 2, 8
    q, k, v = _rand((B, N, Hq, D), 50), _rand((B, N, Hkv, D), 51), _rand((B, N, Hkv, D), 52)
    np.testing.assert_array_equal(oracle_mod.swa_prefill_sinks(q, k, v, 7, 0, 0.3),
                                  oracle_mod.swa_prefill(q, k, v, 7, 0.3))


@pytest.mark.parametrize("W,S", [(5, 4), (1, 2), (3, 10), (40, 4)])
def test_sinks_brute_force(oracle_mod, W, S):
    """Key set of row i built as a set union: last W positions, plus the first S."""
    B, N, Hq, Hkv, D = 1, 30, 2, 1, 8
    q, k, v = _rand((B, N, Hq, D), 53), _rand((B, N, Hkv, D), 54), _rand((B, N, Hkv, D), 55)
    out = oracle_mod.swa_prefill_sinks(q, k, v, W, S, 0.4)
    for i in range(N):
        keys = sorted(set(sorted(range(i + 1))[-W:]) | set(range(min(S, i + 1))))
        for h in range(Hq):
            s = np.array([0.4 * float(q[0, i, h] @ k[0, j, 0]) for j in keys])
            w = np.exp(s - s.max())
            w /= w.sum()
            np.testing.assert_allclose(out[0, i, h], sum(wj * v[0, j, 0] for wj, j in zip(w, keys)),
                                       rtol=1e-12, atol=1e-12)


def test_sink_decode_equals_row_of_prefill(oracle_mod):
    """Streaming decode with a W-slot rolling buffer plus an S-slot sink buffer
    equals row p of one-shot prefill with sinks, at every step."""
    B, N, Hq, Hkv, D, W, S = 2, 45, 4, 2, 8, 8, 4
    q, k, v = _rand((B, N, Hq, D), 56), _rand((B, N, Hkv, D), 57), _rand((B, N, Hkv, D), 58)
    one = oracle_mod.swa_prefill_sinks(q, k, v, W, S, 0.3)
    kc, vc = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    ks, vs = np.zeros((B, S, Hkv, D)), np.zeros((B, S, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    for p in range(N):
        pos = [p] * B
        oracle_mod.cache_append(kc, vc, sp, k[:, p:p + 1], v[:, p:p + 1], pos)
        oracle_mod.sink_append(ks, vs, k[:, p:p + 1], v[:, p:p + 1], pos)
        out = oracle_mod.swa_decode_sinks(q[:, p], kc, vc, sp, ks, vs, pos, W, 0.3)
        np.testing.assert_allclose(out, one[:, p], rtol=1e-12, atol=1e-13)
    # the sink buffer holds exactly the first S positions
    np.testing.assert_array_equal(ks, k[:, :S])
