"""Property tests of the fp64 oracle over random shapes (hypothesis, derandomised
so every run draws the same cases).  Each property ties the oracle to something
outside it: torch's scaled_dot_product_attention in float64 with an explicit
boolean mask (band, both window readings, GQA groups, sinks), or an identity
the method must keep (chunked prefill and decode reproduce one-shot prefill,
the slot map's closed form).  No GPU is used.
"""
import math

import numpy as np
import torch
from hypothesis import HealthCheck, given, settings
from hypothesis import strategies as st

SET = settings(max_examples=30, deadline=None, derandomize=True,
               suppress_health_check=[HealthCheck.function_scoped_fixture, HealthCheck.too_slow])


def _rand(shape, seed):
    return np.random.default_rng(seed).standard_normal(shape)


def _sdpa(q, k, v, scale, mask):
    """torch SDPA in float64 on [B, N, H, D] inputs with K/V heads already expanded."""
    t = lambda a: torch.from_numpy(np.ascontiguousarray(a)).permute(0, 2, 1, 3)
    with torch.no_grad():
        o = torch.nn.functional.scaled_dot_product_attention(t(q), t(k), t(v),
                                                             attn_mask=torch.from_numpy(mask), scale=scale)
    return o.permute(0, 2, 1, 3).numpy()


shapes = st.fixed_dictionaries({
    "B": st.integers(1, 2), "N": st.integers(1, 48), "Hkv": st.integers(1, 3), "G": st.integers(1, 4),
    "D": st.sampled_from([1, 2, 4, 8, 16]), "W": st.integers(1, 60), "seed": st.integers(0, 2 ** 31 - 1),
})


def _inputs(s):
    B, N, Hkv, G, D = s["B"], s["N"], s["Hkv"], s["G"], s["D"]
    r = s["seed"]
    return (_rand((B, N, Hkv * G, D), r), _rand((B, N, Hkv, D), r + 1), _rand((B, N, Hkv, D), r + 2),
            1.0 / math.sqrt(D))


@SET
@given(s=shapes, incl=st.booleans())
def test_prefill_is_sdpa_with_band_mask(oracle_mod, s, incl):
    """Query i attends to keys i-W < j <= i (or i-W <= j <= i under the
    inclusive reading); K/V head h // G serves query head h."""
    q, k, v, scale = _inputs(s)
    N, W, G = s["N"], s["W"], s["G"]
    mode = oracle_mod.WINDOW_INCL_LEFT if incl else oracle_mod.WINDOW_EXCL_LEFT
    out = oracle_mod.swa_prefill(q, k, v, W, scale, mode=mode)
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    mask = (j <= i) & ((j >= i - W) if incl else (j > i - W))
    ref = _sdpa(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), scale, mask)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


@SET
@given(s=shapes, S=st.integers(0, 50))
def test_sinks_are_sdpa_with_window_or_sink_mask(oracle_mod, s, S):
    """With S sinks query i also sees positions j < S (causal), each key once."""
    q, k, v, scale = _inputs(s)
    N, W, G = s["N"], s["W"], s["G"]
    out = oracle_mod.swa_prefill_sinks(q, k, v, W, S, scale)
    i, j = np.arange(N)[:, None], np.arange(N)[None, :]
    mask = (j <= i) & ((j > i - W) | (j < S))
    ref = _sdpa(q, np.repeat(k, G, axis=2), np.repeat(v, G, axis=2), scale, mask)
    np.testing.assert_allclose(out, ref, rtol=1e-10, atol=1e-12)


@SET
@given(s=shapes, data=st.data())
def test_chunked_prefill_reproduces_one_shot(oracle_mod, s, data):
    """Any chunk length C <= W through a W-slot buffer gives one-shot SWA, and
    leaves slot t holding the last position p < N with p mod W = t."""
    q, k, v, scale = _inputs(s)
    B, N, Hkv, D, W = s["B"], s["N"], s["Hkv"], s["D"], s["W"]
    C = data.draw(st.integers(1, W))
    one = oracle_mod.swa_prefill(q, k, v, W, scale)
    kc, vc = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    outs = []
    for s0 in range(0, N, C):
        e = min(N, s0 + C)
        st0 = np.full(B, s0, np.int32)
        outs.append(oracle_mod.swa_chunk(q[:, s0:e], k[:, s0:e], v[:, s0:e], kc, vc, sp, st0, W, scale))
        oracle_mod.cache_append(kc, vc, sp, k[:, s0:e], v[:, s0:e], st0)
    np.testing.assert_allclose(np.concatenate(outs, axis=1), one, rtol=1e-10, atol=1e-12)
    for t in range(min(W, N)):
        p = t + ((N - 1 - t) // W) * W
        assert sp[0, t] == p
        np.testing.assert_array_equal(kc[:, t], k[:, p])


@SET
@given(s=shapes)
def test_decode_reproduces_rows_of_one_shot(oracle_mod, s):
    """Appending position p, then decoding it, gives row p of one-shot SWA, for
    every p (before and after the buffer wraps)."""
    q, k, v, scale = _inputs(s)
    B, N, Hkv, D, W = s["B"], s["N"], s["Hkv"], s["D"], s["W"]
    one = oracle_mod.swa_prefill(q, k, v, W, scale)
    kc, vc = np.zeros((B, W, Hkv, D)), np.zeros((B, W, Hkv, D))
    sp = np.full((B, W), -1, np.int32)
    for p in range(N):
        pos = np.full(B, p, np.int32)
        oracle_mod.cache_append(kc, vc, sp, k[:, p:p + 1], v[:, p:p + 1], pos)
        out = oracle_mod.swa_decode(q[:, p], kc, vc, sp, pos, W, scale)
        np.testing.assert_allclose(out, one[:, p], rtol=1e-10, atol=1e-12)


@SET
@given(W=st.integers(1, 5000), counts=st.lists(st.integers(0, 40000), min_size=1, max_size=4))
def test_slot_map_closed_form(oracle_mod, W, counts):
    """After positions 0..n-1 are written, slot t holds n-1-((n-1-t) mod W) if t < n, else nothing."""
    sp = oracle_mod.slot_positions(np.array(counts, np.int32), W)
    t = np.arange(W)
    for b, n in enumerate(counts):
        expect = np.where(t < n, n - 1 - np.mod(n - 1 - t, W), -1)
        np.testing.assert_array_equal(sp[b], expect)
