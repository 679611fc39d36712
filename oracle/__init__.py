"""fp64 CPU oracle for sliding-window GQA attention and the rolling-buffer cache.

TEST INFRASTRUCTURE ONLY.  The library never imports this package; only the
tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of ``bench.py`` do.
It shares no code with the CUDA path: the arithmetic lives in
``swa_oracle.c`` (plain C, double precision), compiled here with gcc.  This
module only marshals numpy arrays into that library.

Page citations for every function are in ``swa_oracle.c``.
"""
from __future__ import annotations

import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "swa_oracle.c")
_LIB_PATH = os.path.join(_HERE, "libswa_oracle.so")
_lock = threading.Lock()
_lib = None

WINDOW_EXCL_LEFT = 0  # keys j with i-W <  j <= i  (W keys, self included)
WINDOW_INCL_LEFT = 1  # keys j with i-W <= j <= i  (W+1 keys)


def build(force: bool = False) -> str:
    """Compile swa_oracle.c into libswa_oracle.so (gcc, OpenMP)."""
    stale = (not os.path.exists(_LIB_PATH)
             or os.path.getmtime(_LIB_PATH) < os.path.getmtime(_SRC))
    if force or stale:
        tmp = _LIB_PATH + f".tmp{os.getpid()}"
        subprocess.run(["gcc", "-O2", "-fopenmp", "-shared", "-fPIC", "-std=c11",
                        "-Wall", "-Wextra", _SRC, "-o", tmp, "-lm"], check=True)
        os.replace(tmp, _LIB_PATH)
    return _LIB_PATH


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = ctypes.CDLL(build())
            dp = ctypes.POINTER(ctypes.c_double)
            ip = ctypes.POINTER(ctypes.c_int32)
            lp = ctypes.POINTER(ctypes.c_int64)
            vp = ctypes.c_void_p
            i, d = ctypes.c_int, ctypes.c_double
            lib.oracle_swa_prefill.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, d, i, lp, ctypes.c_int64]
            lib.oracle_cache_append.argtypes = [vp, vp, ip, vp, vp, ip, i, i, i, i, i, i]
            lib.oracle_slot_positions.argtypes = [ip, i, i, ip]
            lib.oracle_swa_chunk.argtypes = [dp, dp, dp, dp, dp, ip, ip, dp, i, i, i, i, i, i, d, i]
            lib.oracle_swa_decode.argtypes = [dp, dp, dp, ip, ip, dp, i, i, i, i, i, d, i]
            lib.oracle_rope.argtypes = [dp, ip, i, i, i, i, d]
            lib.oracle_rope.restype = ctypes.c_int
            lib.oracle_swa_prefill_sinks.argtypes = [dp, dp, dp, dp, i, i, i, i, i, i, i, d, lp, ctypes.c_int64]
            lib.oracle_sink_append.argtypes = [vp, vp, vp, vp, ip, i, i, i, i, i, i]
            lib.oracle_swa_decode_sinks.argtypes = [dp, dp, dp, ip, dp, dp, ip, dp, i, i, i, i, i, i, d]
            for f in (lib.oracle_swa_prefill_sinks, lib.oracle_sink_append, lib.oracle_swa_decode_sinks):
                f.restype = ctypes.c_int
            for f in (lib.oracle_swa_prefill, lib.oracle_cache_append, lib.oracle_slot_positions,
                      lib.oracle_swa_chunk, lib.oracle_swa_decode):
                f.restype = ctypes.c_int
            _lib = lib
    return _lib


def _f64(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float64))


def _i32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.int32))


def _dp(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def _ip(a: np.ndarray):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_int32))


def set_threads(n: int | None) -> None:
    """Bound the OpenMP team of later oracle calls (None: leave the default)."""
    if n is not None:
        os.environ["OMP_NUM_THREADS"] = str(int(n))


def swa_prefill(q, k, v, W: int, scale: float, mode: int = WINDOW_EXCL_LEFT, rows=None) -> np.ndarray:
    """One-shot sliding-window GQA attention.

    q: [B, N, Hq, D]; k, v: [B, N, Hkv, D] (any float dtype, converted exactly
    to float64).  rows: optional 1-D sequence of query positions; the result
    is then [B, len(rows), Hq, D] instead of [B, N, Hq, D].
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    assert k.shape == (B, N, Hkv, D) and v.shape == k.shape
    if rows is None:
        out = np.empty((B, N, Hq, D), np.float64)
        rp, nr = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.empty((B, r.size, Hq, D), np.float64)
        rp, nr = r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), r.size
    rc = _load().oracle_swa_prefill(_dp(q), _dp(k), _dp(v), _dp(out), B, N, Hq, Hkv, D,
                                    int(W), float(scale), int(mode), rp, nr)
    if rc != 0:
        raise ValueError("oracle_swa_prefill: bad arguments")
    return out


def cache_append(k_cache: np.ndarray, v_cache: np.ndarray, slot_pos, k_new, v_new, pos) -> None:
    """In-place rolling-buffer write: position pos[b]+t goes to slot (pos[b]+t) mod W.

    k_cache, v_cache: [B, W, Hkv, D] contiguous arrays of any element type
    (bytes are copied unchanged); k_new, v_new: [B, T, Hkv, D] of the same
    type; slot_pos: int32 [B, W] array updated in place, or None.
    """
    B, W, Hkv, D = k_cache.shape
    T = k_new.shape[1]
    for a in (k_cache, v_cache):
        assert a.flags.c_contiguous
    kn = np.ascontiguousarray(k_new, dtype=k_cache.dtype)
    vn = np.ascontiguousarray(v_new, dtype=k_cache.dtype)
    p = _i32(pos)
    sp = None
    if slot_pos is not None:
        assert slot_pos.dtype == np.int32 and slot_pos.flags.c_contiguous
        sp = _ip(slot_pos)
    rc = _load().oracle_cache_append(k_cache.ctypes.data, v_cache.ctypes.data, sp,
                                     kn.ctypes.data, vn.ctypes.data, _ip(p),
                                     B, T, Hkv, D, W, k_cache.dtype.itemsize)
    if rc != 0:
        raise ValueError("oracle_cache_append: bad arguments")


def slot_positions(count, W: int) -> np.ndarray:
    """Slot -> logical position map after positions 0..count[b]-1 were written."""
    c = _i32(count)
    out = np.empty((c.size, W), np.int32)
    rc = _load().oracle_slot_positions(_ip(c), c.size, int(W), _ip(out))
    if rc != 0:
        raise ValueError("oracle_slot_positions: bad arguments")
    return out


def swa_chunk(q, k, v, k_cache, v_cache, slot_pos, start_pos, W: int, scale: float,
              mode: int = WINDOW_EXCL_LEFT) -> np.ndarray:
    """Chunked pre-fill attention of one chunk over [cache within window] + [chunk, causal].

    q: [B, C, Hq, D]; k, v: [B, C, Hkv, D]; k_cache, v_cache: [B, W, Hkv, D];
    slot_pos: int32 [B, W] (-1 = empty); start_pos: [B].  The cache is read
    as it is (the chunk is not written); returns [B, C, Hq, D] float64.
    """
    q, k, v = _f64(q), _f64(k), _f64(v)
    kc, vc = _f64(k_cache), _f64(v_cache)
    sp, st = _i32(slot_pos), _i32(start_pos)
    B, C, Hq, D = q.shape
    Hkv = k.shape[2]
    out = np.empty((B, C, Hq, D), np.float64)
    rc = _load().oracle_swa_chunk(_dp(q), _dp(k), _dp(v), _dp(kc), _dp(vc), _ip(sp), _ip(st),
                                  _dp(out), B, C, Hq, Hkv, D, int(W), float(scale), int(mode))
    if rc != 0:
        raise ValueError("oracle_swa_chunk: bad arguments")
    return out


def swa_decode(q, k_cache, v_cache, slot_pos, pos, W: int, scale: float,
               mode: int = WINDOW_EXCL_LEFT) -> np.ndarray:
    """Decode attention of one new token per sequence (already appended at pos[b]).

    q: [B, Hq, D]; k_cache, v_cache: [B, W, Hkv, D]; slot_pos: int32 [B, W];
    pos: [B].  Returns [B, Hq, D] float64.
    """
    q = _f64(q)
    kc, vc = _f64(k_cache), _f64(v_cache)
    sp, p = _i32(slot_pos), _i32(pos)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    out = np.empty((B, Hq, D), np.float64)
    rc = _load().oracle_swa_decode(_dp(q), _dp(kc), _dp(vc), _ip(sp), _ip(p), _dp(out),
                                   B, Hq, Hkv, D, int(W), float(scale), int(mode))
    if rc != 0:
        raise ValueError("oracle_swa_decode: bad arguments")
    return out


def rope(x, pos, theta: float = 10000.0) -> np.ndarray:
    """Rotary embedding of x [B, T, H, D] at positions pos[b] + t (adjacent
    pairs, angle p * theta^(-2i/D)); returns a new float64 array."""
    y = _f64(x).copy()
    p = _i32(pos)
    B, T, H, D = y.shape
    rc = _load().oracle_rope(_dp(y), _ip(p), B, T, H, D, float(theta))
    if rc != 0:
        raise ValueError("oracle_rope: bad arguments")
    return y


def swa_prefill_sinks(q, k, v, W: int, S: int, scale: float, rows=None) -> np.ndarray:
    """One-shot SWA with S attention-sink positions: query i sees its window
    (i-W, i] and positions j < S (j <= i).  Shapes as swa_prefill."""
    q, k, v = _f64(q), _f64(k), _f64(v)
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if rows is None:
        out = np.empty((B, N, Hq, D), np.float64)
        rp, nr = None, 0
    else:
        r = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
        out = np.empty((B, r.size, Hq, D), np.float64)
        rp, nr = r.ctypes.data_as(ctypes.POINTER(ctypes.c_int64)), r.size
    rc = _load().oracle_swa_prefill_sinks(_dp(q), _dp(k), _dp(v), _dp(out), B, N, Hq, Hkv, D,
                                          int(W), int(S), float(scale), rp, nr)
    if rc != 0:
        raise ValueError("oracle_swa_prefill_sinks: bad arguments")
    return out


def sink_append(k_sink: np.ndarray, v_sink: np.ndarray, k_new, v_new, pos) -> None:
    """In place: new tokens at positions p < S also go to sink slot p.
    k_sink, v_sink: [B, S, Hkv, D]; k_new, v_new: [B, T, Hkv, D] (same dtype)."""
    B, S, Hkv, D = k_sink.shape
    T = k_new.shape[1]
    kn = np.ascontiguousarray(k_new, dtype=k_sink.dtype)
    vn = np.ascontiguousarray(v_new, dtype=k_sink.dtype)
    rc = _load().oracle_sink_append(k_sink.ctypes.data, v_sink.ctypes.data, kn.ctypes.data, vn.ctypes.data,
                                    _ip(_i32(pos)), B, T, Hkv, D, S, k_sink.dtype.itemsize)
    if rc != 0:
        raise ValueError("oracle_sink_append: bad arguments")


def swa_decode_sinks(q, k_cache, v_cache, slot_pos, k_sink, v_sink, pos, W: int, scale: float) -> np.ndarray:
    """Decode with sinks: window keys from the rolling buffer, sink positions
    that left the window from the sink buffer [B, S, Hkv, D]."""
    q = _f64(q)
    kc, vc, ks, vs = _f64(k_cache), _f64(v_cache), _f64(k_sink), _f64(v_sink)
    sp, p = _i32(slot_pos), _i32(pos)
    B, Hq, D = q.shape
    Hkv = kc.shape[2]
    S = ks.shape[1]
    out = np.empty((B, Hq, D), np.float64)
    rc = _load().oracle_swa_decode_sinks(_dp(q), _dp(kc), _dp(vc), _ip(sp), _dp(ks), _dp(vs), _ip(p), _dp(out),
                                         B, Hq, Hkv, D, int(W), int(S), float(scale))
    if rc != 0:
        raise ValueError("oracle_swa_decode_sinks: bad arguments")
    return out
