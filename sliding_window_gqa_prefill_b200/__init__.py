"""Python binding of libswa: sliding-window GQA attention over a rolling-buffer
KV cache on B200 (sm_100a).

The binding only marshals arguments: it checks tensor dtype, shape, device
and contiguity, passes device pointers and the current CUDA stream to the C
ABI declared in ``include/swa.h``, and turns a non-OK status into an
exception.  Every step of the computation runs in the CUDA kernels of
``libswa.so``; there is no fallback.  PyTorch only provides device memory and
streams.
"""
from __future__ import annotations

import contextlib
import ctypes
import os
import subprocess
import threading

__all__ = [
    "SwaError", "build", "lib", "swa_prefill", "swa_prefill_chunk", "swa_cache_append",
    "swa_decode", "swa_decode_workspace_size", "swa_decode_noalloc", "swa_prefill_varlen",
    "swa_prefill_chunk_varlen", "swa_prefill_sinks", "swa_prefill_chunk_sinks", "swa_cache_append_sinks",
    "swa_decode_sinks", "swa_rope", "swa_get_device_status", "swa_set_wait_limit_ns",
    "swa_selftest_wait_timeout", "swa_selftest_exp2", "SWA_OK", "SWA_ERR_INVALID_ARG",
    "SWA_ERR_UNSUPPORTED", "SWA_ERR_CUDA", "SWA_ERR_TIMEOUT", "SWA_WINDOW_EXCL_LEFT",
    "SWA_WINDOW_INCL_LEFT", "bounds_checked",
]

_PKG = os.path.dirname(os.path.abspath(__file__))
_ROOT = os.path.dirname(_PKG)
LIB_PATH = os.path.join(_PKG, "libswa.so")
# the same library with every kernel index checked (SWA_BOUNDS_CHECK): a failed
# check records SWA_ERR_INVALID_ARG and skips the access; for tests and debugging
DEBUG_LIB_PATH = os.path.join(_PKG, "libswa_debug.so")
HEADER = os.path.join(_ROOT, "include", "swa.h")
_SOURCES = [os.path.join(_PKG, "csrc", f) for f in
            ("swa_api.cu", "device_common.cuh", "prefill_plan.cuh", "prefill_kernel.cuh", "decode_kernel.cuh")]

SWA_OK, SWA_ERR_INVALID_ARG, SWA_ERR_UNSUPPORTED, SWA_ERR_CUDA, SWA_ERR_TIMEOUT = 0, 1, 2, 3, 4
SWA_WINDOW_EXCL_LEFT, SWA_WINDOW_INCL_LEFT = 0, 1

NVCC_FLAGS = ["-gencode", "arch=compute_100a,code=sm_100a", "-O3", "-lineinfo", "-std=c++17",
              "-Xcompiler", "-fPIC", "-shared"]


class SwaError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        name = {0: "SWA_OK", 1: "SWA_ERR_INVALID_ARG", 2: "SWA_ERR_UNSUPPORTED", 3: "SWA_ERR_CUDA",
                4: "SWA_ERR_TIMEOUT"}.get(status, f"status {status}")
        extra = ""
        if status == SWA_ERR_CUDA and _libs:
            extra = f" (cuda error {lib().swa_last_cuda_error()})"
        super().__init__(f"{what}: {name}{extra}")


def build(force: bool = False, verbose: bool = False, debug: bool = False) -> str:
    """Compile libswa.so (debug: libswa_debug.so, index-checked) for sm_100a in
    the package directory (nvcc)."""
    path = DEBUG_LIB_PATH if debug else LIB_PATH
    stale = not os.path.exists(path) or any(
        os.path.getmtime(s) > os.path.getmtime(path) for s in _SOURCES + [HEADER])
    if force or stale:
        tmp = path + f".tmp{os.getpid()}"
        cmd = ["nvcc", *NVCC_FLAGS, *(["-DSWA_BOUNDS_CHECK"] if debug else []),
               *(["-Xptxas", "-v"] if verbose else []), "-o", tmp, os.path.join(_PKG, "csrc", "swa_api.cu")]
        subprocess.run(cmd, check=True)
        os.replace(tmp, path)
    return path


_lock = threading.Lock()
_libs = {}
# SWA_BOUNDS_CHECK=1 in the environment makes every call of the process use
# the index-checked library (as inside bounds_checked())
_use_debug = os.environ.get("SWA_BOUNDS_CHECK", "") == "1"


@contextlib.contextmanager
def bounds_checked():
    """Within the block, every call goes to libswa_debug.so, whose kernels check
    each row, slot and TMA coordinate they compute against its tensor's extent
    (a failed check records SWA_ERR_INVALID_ARG; nothing traps).  Not
    thread-safe: it switches the module-wide library."""
    global _use_debug
    prev = _use_debug
    _use_debug = True
    try:
        yield
    finally:
        _use_debug = prev


def lib() -> ctypes.CDLL:
    """The loaded libswa.so (libswa_debug.so inside bounds_checked()).  Raises
    if it has not been built."""
    path = DEBUG_LIB_PATH if _use_debug else LIB_PATH
    with _lock:
        if path not in _libs:
            if not os.path.exists(path):
                raise RuntimeError(f"{os.path.basename(path)} not built ({path}); call "
                                   "sliding_window_gqa_prefill_b200.build()")
            L = ctypes.CDLL(path)
            vp, i, f, st = ctypes.c_void_p, ctypes.c_int, ctypes.c_float, ctypes.c_void_p
            L.swa_prefill.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, st]
            L.swa_prefill_chunk.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, st]
            L.swa_cache_append.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, st]
            L.swa_decode.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, vp, ctypes.c_size_t, st]
            L.swa_decode_noalloc.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, st]
            L.swa_decode_noalloc.restype = ctypes.c_int
            L.swa_rope.argtypes = [vp, vp, i, i, i, i, f, st]
            L.swa_cache_append_rope.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, st]
            L.swa_prefill_rope.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, f, st]
            L.swa_prefill_chunk_rope.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, f, st]
            L.swa_decode_rope.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, f, f, vp, ctypes.c_size_t, st]
            for fn in (L.swa_rope, L.swa_cache_append_rope, L.swa_prefill_rope, L.swa_prefill_chunk_rope,
                       L.swa_decode_rope):
                fn.restype = ctypes.c_int
            L.swa_prefill_varlen.argtypes = [vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, st]
            L.swa_prefill_chunk_varlen.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, st]
            L.swa_prefill_varlen.restype = ctypes.c_int
            L.swa_prefill_chunk_varlen.restype = ctypes.c_int
            L.swa_prefill_sinks.argtypes = [vp, vp, vp, vp, i, i, i, i, i, i, i, f, st]
            L.swa_cache_append_sinks.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, st]
            L.swa_decode_sinks.argtypes = [vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, f, vp, ctypes.c_size_t, st]
            L.swa_prefill_chunk_sinks.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, vp, i, i, i, i, i, i, i, f, st]
            for fn in (L.swa_prefill_sinks, L.swa_cache_append_sinks, L.swa_decode_sinks,
                       L.swa_prefill_chunk_sinks):
                fn.restype = ctypes.c_int
            L.swa_decode_workspace_size.argtypes = [i, i, i, i, i]
            L.swa_decode_workspace_size.restype = ctypes.c_size_t
            L.swa_get_device_status.argtypes = [st]
            L.swa_set_wait_limit_ns.argtypes = [ctypes.c_ulonglong]
            L.swa_selftest_wait_timeout.argtypes = [st]
            L.swa_selftest_exp2.argtypes = [vp, vp, i, st]
            L.swa_selftest_exp2.restype = ctypes.c_int
            L.swa_status_string.argtypes = [i]
            L.swa_status_string.restype = ctypes.c_char_p
            L.swa_last_cuda_error.argtypes = []
            for fn in (L.swa_prefill, L.swa_prefill_chunk, L.swa_cache_append, L.swa_decode,
                       L.swa_get_device_status, L.swa_set_wait_limit_ns,
                       L.swa_selftest_wait_timeout, L.swa_last_cuda_error):
                fn.restype = ctypes.c_int
            _libs[path] = L
    return _libs[path]


def _check(status: int, what: str) -> None:
    if status != SWA_OK:
        raise SwaError(status, what)


def _stream_handle(stream=None) -> int:
    import torch
    s = torch.cuda.current_stream() if stream is None else stream
    return int(s.cuda_stream)


def _bf16(t, name: str, shape=None):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda:
        raise TypeError(f"{name}: expected a CUDA tensor")
    if t.dtype != torch.bfloat16:
        raise TypeError(f"{name}: expected bfloat16, got {t.dtype}")
    if not t.is_contiguous():
        raise ValueError(f"{name}: must be contiguous")
    if shape is not None and tuple(t.shape) != tuple(shape):
        raise ValueError(f"{name}: expected shape {tuple(shape)}, got {tuple(t.shape)}")
    return t.data_ptr()


def _i32(t, name: str, n: int):
    import torch
    if not isinstance(t, torch.Tensor) or not t.is_cuda or t.dtype != torch.int32:
        raise TypeError(f"{name}: expected an int32 CUDA tensor")
    if not t.is_contiguous() or t.numel() != n:
        raise ValueError(f"{name}: expected {n} contiguous int32 values")
    return t.data_ptr()


def swa_prefill(q, k, v, W: int, scale: float, out=None, window_mode: int = SWA_WINDOW_EXCL_LEFT,
                stream=None, rope_theta: float | None = None):
    """One-shot SWA prefill.  q [B,N,Hq,D], k/v [B,N,Hkv,D] bf16 -> out [B,N,Hq,D].

    rope_theta: if given, q is unrotated and gets the rotary embedding inside
    the kernel (swa_prefill_rope); k must already be rotated."""
    import torch
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    args = (_bf16(q, "q"), _bf16(k, "k", (B, N, Hkv, D)), _bf16(v, "v", (B, N, Hkv, D)),
            _bf16(out, "out", (B, N, Hq, D)), B, N, Hq, Hkv, D, int(W), int(window_mode), float(scale))
    if rope_theta is None:
        _check(lib().swa_prefill(*args, _stream_handle(stream)), "swa_prefill")
    else:
        _check(lib().swa_prefill_rope(*args, float(rope_theta), _stream_handle(stream)), "swa_prefill_rope")
    return out


def swa_prefill_chunk(q, k, v, k_cache, v_cache, start_pos, W: int, scale: float, out=None,
                      stream=None, rope_theta: float | None = None):
    """Chunked prefill of one chunk through the rolling buffer (updates the cache).

    rope_theta: if given, q is unrotated (rotated in the kernel); k must already
    be rotated and the cache holds rotated keys (swa_prefill_chunk_rope)."""
    import torch
    B, C, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    args = (_bf16(q, "q"), _bf16(k, "k", (B, C, Hkv, D)), _bf16(v, "v", (B, C, Hkv, D)),
            _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
            _i32(start_pos, "start_pos", B), _bf16(out, "out", (B, C, Hq, D)), B, C, Hq, Hkv, D, int(W),
            float(scale))
    if rope_theta is None:
        _check(lib().swa_prefill_chunk(*args, _stream_handle(stream)), "swa_prefill_chunk")
    else:
        _check(lib().swa_prefill_chunk_rope(*args, float(rope_theta), _stream_handle(stream)),
               "swa_prefill_chunk_rope")
    return out


def swa_cache_append(k_new, v_new, k_cache, v_cache, pos, stream=None,
                     rope_theta: float | None = None) -> None:
    """Write k_new/v_new [B,T,Hkv,D] at slots (pos[b]+t) mod W of the caches [B,W,Hkv,D].

    rope_theta: if given, the keys are rotated on the way in (swa_cache_append_rope)."""
    B, T, Hkv, D = k_new.shape
    W = k_cache.shape[1]
    args = (_bf16(k_new, "k_new"), _bf16(v_new, "v_new", (B, T, Hkv, D)),
            _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
            _i32(pos, "pos", B), B, T, Hkv, D, W)
    if rope_theta is None:
        _check(lib().swa_cache_append(*args, _stream_handle(stream)), "swa_cache_append")
    else:
        _check(lib().swa_cache_append_rope(*args, float(rope_theta), _stream_handle(stream)),
               "swa_cache_append_rope")


def swa_rope(x, pos, theta: float = 10000.0, stream=None):
    """Rotate x [B,T,H,D] (bf16, CUDA) in place at positions pos[b]+t; returns x."""
    B, T, H, D = x.shape
    _check(lib().swa_rope(_bf16(x, "x"), _i32(pos, "pos", B), B, T, H, D, float(theta),
                          _stream_handle(stream)), "swa_rope")
    return x


def swa_decode_workspace_size(B: int, Hq: int, Hkv: int, D: int, W: int) -> int:
    return int(lib().swa_decode_workspace_size(B, Hq, Hkv, D, W))


def swa_decode(q, k_cache, v_cache, pos, scale: float, out=None, workspace=None, stream=None,
               rope_theta: float | None = None):
    """Decode one token per sequence.  q [B,Hq,D]; caches [B,W,Hkv,D]; pos int32 [B].

    rope_theta: if given, q is unrotated and rotated at pos[b] in the kernel
    (swa_decode_rope); the cache must hold rotated keys."""
    import torch
    B, Hq, D = q.shape
    W, Hkv = k_cache.shape[1], k_cache.shape[2]
    if out is None:
        out = torch.empty_like(q)
    need = swa_decode_workspace_size(B, Hq, Hkv, D, W)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    head = (_bf16(q, "q"), _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
            _i32(pos, "pos", B), _bf16(out, "out", (B, Hq, D)), B, Hq, Hkv, D, W, float(scale))
    tail = (workspace.data_ptr(), workspace.numel() * workspace.element_size(), _stream_handle(stream))
    if rope_theta is None:
        _check(lib().swa_decode(*head, *tail), "swa_decode")
    else:
        _check(lib().swa_decode_rope(*head, float(rope_theta), *tail), "swa_decode_rope")
    return out


def swa_decode_noalloc(q, k_cache, v_cache, pos, scale: float, out, stream=None):
    """Decode like swa_decode with the split partials in the library's static
    device scratch (SWA_DECODE_NOALLOC_SCRATCH_BYTES): nothing is allocated, so
    out [B,Hq,D] must be given.  Calls that overlap on the GPU share that one
    scratch array and race: serialise them."""
    B, Hq, D = q.shape
    W, Hkv = k_cache.shape[1], k_cache.shape[2]
    _check(lib().swa_decode_noalloc(
        _bf16(q, "q"), _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
        _i32(pos, "pos", B), _bf16(out, "out", (B, Hq, D)), B, Hq, Hkv, D, W, float(scale), _stream_handle(stream)),
        "swa_decode_noalloc")
    return out


def swa_get_device_status(stream=None) -> int:
    """Synchronise the stream and return (and reset) the device status word."""
    return int(lib().swa_get_device_status(_stream_handle(stream)))


def swa_set_wait_limit_ns(limit_ns: int) -> None:
    _check(lib().swa_set_wait_limit_ns(int(limit_ns)), "swa_set_wait_limit_ns")


def swa_selftest_exp2(x, stream=None):
    """2^x by the prefill kernel's FMA-pipe exponential (test hook); x float32 CUDA."""
    import torch
    if not (isinstance(x, torch.Tensor) and x.is_cuda and x.dtype == torch.float32 and x.is_contiguous()):
        raise TypeError("x: expected a contiguous float32 CUDA tensor")
    y = torch.empty_like(x)
    _check(lib().swa_selftest_exp2(x.data_ptr(), y.data_ptr(), x.numel(), _stream_handle(stream)),
           "swa_selftest_exp2")
    return y


def swa_selftest_wait_timeout(stream=None) -> None:
    _check(lib().swa_selftest_wait_timeout(_stream_handle(stream)), "swa_selftest_wait_timeout")


def swa_prefill_varlen(q, k, v, cu_seqlens, W: int, scale: float, out=None,
                       window_mode: int = SWA_WINDOW_EXCL_LEFT, stream=None):
    """One-shot prefill of a packed variable-length batch.  q [total,Hq,D],
    k/v [total,Hkv,D] bf16; cu_seqlens int32 CUDA [B+1]."""
    import torch
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    _check(lib().swa_prefill_varlen(_bf16(q, "q"), _bf16(k, "k", (total, Hkv, D)), _bf16(v, "v", (total, Hkv, D)),
                                    _bf16(out, "out", (total, Hq, D)), _i32(cu_seqlens, "cu_seqlens", B + 1),
                                    B, total, Hq, Hkv, D, int(W), int(window_mode), float(scale),
                                    _stream_handle(stream)), "swa_prefill_varlen")
    return out


def swa_prefill_chunk_varlen(q, k, v, k_cache, v_cache, start_pos, cu_seqlens, W: int, scale: float,
                             out=None, stream=None):
    """One chunk per sequence of a packed batch through the rolling buffers
    [B,W,Hkv,D]; a length-1 sequence is a decode step.  Updates the caches."""
    import torch
    total, Hq, D = q.shape
    Hkv = k.shape[1]
    B = cu_seqlens.numel() - 1
    if out is None:
        out = torch.empty_like(q)
    _check(lib().swa_prefill_chunk_varlen(
        _bf16(q, "q"), _bf16(k, "k", (total, Hkv, D)), _bf16(v, "v", (total, Hkv, D)),
        _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
        _i32(start_pos, "start_pos", B), _i32(cu_seqlens, "cu_seqlens", B + 1), _bf16(out, "out", (total, Hq, D)),
        B, total, Hq, Hkv, D, int(W), float(scale), _stream_handle(stream)), "swa_prefill_chunk_varlen")
    return out


def swa_prefill_sinks(q, k, v, W: int, S: int, scale: float, out=None, stream=None):
    """One-shot prefill where positions j < S stay visible beside each window."""
    import torch
    B, N, Hq, D = q.shape
    Hkv = k.shape[2]
    if out is None:
        out = torch.empty_like(q)
    _check(lib().swa_prefill_sinks(_bf16(q, "q"), _bf16(k, "k", (B, N, Hkv, D)), _bf16(v, "v", (B, N, Hkv, D)),
                                   _bf16(out, "out", (B, N, Hq, D)), B, N, Hq, Hkv, D, int(W), int(S), float(scale),
                                   _stream_handle(stream)), "swa_prefill_sinks")
    return out


def swa_prefill_chunk_sinks(q, k, v, k_cache, v_cache, k_sink, v_sink, start_pos, W: int, scale: float,
                            out=None, stream=None):
    """Chunked prefill of one chunk with the sink positions that left each
    query's window read from the sink buffers [B,S,Hkv,D]; updates the cache
    and the sink buffers (swa_prefill_chunk_sinks)."""
    import torch
    B, C, Hq, D = q.shape
    Hkv, S = k.shape[2], k_sink.shape[1]
    if out is None:
        out = torch.empty_like(q)
    _check(lib().swa_prefill_chunk_sinks(
        _bf16(q, "q"), _bf16(k, "k", (B, C, Hkv, D)), _bf16(v, "v", (B, C, Hkv, D)),
        _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
        _bf16(k_sink, "k_sink", (B, S, Hkv, D)), _bf16(v_sink, "v_sink", (B, S, Hkv, D)),
        _i32(start_pos, "start_pos", B), _bf16(out, "out", (B, C, Hq, D)), B, C, Hq, Hkv, D, int(W), int(S),
        float(scale), _stream_handle(stream)), "swa_prefill_chunk_sinks")
    return out


def swa_cache_append_sinks(k_new, v_new, k_cache, v_cache, k_sink, v_sink, pos, stream=None) -> None:
    """Rolling-buffer write that also keeps positions < S in the sink buffers [B,S,Hkv,D]."""
    B, T, Hkv, D = k_new.shape
    W, S = k_cache.shape[1], k_sink.shape[1]
    _check(lib().swa_cache_append_sinks(
        _bf16(k_new, "k_new"), _bf16(v_new, "v_new", (B, T, Hkv, D)), _bf16(k_cache, "k_cache", (B, W, Hkv, D)),
        _bf16(v_cache, "v_cache", (B, W, Hkv, D)), _bf16(k_sink, "k_sink", (B, S, Hkv, D)),
        _bf16(v_sink, "v_sink", (B, S, Hkv, D)), _i32(pos, "pos", B), B, T, Hkv, D, W, S,
        _stream_handle(stream)), "swa_cache_append_sinks")


def swa_decode_sinks(q, k_cache, v_cache, k_sink, v_sink, pos, scale: float, out=None, workspace=None,
                     stream=None):
    """Decode over the window plus the sink positions that left it."""
    import torch
    B, Hq, D = q.shape
    W, Hkv = k_cache.shape[1], k_cache.shape[2]
    S = k_sink.shape[1]
    if out is None:
        out = torch.empty_like(q)
    need = swa_decode_workspace_size(B, Hq, Hkv, D, W + S)
    if workspace is None:
        workspace = torch.empty(max(need, 256), dtype=torch.uint8, device=q.device)
    _check(lib().swa_decode_sinks(
        _bf16(q, "q"), _bf16(k_cache, "k_cache", (B, W, Hkv, D)), _bf16(v_cache, "v_cache", (B, W, Hkv, D)),
        _bf16(k_sink, "k_sink", (B, S, Hkv, D)), _bf16(v_sink, "v_sink", (B, S, Hkv, D)), _i32(pos, "pos", B),
        _bf16(out, "out", (B, Hq, D)), B, Hq, Hkv, D, W, S, float(scale), workspace.data_ptr(),
        workspace.numel() * workspace.element_size(), _stream_handle(stream)), "swa_decode_sinks")
    return out
