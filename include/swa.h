/*
 * swa.h -- C ABI of libswa: causal sliding-window attention with grouped
 * query heads over a rolling-buffer KV cache, on NVIDIA B200 (sm_100a).
 *
 * The operations follow pages written about the Mistral 7B paper
 * (arXiv:2310.06825):
 *  - "Mistral 7B -- Sliding Window Attention" summary (irregular6612.github.io),
 *    sections "Methods", "핵심 구성요소" and "Rolling Buffer KV Cache 동작 설명";
 *  - review at manon006.tistory.com/118, sections 2.2, 3.2-3.4, 4.1 (Fig. 2, 3);
 *  - "Mistral 7B: Engineering Extreme Efficiency in LLMs" (flashpapers.ai),
 *    sections 1 (GQA), 2 (SWA equation), 3 (rolling buffer), 4 (pre-fill and
 *    chunking).
 *
 * Conventions shared by every call
 *  - Tensors are caller-owned DEVICE memory, bfloat16 (stored as uint16_t),
 *    contiguous row-major, with the shapes given per call.  Every tensor base
 *    address must be 16-byte aligned; a prefill output that is 32-byte
 *    aligned is written with 32-byte stores (same values, fewer store
 *    instructions).  The library never allocates, frees or
 *    retains them; it never synchronises a stream except in
 *    swa_get_device_status().
 *  - Positions are 0-based int32 values in DEVICE memory, so a sequence of
 *    calls can be captured in a CUDA graph and replayed with new positions.
 *    Every position a call covers (start + length - 1) must fit in int32;
 *    a negative position is recorded as SWA_ERR_INVALID_ARG in the device
 *    status word (appends, RoPE and decode then skip that sequence; chunked
 *    prefill attends as if the chunk started at position 0).
 *  - Window: query position i attends to key positions j with i-W < j <= i
 *    (W keys, itself included).  The pages print this window two ways
 *    ("[i-W, i-1]" and "j = i-W .. i"); the reading above is the one under
 *    which a W-slot buffer written at slot p mod W holds every key a query
 *    needs.  swa_prefill() also accepts the other reading, i-W <= j <= i
 *    (SWA_WINDOW_INCL_LEFT), which is the same as W+1 under the default.
 *  - Grouped-query heads: query head h reads KV head h / (Hq / Hkv)
 *    (contiguous groups; Mistral-7B: 32 query heads, 8 KV heads).
 *  - Rolling buffer: the K/V of position p live in slot p mod W of a
 *    [B, W, Hkv, D] cache; memory stays W entries whatever the length.
 *  - Supported: D in {64, 128}; Hq % Hkv == 0; W >= 1.  Arithmetic: bf16
 *    inputs, fp32 accumulation and softmax, bf16 outputs (round to nearest).
 *  - Streams: every call is asynchronous on `stream` (NULL = legacy default
 *    stream) of the current CUDA device.
 *  - Errors: argument checks run on the host before anything is launched and
 *    return SWA_ERR_INVALID_ARG or SWA_ERR_UNSUPPORTED with nothing enqueued.
 *    A failed launch returns SWA_ERR_CUDA.  Kernels never trap: each bounded
 *    wait that runs out records SWA_ERR_TIMEOUT in a device status word, the
 *    kernel releases what it holds and returns; swa_get_device_status()
 *    reports it.
 */
#ifndef SWA_H_
#define SWA_H_

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

/* Same type as cudaStream_t / CUstream. */
typedef struct CUstream_st *swa_stream_t;

typedef enum {
    SWA_OK = 0,
    SWA_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer */
    SWA_ERR_UNSUPPORTED = 2, /* valid request outside what the kernels cover */
    SWA_ERR_CUDA = 3,        /* a CUDA runtime/driver call failed */
    SWA_ERR_TIMEOUT = 4      /* a device-side bounded wait ran out */
} swa_status_t;

typedef enum {
    SWA_WINDOW_EXCL_LEFT = 0, /* keys j with i-W <  j <= i (default) */
    SWA_WINDOW_INCL_LEFT = 1  /* keys j with i-W <= j <= i */
} swa_window_mode_t;

/*
 * swa_prefill -- one-shot sliding-window GQA attention over a whole prompt.
 * Pages: the SWA mask of "핵심 구성요소" and the equation of section 2 of
 * "Engineering Extreme Efficiency"; work is O(N*W) (fully masked key tiles
 * are never visited).
 *   q, out : [B, N, Hq, D]       k, v : [B, N, Hkv, D]
 *   out[b,i,h,:] = sum_j softmax_j(scale * <q[b,i,h], k[b,j,g]>) v[b,j,g]
 *   over the window of i, g = h / (Hq/Hkv).  W >= N is dense causal.
 * window_mode: swa_window_mode_t.  scale: softmax scale, finite and > 0.
 */
swa_status_t swa_prefill(const void *q, const void *k, const void *v, void *out,
                         int B, int N, int Hq, int Hkv, int D, int W,
                         int window_mode, float scale, swa_stream_t stream);

/*
 * swa_prefill_chunk -- pre-fill one chunk of C positions through the rolling
 * buffer.  Pages: "Pre-fill + Chunking" in "Methods" and "핵심 구성요소", the
 * pre-fill paragraph of the rolling-buffer section, section 4.1 / Figure 3
 * of the review, section 4 of "Engineering Extreme Efficiency".
 *   q, out : [B, C, Hq, D]       k, v : [B, C, Hkv, D]   (this chunk)
 *   k_cache, v_cache : [B, W, Hkv, D], read and then updated in place
 *   start_pos : int32 [B] device array, position of the chunk's first token
 * Query s0+t (s0 = start_pos[b]) attends to the cached positions inside its
 * window (the cache must hold positions s0-W .. s0-1 at slot p mod W, or be
 * empty below position 0) and causally to the chunk itself.  After the
 * attention the chunk's K/V are written at slots (s0+t) mod W (attend first,
 * then write: with C = W the chunk replaces every slot).  Requires C <= W.
 */
swa_status_t swa_prefill_chunk(const void *q, const void *k, const void *v,
                               void *k_cache, void *v_cache,
                               const int32_t *start_pos, void *out, int B,
                               int C, int Hq, int Hkv, int D, int W,
                               float scale, swa_stream_t stream);

/*
 * swa_cache_append -- rolling-buffer write.  Pages: write step of
 * "Rolling Buffer KV Cache 동작 설명" (slot = p % W), section 3.3 of the
 * review, section 3 of "Engineering Extreme Efficiency".
 *   k_new, v_new : [B, T, Hkv, D]      k_cache, v_cache : [B, W, Hkv, D]
 *   pos : int32 [B] device array, position of each sequence's first new token
 * cache[b, (pos[b]+t) mod W] = new[b, t], bit for bit.  Requires T <= W so
 * that no two new tokens share a slot.  Positions must be >= 0.
 */
swa_status_t swa_cache_append(const void *k_new, const void *v_new,
                              void *k_cache, void *v_cache, const int32_t *pos,
                              int B, int T, int Hkv, int D, int W,
                              swa_stream_t stream);

/*
 * swa_decode -- one query token per sequence against the rolling buffer.
 * Pages: read step of "Rolling Buffer KV Cache 동작 설명" (a query at p reads
 * positions p-W+1 .. p, which may wrap around the buffer), section 3.4 of the
 * review (decode is bound by cache reads; GQA cuts them).
 *   q, out : [B, Hq, D]      k_cache, v_cache : [B, W, Hkv, D]
 *   pos : int32 [B] device array, position of the new token, whose K/V must
 *         already be in the cache (swa_cache_append first).
 * Each sequence reads slots 0 .. min(pos[b]+1, W)-1; softmax is order-free,
 * so the wrap needs no reordering.  Any group size Hq/Hkv (Mistral-7B: 4): the
 * query heads of a group are the rows of a tensor-core tile, up to 8 at a
 * time, so a group of G heads runs as G / Gt groups of Gt heads (Gt the
 * largest divisor of G up to 8), each reading the K/V head again; the same
 * holds for the _rope, _sinks and _noalloc forms.  Hkv * G / Gt above 65535
 * returns SWA_ERR_UNSUPPORTED.
 * workspace: device scratch of at least swa_decode_workspace_size() bytes,
 *   256-byte aligned, owned by the caller; its contents need no set-up and are
 *   overwritten.  Calls that share a workspace must not overlap on the GPU.
 *   When the window takes exactly 4 splits (without sinks) the splits are
 *   merged on chip and the workspace is left untouched; it is still checked
 *   and must still be passed.
 */
swa_status_t swa_decode(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *pos, void *out, int B, int Hq, int Hkv,
                        int D, int W, float scale, void *workspace,
                        size_t workspace_bytes, swa_stream_t stream);

/* Workspace bytes swa_decode needs for these sizes (0 if they are invalid).
 * The window is cut into splits of up to 1024 keys, smaller (down to 256)
 * when B * Hkv is small, so that a small batch still spreads over the GPU;
 * the split length, and so this size, depends on B, Hkv and W only. */
size_t swa_decode_workspace_size(int B, int Hq, int Hkv, int D, int W);

/*
 * swa_decode_noalloc -- swa_decode without a caller-provided workspace.
 * The pages have no counterpart: this is an interface convenience only.
 *
 * Some callers cannot hand the library scratch memory.  A plug-in hosted by
 * an application that owns all device memory through its own pool may not
 * call cudaMalloc at all; a latency-critical serving loop cannot afford it,
 * because cudaMalloc may synchronise the device and stall every stream; and a
 * caller that plans its memory budget once at start-up has no way to grow it
 * per request.
 * This entry point takes the same inputs and outputs as swa_decode but keeps
 * its split partials in a scratch array that the library reserves statically
 * in device memory: SWA_DECODE_NOALLOC_SCRATCH_BYTES (16 MiB) on every GPU
 * where the library is loaded, held until the process exits.  It allocates
 * nothing and calls no allocating routine.
 *
 * Limits and behaviour:
 *  - sizes whose workspace (swa_decode_workspace_size) exceeds
 *    SWA_DECODE_NOALLOC_SCRATCH_BYTES are rejected with SWA_ERR_UNSUPPORTED
 *    before anything is launched (B=64, Hq=32, D=128, W=4096 needs 4.3 MB);
 *  - the first call on a device looks up the scratch array's device address
 *    (cudaGetSymbolAddress) with that device current; make that first call
 *    before any stream capture.  The address is kept for the life of the
 *    process: resetting the device (cudaDeviceReset) after that first call is
 *    not supported, since the kept address would no longer be valid;
 *  - all calls share the one array and it keeps the last call's contents;
 *    nothing in it needs to start at zero.  Calls that overlap on the GPU
 *    (different streams, or different host threads without ordering) race on
 *    it and give wrong results: serialise them.
 */
#define SWA_DECODE_NOALLOC_SCRATCH_BYTES (16u << 20)
swa_status_t swa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *pos, void *out, int B, int Hq, int Hkv, int D,
                                int W, float scale, swa_stream_t stream);

/*
 * Variable-length batches in one launch (serving flow of pre-fill chunks and
 * decode tokens mixed, section 4.1 and 4.3 of the manon006 review).  The
 * sequences are packed: q/out [total, Hq, D], k/v [total, Hkv, D] with
 * sequence b in rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (cu_seqlens: int32
 * [B+1] device array, cu_seqlens[0] = 0, non-decreasing, cu_seqlens[B] =
 * total; empty sequences allowed).  B <= 256.  Malformed offsets are recorded
 * as SWA_ERR_INVALID_ARG in the device status word.
 */

/* swa_prefill_varlen -- one-shot prefill of each sequence (positions 0..n_b-1). */
swa_status_t swa_prefill_varlen(const void *q, const void *k, const void *v, void *out,
                                const int32_t *cu_seqlens, int B, int total, int Hq, int Hkv, int D,
                                int W, int window_mode, float scale, swa_stream_t stream);

/* swa_prefill_chunk_varlen -- one pre-fill chunk per sequence through its
 * rolling buffer (k_cache, v_cache [B, W, Hkv, D]), sequence b starting at
 * position start_pos[b].  A sequence of length 1 is a decode step (it sees
 * its own key and the W-1 positions before it), so pre-fill chunks and decode
 * tokens share one call.  Any length is accepted: a sequence longer than W
 * leaves its last W positions in the buffer.  Attend first, then write.
 * The length-1 sequences are computed by the decode kernel (reading their
 * own key and value from the packed k/v rows, heads taken as in swa_decode)
 * and the others by the prefill kernel.  Up to three kernels on `stream`. */
swa_status_t swa_prefill_chunk_varlen(const void *q, const void *k, const void *v, void *k_cache,
                                      void *v_cache, const int32_t *start_pos,
                                      const int32_t *cu_seqlens, void *out, int B, int total,
                                      int Hq, int Hkv, int D, int W, float scale,
                                      swa_stream_t stream);

/*
 * Attention sinks (StreamingLLM; aionda.blog "LLM 추론용 SWA", sections on why
 * a plain sliding window is not enough and on inference-time SWA: the first
 * few tokens -- four suffice -- keep their key/values besides the recent
 * window, the middle is dropped).  Adopted reading: query i attends to its
 * window (i-W < j <= i) and to positions j < S, each key once.  The sinks
 * live in their own buffer k_sink, v_sink [B, S, Hkv, D] (position j at slot
 * j), beside the W-slot rolling buffer.
 */

/* swa_prefill_sinks -- one-shot prefill with S sink positions (S >= 0). */
swa_status_t swa_prefill_sinks(const void *q, const void *k, const void *v, void *out, int B, int N,
                               int Hq, int Hkv, int D, int W, int S, float scale,
                               swa_stream_t stream);

/* swa_prefill_chunk_sinks -- swa_prefill_chunk with S sink positions: each
 * query at position i also attends to the sink positions j < S with
 * j <= i - W (those that have left its window), read from the sink buffers
 * k_sink / v_sink [B, S, Hkv, D], whose slot j must hold position j (written
 * by an earlier chunk of this call family or by swa_cache_append_sinks).
 * After the attention the chunk goes into the rolling buffer and its
 * positions below S into the sink buffers.  A prompt pre-filled this way
 * continues with swa_cache_append_sinks + swa_decode_sinks; the result equals
 * swa_prefill_sinks over the whole prompt.  Fixed-length batches only; errors
 * as swa_prefill_chunk, plus S < 0 or null / unaligned sink buffers with
 * S > 0 -> SWA_ERR_INVALID_ARG. */
swa_status_t swa_prefill_chunk_sinks(const void *q, const void *k, const void *v, void *k_cache,
                                     void *v_cache, void *k_sink, void *v_sink, const int32_t *start_pos,
                                     void *out, int B, int C, int Hq, int Hkv, int D, int W, int S,
                                     float scale, swa_stream_t stream);

/* swa_cache_append_sinks -- swa_cache_append that also stores new tokens
 * with position p < S at sink slot p. */
swa_status_t swa_cache_append_sinks(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                                    void *k_sink, void *v_sink, const int32_t *pos, int B, int T,
                                    int Hkv, int D, int W, int S, swa_stream_t stream);

/* swa_decode_sinks -- swa_decode plus the sink positions that have left the
 * window (j < S, j <= pos-W), read from the sink buffer.  The workspace is
 * sized by swa_decode_workspace_size(B, Hq, Hkv, D, W + S). */
swa_status_t swa_decode_sinks(const void *q, const void *k_cache, const void *v_cache,
                              const void *k_sink, const void *v_sink, const int32_t *pos, void *out,
                              int B, int Hq, int Hkv, int D, int W, int S, float scale,
                              void *workspace, size_t workspace_bytes, swa_stream_t stream);

/*
 * Rotary position embedding (RoPE).  The pages give only its base, theta =
 * 10000, in the Table 1 line of "Methods" of the "Mistral 7B -- Sliding
 * Window Attention" summary.  Adopted convention (the original RoFormer
 * pairing): adjacent elements (2i, 2i+1) of a head vector at position p turn
 * by the angle p * theta^(-2i/D):
 *   (x0, x1) -> (x0 cos a - x1 sin a, x0 sin a + x1 cos a).
 * Angles are formed and reduced in double precision; the rotation runs in
 * fp32 and rotated tensors are stored in bf16.  theta must be finite and > 1.
 */

/* swa_rope -- rotate x [B, T, H, D] (bf16, device) in place, row (b, t) at
 * position pos[b] + t (pos: int32 [B], device). */
swa_status_t swa_rope(void *x, const int32_t *pos, int B, int T, int H, int D, float theta,
                      swa_stream_t stream);

/* swa_cache_append_rope -- swa_cache_append that rotates the keys on their
 * way into the cache (the cache holds rotated keys; values are copied). */
swa_status_t swa_cache_append_rope(const void *k_new, const void *v_new, void *k_cache,
                                   void *v_cache, const int32_t *pos, int B, int T, int Hkv,
                                   int D, int W, float theta, swa_stream_t stream);

/* swa_prefill_rope -- swa_prefill with q given unrotated: each Q tile is
 * rotated (positions 0..N-1) in shared memory right after its TMA load.  k
 * must already be rotated (swa_rope).  Same arguments as swa_prefill plus
 * theta. */
swa_status_t swa_prefill_rope(const void *q, const void *k, const void *v, void *out, int B, int N,
                              int Hq, int Hkv, int D, int W, int window_mode, float scale,
                              float theta, swa_stream_t stream);

/* swa_prefill_chunk_rope -- swa_prefill_chunk with q given unrotated (rotated
 * at load, positions start_pos[b] + t); the chunk's k must already be rotated
 * and the cache holds rotated keys (swa_cache_append_rope or this call). */
swa_status_t swa_prefill_chunk_rope(const void *q, const void *k, const void *v, void *k_cache,
                                    void *v_cache, const int32_t *start_pos, void *out, int B,
                                    int C, int Hq, int Hkv, int D, int W, float scale, float theta,
                                    swa_stream_t stream);

/* swa_decode_rope -- swa_decode with q given unrotated (rotated in fp32 at
 * position pos[b] while loaded); the cache holds rotated keys. */
swa_status_t swa_decode_rope(const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *pos, void *out, int B, int Hq, int Hkv, int D, int W,
                             float scale, float theta, void *workspace, size_t workspace_bytes,
                             swa_stream_t stream);

/*
 * swa_get_device_status -- synchronise `stream`, then return (and reset to
 * SWA_OK) the device status word that kernels of this library set when a
 * bounded wait runs out.  Returns SWA_ERR_CUDA if synchronisation fails.
 */
swa_status_t swa_get_device_status(swa_stream_t stream);

/*
 * swa_set_wait_limit_ns -- limit, in nanoseconds, of every device-side wait
 * of kernels launched afterwards on the current device (default 1 s).
 * Test hook for the timeout path; 0 makes every wait that is not already
 * satisfied fail at once.
 */
swa_status_t swa_set_wait_limit_ns(unsigned long long limit_ns);

/*
 * swa_selftest_wait_timeout -- launch one block that waits on a shared-memory
 * barrier nothing arrives on, with the current wait limit.  The wait runs out,
 * the kernel records SWA_ERR_TIMEOUT and returns; read it with
 * swa_get_device_status().  Exercises the timeout path without any fault.
 */
swa_status_t swa_selftest_wait_timeout(swa_stream_t stream);

/*
 * swa_selftest_exp2 -- test hook: y[i] = 2^x[i] computed by the FMA-pipe
 * exponential the prefill kernel uses for a share of its softmax
 * (polynomial after Cody-Waite range reduction; relative error below 2e-4
 * for x >= -126; inputs below -126, -inf included, give values in
 * [0, 2^-125]).  x, y: n floats in device memory.
 */
swa_status_t swa_selftest_exp2(const float *x, float *y, int n, swa_stream_t stream);

/* Human-readable name of a status code. */
const char *swa_status_string(swa_status_t status);

/* Last CUDA error code seen by the library on this thread (0 if none). */
int swa_last_cuda_error(void);

#ifdef __cplusplus
}
#endif

#endif /* SWA_H_ */
