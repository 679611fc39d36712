// decode_kernel.cuh -- split-KV single-token decode over the rolling buffer,
// and the rolling-buffer append/scatter.
//
// Decode: one new query token per sequence b at position pos[b], whose K/V
// were already appended at slot pos[b] mod W.  The window (pos-W, pos] is
// exactly the slots 0 .. L-1, L = min(pos+1, W) (read step of "Rolling Buffer
// KV Cache 동작 설명", "Mistral 7B -- Sliding Window Attention" summary).
// Softmax over a set of keys does not depend on their order, so the wrapped
// buffer is read front to back with no reordering.  The query heads of one
// GQA group read each K/V row once (section 3.4 of the manon006 review: GQA
// cuts decode's cache reads).
//
// Memory-bound design (CUDA cores; the contraction is 4 x D per key, far
// below what tensor cores need to pay off):
//  * grid (split, kv head, sequence); a block of 4 warps streams one split of
//    up to SPLIT keys.  Each lane owns 8 consecutive d of a key row, so a
//    key row is read by D/8 lanes with 16-byte coalesced copies.
//  * cp.async 16-byte copies into a per-warp 4-stage shared-memory ring keep
//    several KB per warp in flight.
//  * per key: partial dot products for all G heads of the group, reduced
//    across the D/8 lanes of the row by a transposing butterfly (each level
//    halves the values a lane holds), so a key x head score costs about one
//    shuffle.  Online softmax per head in base 2 (scale folded into q); the
//    exponent offset of a head is raised (exact maximum over the iteration,
//    rescale of l and o) only when a score exceeds it by more than 2^8, so
//    most iterations skip the per-iteration maximum entirely.
//  * warps and splits are merged by log-sum-exp: in shared memory inside a
//    block, and by swa_decode_combine_kernel across splits.
#pragma once

#include "device_common.cuh"

namespace swa {

constexpr int kDecodeSplit = 512;      // keys per block
constexpr int kDecodeWarps = 4;
constexpr int kDecodeStages = 4;

__host__ __device__ constexpr int ilog2c(int x) { return x <= 1 ? 0 : 1 + ilog2c(x >> 1); }

template <int D, int G>
struct DecodeCfg {
    static constexpr int LPR = D / 8;                 // lanes per key row
    static constexpr int R = 32 / LPR;                // key rows per warp-wide load
    static constexpr int KPR = 4;                     // keys per row group per iteration
    static constexpr int KI = R * KPR;                // keys per warp iteration
    static constexpr int NV = KPR * G;                // partial sums per lane
    static constexpr int TLEV = (ilog2c(NV) < ilog2c(LPR)) ? ilog2c(NV) : ilog2c(LPR);
    static constexpr int VPL = NV >> TLEV;            // values per lane after the butterfly
    static constexpr int STAGE_BYTES = 2 * KI * D * 2;   // K and V rows of one iteration
    static constexpr int WARP_RING = kDecodeStages * STAGE_BYTES;
    static constexpr int OFF_SCORE = kDecodeWarps * WARP_RING;   // per warp [KI][G] floats
    static constexpr int OFF_MERGE = OFF_SCORE + kDecodeWarps * KI * G * 4;
    static constexpr int MERGE_BYTES = kDecodeWarps * G * (D + 2) * 4;
    static constexpr int SMEM_BYTES = OFF_MERGE + MERGE_BYTES;
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(G >= 1 && G <= 8 && (G & (G - 1)) == 0, "group size 1, 2, 4 or 8");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// G consecutive floats of shared memory, vectorised where G allows.
template <int G>
__device__ __forceinline__ void load_g(const float *p, float (&out)[G]) {
    if constexpr (G % 4 == 0) {
#pragma unroll
        for (int i = 0; i < G / 4; ++i) {
            const float4 t = reinterpret_cast<const float4 *>(p)[i];
            out[4 * i] = t.x;
            out[4 * i + 1] = t.y;
            out[4 * i + 2] = t.z;
            out[4 * i + 3] = t.w;
        }
    } else if constexpr (G == 2) {
        const float2 t = *reinterpret_cast<const float2 *>(p);
        out[0] = t.x;
        out[1] = t.y;
    } else {
        out[0] = p[0];
    }
}

__device__ __forceinline__ void bf16x8_to_f32(const uint4 &v, float (&f)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
        f[2 * i] = __uint_as_float(w[i] << 16);
        f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
}

// Partial result of one (sequence, kv head, split): per head m (base-2 max),
// l (sum of 2^(s-m)) and o[D] (sum of 2^(s-m) v).  Layout in the workspace:
// ml[((b*Hkv + g)*nsplit_max + s)*G + h] = {m, l};  o[...*D + d].
// SINKS: keys past the window's come from the sink buffer (attention sinks);
// compiled out of the plain decode.
template <int D, int G, bool SINKS>
__global__ void __launch_bounds__(kDecodeWarps * 32)
swa_decode_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kc,
                  const __nv_bfloat16 *__restrict__ vc, const int32_t *__restrict__ pos,
                  __nv_bfloat16 *__restrict__ out, float2 *__restrict__ ws_ml,
                  float *__restrict__ ws_o, int Hkv, int W, int nsplit_max, float scale_log2,
                  int rope, const RopeTable rope_freq, const __nv_bfloat16 *__restrict__ ksink,
                  const __nv_bfloat16 *__restrict__ vsink, int S) {
    using Cfg = DecodeCfg<D, G>;
    constexpr int LPR = Cfg::LPR, KPR = Cfg::KPR, KI = Cfg::KI, NV = Cfg::NV;
    constexpr int TLEV = Cfg::TLEV, VPL = Cfg::VPL;
    extern __shared__ __align__(128) uint8_t smem[];

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int Hq = Hkv * G;
    const int p = __ldg(pos + b);
    if (p < 0) {                                    // invalid position: record, write nothing
        if (threadIdx.x == 0 && split == 0 && g == 0) record_status(kStatusInvalid);
        return;
    }
    const int Lw = (p >= W - 1) ? W : p + 1;           // keys in the rolling buffer
    // sink positions that left the window: slots 0 .. ns-1 of the sink buffer,
    // numbered after the window's keys
    const int ns = (SINKS && S > 0 && p >= W) ? min(S, p - W + 1) : 0;
    const int L = Lw + ns;
    const int begin = split * kDecodeSplit;
    if (begin >= L) return;
    const int end = min(L, begin + kDecodeSplit);
    const int nsplit = (L + kDecodeSplit - 1) / kDecodeSplit;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int row = lane / LPR;             // row group of this lane
    const int sub = lane % LPR;             // which 8 d of the row
    const uint32_t ring = smem_addr(smem + warp * Cfg::WARP_RING);
    float *score = reinterpret_cast<float *>(smem + Cfg::OFF_SCORE) + warp * KI * G;

    // q for every head of the group, d = sub*8 .. sub*8+7, pre-scaled to base 2,
    // as four (even, odd) pairs for the packed two-lane FMA
    float2 q2[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        const uint4 raw = __ldg(reinterpret_cast<const uint4 *>(q + ((size_t)b * Hq + g * G + h) * D) + sub);
        float qf[8];
        bf16x8_to_f32(raw, qf);
        if (rope) {            // rotary embedding of the query at its position, in fp32
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                float c, sn;
                rope_cos_sin((double)p, rope_freq.f[sub * 4 + e], c, sn);
                const float x0 = qf[2 * e], x1 = qf[2 * e + 1];
                qf[2 * e] = x0 * c - x1 * sn;
                qf[2 * e + 1] = x0 * sn + x1 * c;
            }
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) q2[h][e] = make_float2(qf[2 * e] * scale_log2, qf[2 * e + 1] * scale_log2);
    }

    const size_t row_stride = (size_t)Hkv * D;     // elements between consecutive slots
    const __nv_bfloat16 *kbase = kc + ((size_t)b * W * Hkv + g) * D + sub * 8;
    const __nv_bfloat16 *vbase = vc + ((size_t)b * W * Hkv + g) * D + sub * 8;
    const __nv_bfloat16 *ksbase = ns ? ksink + ((size_t)b * S * Hkv + g) * D + sub * 8 : kbase;
    const __nv_bfloat16 *vsbase = ns ? vsink + ((size_t)b * S * Hkv + g) * D + sub * 8 : vbase;

    const int n_iter_total = (end - begin + KI - 1) / KI;
    const int my_iters = (n_iter_total > warp) ? (n_iter_total - warp + kDecodeWarps - 1) / kDecodeWarps : 0;

    // stage layout: K rows [KI][D] then V rows [KI][D]
    auto issue = [&](int it_local, int stage) {
        const int it = warp + it_local * kDecodeWarps;
        const uint32_t st = ring + stage * Cfg::STAGE_BYTES;
#pragma unroll
        for (int kk = 0; kk < KPR; ++kk) {
            const int kr = row * KPR + kk;
            const int key = min(begin + it * KI + kr, end - 1);      // clamp: always in bounds
            const uint32_t off = (uint32_t)((kr * D + sub * 8) * 2);
            if (SINKS) {
                const bool sink = key >= Lw;
                const size_t rowi = (size_t)(sink ? key - Lw : key) * row_stride;
                cp_async16(st + off, (sink ? ksbase : kbase) + rowi);
                cp_async16(st + KI * D * 2 + off, (sink ? vsbase : vbase) + rowi);
            } else {
                cp_async16(st + off, kbase + (size_t)key * row_stride);
                cp_async16(st + KI * D * 2 + off, vbase + (size_t)key * row_stride);
            }
        }
    };

    // m_run: running base-2 maximum per head (equal in all lanes);
    // l_run: this lane's share of the running sum per head (each key x head
    // is counted by exactly one lane); o2: this lane's row-group partial of
    // the output for its 8 d, per head
    float m_run[G], l_run[G];
    float2 o2[G][4];
#pragma unroll
    for (int h = 0; h < G; ++h) {
        m_run[h] = -INFINITY;
        l_run[h] = 0.f;
#pragma unroll
        for (int e = 0; e < 4; ++e) o2[h][e] = make_float2(0.f, 0.f);
    }

#pragma unroll
    for (int s = 0; s < kDecodeStages - 1; ++s) {
        if (s < my_iters) issue(s, s);
        cp_async_commit();
    }

    // value index of v[i] after the butterfly = vidx0 + i; lanes that only
    // hold copies (when NV < LPR) do not write
    int vidx0 = 0;
    {
        int half = NV;
#pragma unroll
        for (int lev = 0; lev < TLEV; ++lev) {
            half >>= 1;
            const int off = LPR >> (lev + 1);
            if (sub & off) vidx0 += half;
        }
    }
    const bool writer = (TLEV == ilog2c(LPR)) || ((sub & ((LPR >> TLEV) - 1)) == 0);

    for (int it_local = 0; it_local < my_iters; ++it_local) {
        const int stage = it_local % kDecodeStages;
        cp_async_wait<kDecodeStages - 2>();
        __syncwarp();
        {
            const int nxt = it_local + kDecodeStages - 1;
            if (nxt < my_iters) issue(nxt, nxt % kDecodeStages);
            cp_async_commit();
        }
        const uint8_t *st = smem + warp * Cfg::WARP_RING + stage * Cfg::STAGE_BYTES;
        const int it = warp + it_local * kDecodeWarps;
        const int key_base = begin + it * KI;

        // partial dot products over this lane's 8 d: value index kk*G + h
        float v[NV];
#pragma unroll
        for (int kk = 0; kk < KPR; ++kk) {
            const int kr = row * KPR + kk;
            float kf[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(st + (kr * D + sub * 8) * 2), kf);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                float2 acc = make_float2(0.f, 0.f);
#pragma unroll
                for (int e = 0; e < 4; ++e) acc = ffma2(q2[h][e], make_float2(kf[2 * e], kf[2 * e + 1]), acc);
                v[kk * G + h] = acc.x + acc.y;
            }
        }
        // transposing butterfly across the LPR lanes of the row
#pragma unroll
        for (int lev = 0; lev < ilog2c(LPR); ++lev) {
            const int off = LPR >> (lev + 1);
            if (lev < TLEV) {
                const int half = NV >> (lev + 1);
                const bool upper = (sub & off) != 0;
#pragma unroll
                for (int i = 0; i < NV / 2; ++i) {
                    if (i < half) {
                        const float send = upper ? v[i] : v[i + half];
                        const float keep = upper ? v[i + half] : v[i];
                        v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
                    }
                }
            } else {
#pragma unroll
                for (int i = 0; i < VPL; ++i) v[i] += __shfl_xor_sync(0xffffffffu, v[i], off);
            }
        }
        // keys past the split masked; a score more than 2^8 above the running
        // offset of its head (always so on the first iteration) makes the warp
        // take the exact maximum over the iteration and rescale; otherwise the
        // offset stays (p = 2^(s - offset) <= 2^8, exact after normalisation)
        bool big = false;
        if (writer) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int idx = vidx0 + i;
                const int kr = row * KPR + idx / G, h = idx % G;
                v[i] = (key_base + kr < end) ? v[i] : -INFINITY;
                float mh = m_run[0];
#pragma unroll
                for (int hh = 1; hh < G; ++hh) mh = (h == hh) ? m_run[hh] : mh;
                big |= v[i] > mh + 8.0f;
            }
        }
        if (__any_sync(0xffffffffu, big)) {
            if (writer) {
#pragma unroll
                for (int i = 0; i < VPL; ++i) {
                    const int idx = vidx0 + i;
                    score[(row * KPR + idx / G) * G + idx % G] = v[i];
                }
            }
            __syncwarp();
            float m_new[G];
#pragma unroll
            for (int h = 0; h < G; ++h) m_new[h] = m_run[h];
#pragma unroll
            for (int kr = 0; kr < KI; ++kr) {
                float sv[G];
                load_g<G>(score + kr * G, sv);
#pragma unroll
                for (int h = 0; h < G; ++h) m_new[h] = fmaxf(m_new[h], sv[h]);
            }
            __syncwarp();                        // every lane has read the scores
#pragma unroll
            for (int h = 0; h < G; ++h) {
                if (m_new[h] > m_run[h]) {       // uniform across the warp
                    const float alpha = ex2_approx(m_run[h] - m_new[h]);   // 0 when m_run = -inf
                    l_run[h] *= alpha;
#pragma unroll
                    for (int e = 0; e < 4; ++e) o2[h][e] = make_float2(o2[h][e].x * alpha, o2[h][e].y * alpha);
                    m_run[h] = m_new[h];
                }
            }
        }
        // one exponential per key x head, by the lane that holds it
        if (writer) {
#pragma unroll
            for (int i = 0; i < VPL; ++i) {
                const int idx = vidx0 + i;
                const int kr = row * KPR + idx / G, h = idx % G;
                float mh = m_run[0];
#pragma unroll
                for (int hh = 1; hh < G; ++hh) mh = (h == hh) ? m_run[hh] : mh;
                const float pw = ex2_approx(v[i] - mh);
#pragma unroll
                for (int hh = 0; hh < G; ++hh) l_run[hh] += (h == hh) ? pw : 0.f;
                score[kr * G + h] = pw;
            }
        }
        __syncwarp();
        // P V for the KPR keys of this lane's row
#pragma unroll
        for (int kk = 0; kk < KPR; ++kk) {
            const int kr = row * KPR + kk;
            float vf[8];
            bf16x8_to_f32(*reinterpret_cast<const uint4 *>(st + KI * D * 2 + (kr * D + sub * 8) * 2), vf);
            float pw[G];
            load_g<G>(score + kr * G, pw);
#pragma unroll
            for (int h = 0; h < G; ++h) {
                const float2 p2 = make_float2(pw[h], pw[h]);
#pragma unroll
                for (int e = 0; e < 4; ++e) o2[h][e] = ffma2(p2, make_float2(vf[2 * e], vf[2 * e + 1]), o2[h][e]);
            }
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    // merge within the warp: o over the row groups (lanes with equal sub),
    // l over every lane
#pragma unroll
    for (int off = LPR; off < 32; off <<= 1) {
#pragma unroll
        for (int h = 0; h < G; ++h)
#pragma unroll
            for (int e = 0; e < 4; ++e) {
                o2[h][e].x += __shfl_xor_sync(0xffffffffu, o2[h][e].x, off);
                o2[h][e].y += __shfl_xor_sync(0xffffffffu, o2[h][e].y, off);
            }
    }
#pragma unroll
    for (int off = 1; off < 32; off <<= 1)
#pragma unroll
        for (int h = 0; h < G; ++h) l_run[h] += __shfl_xor_sync(0xffffffffu, l_run[h], off);
    float o[G][8];
#pragma unroll
    for (int h = 0; h < G; ++h)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            o[h][2 * e] = o2[h][e].x;
            o[h][2 * e + 1] = o2[h][e].y;
        }
    // merge the warps of the block in shared memory
    float *mg = reinterpret_cast<float *>(smem + Cfg::OFF_MERGE);    // [warp][G][D+2]
    if (row == 0) {
#pragma unroll
        for (int h = 0; h < G; ++h) {
            float *dst = mg + (warp * G + h) * (D + 2);
#pragma unroll
            for (int e = 0; e < 8; ++e) dst[sub * 8 + e] = o[h][e];
            if (sub == 0) {
                dst[D] = m_run[h];
                dst[D + 1] = l_run[h];
            }
        }
    }
    __syncthreads();
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, d = idx % D;
        float m = -INFINITY;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) m = fmaxf(m, mg[(w * G + h) * (D + 2) + D]);
        float l = 0.f, acc = 0.f;
#pragma unroll
        for (int w = 0; w < kDecodeWarps; ++w) {
            const float *src = mg + (w * G + h) * (D + 2);
            const float sc = (src[D] == -INFINITY) ? 0.f : ex2_approx(src[D] - m);
            l += src[D + 1] * sc;
            acc += src[d] * sc;
        }
        if (nsplit == 1) {
            out[((size_t)b * Hq + g * G + h) * D + d] = __float2bfloat16_rn(acc / l);
        } else {
            const size_t slot = ((size_t)(b * Hkv + g) * nsplit_max + split) * G + h;
            ws_o[slot * D + d] = acc;
            if (d == 0) ws_ml[slot] = make_float2(m, l);
        }
    }
}

// Log-sum-exp merge of the splits of each (sequence, kv head) into bf16 out.
template <int D, int G>
__global__ void __launch_bounds__(1024)
swa_decode_combine_kernel(const int32_t *__restrict__ pos, const float2 *__restrict__ ws_ml,
                          const float *__restrict__ ws_o, __nv_bfloat16 *__restrict__ out,
                          int Hkv, int W, int nsplit_max, int S) {
    const int g = blockIdx.x, b = blockIdx.y;
    const int Hq = Hkv * G;
    const int p = __ldg(pos + b);
    if (p < 0) return;
    const int ns = (S > 0 && p >= W) ? min(S, p - W + 1) : 0;
    const int L = ((p >= W - 1) ? W : p + 1) + ns;
    const int nsplit = (L + kDecodeSplit - 1) / kDecodeSplit;
    if (nsplit <= 1) return;
    const size_t base = (size_t)(b * Hkv + g) * nsplit_max;
    constexpr int kUnrolled = 16;            // splits loaded side by side (W <= 8192)
    for (int idx = threadIdx.x; idx < G * D; idx += blockDim.x) {
        const int h = idx / D, d = idx % D;
        float m = -INFINITY, l = 0.f, acc = 0.f;
        if (nsplit <= kUnrolled) {
            float ms[kUnrolled], ls[kUnrolled], os[kUnrolled];
#pragma unroll
            for (int s = 0; s < kUnrolled; ++s) {
                if (s < nsplit) {
                    const float2 ml = ws_ml[(base + s) * G + h];
                    ms[s] = ml.x;
                    ls[s] = ml.y;
                    os[s] = ws_o[((base + s) * G + h) * D + d];
                } else {
                    ms[s] = -INFINITY;
                    ls[s] = 0.f;
                    os[s] = 0.f;
                }
            }
#pragma unroll
            for (int s = 0; s < kUnrolled; ++s) m = fmaxf(m, ms[s]);
#pragma unroll
            for (int s = 0; s < kUnrolled; ++s) {
                const float sc = (s < nsplit) ? ex2_approx(ms[s] - m) : 0.f;
                l += ls[s] * sc;
                acc += os[s] * sc;
            }
        } else {
            for (int s = 0; s < nsplit; ++s) m = fmaxf(m, ws_ml[(base + s) * G + h].x);
            for (int s = 0; s < nsplit; ++s) {
                const float2 ml = ws_ml[(base + s) * G + h];
                const float sc = ex2_approx(ml.x - m);
                l += ml.y * sc;
                acc += ws_o[((base + s) * G + h) * D + d] * sc;
            }
        }
        out[((size_t)b * Hq + g * G + h) * D + d] = __float2bfloat16_rn(acc / l);
    }
}

// Rolling-buffer write: cache[b, (pos[b]+t) mod W, h, :] = new[b, t, h, :],
// 16-byte copies, grid-stride over every (b, t, h, 16-byte chunk) of K and V.
// Write step of "Rolling Buffer KV Cache 동작 설명" (slot = p % W).
// With rope != 0 the keys are rotated (rotary embedding at their position)
// on the way into the cache; values are copied unchanged.
__global__ void swa_append_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                  uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                  const int32_t *__restrict__ pos, int B, int T, int W,
                                  int row_vec, int head_vec, int rope, const RopeTable rope_freq,
                                  uint4 *__restrict__ k_sink, uint4 *__restrict__ v_sink, int S) {
    // row_vec = Hkv*D*2/16 sixteen-byte vectors per (b, t) row
    const long long total = (long long)B * T * row_vec;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i % row_vec);
        const long long bt = i / row_vec;
        const int t = (int)(bt % T);
        const int b = (int)(bt / T);
        const int p0 = __ldg(pos + b);
        if (p0 < 0) {                               // invalid position: record, skip
            record_status(kStatusInvalid);
            continue;
        }
        const long long p = (long long)p0 + t;
        const int slot = (int)(p % W);
        const size_t dst = ((size_t)b * W + slot) * row_vec + c;
        uint4 kv = __ldg(k_new + i);
        if (rope) kv = rope_rotate8(kv, (c % head_vec) * 4, (double)p, rope_freq);
        const uint4 vv = __ldg(v_new + i);
        k_cache[dst] = kv;
        v_cache[dst] = vv;
        if (p < S) {                     // attention sinks: positions below S kept for good
            const size_t sdst = ((size_t)b * S + p) * row_vec + c;
            k_sink[sdst] = kv;
            v_sink[sdst] = vv;
        }
    }
}

}  // namespace swa

namespace swa {

// Rolling-buffer write for a packed variable-length batch: k_new/v_new
// [total, Hkv, D]; row r belongs to the sequence b with cu[b] <= r < cu[b+1]
// and has position start_pos[b] + (r - cu[b]).  A sequence longer than W
// writes only its last W rows (the earlier ones would be overwritten), so no
// two rows of one call share a slot.
__global__ void swa_append_varlen_kernel(const uint4 *__restrict__ k_new, const uint4 *__restrict__ v_new,
                                         uint4 *__restrict__ k_cache, uint4 *__restrict__ v_cache,
                                         const int32_t *__restrict__ start_pos,
                                         const int32_t *__restrict__ cu, int B, int total, int W,
                                         int row_vec) {
    const long long n = (long long)total * row_vec;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < n;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i % row_vec);
        const int r = (int)(i / row_vec);
        int lo = 0, hi = B - 1;                       // last b with cu[b] <= r
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (__ldg(cu + mid) <= r) lo = mid; else hi = mid - 1;
        }
        const int c0 = __ldg(cu + lo), c1 = __ldg(cu + lo + 1);
        const int s0 = __ldg(start_pos + lo);
        if (r < c0 || r >= c1 || s0 < 0) {            // malformed offsets or position
            record_status(kStatusInvalid);
            continue;
        }
        const int t = r - c0;
        if (t < (c1 - c0) - W) continue;              // overwritten later in this call
        const int slot = (int)(((long long)s0 + t) % W);
        const size_t dst = ((size_t)lo * W + slot) * row_vec + c;
        k_cache[dst] = __ldg(k_new + i);
        v_cache[dst] = __ldg(v_new + i);
    }
}

// In-place rotary embedding of x [B, T, H, D] (bf16), row (b, t) at position
// pos[b] + t; 16-byte words of four adjacent pairs, grid-stride.
__global__ void swa_rope_kernel(uint4 *__restrict__ x, const int32_t *__restrict__ pos, int B, int T,
                                int row_vec, int head_vec, const RopeTable rope_freq) {
    const long long total = (long long)B * T * row_vec;
    for (long long i = blockIdx.x * (long long)blockDim.x + threadIdx.x; i < total;
         i += (long long)gridDim.x * blockDim.x) {
        const int c = (int)(i % row_vec);
        const long long bt = i / row_vec;
        const int t = (int)(bt % T);
        const int b = (int)(bt / T);
        const int p0 = __ldg(pos + b);
        if (p0 < 0) {
            record_status(kStatusInvalid);
            continue;
        }
        x[i] = rope_rotate8(x[i], (c % head_vec) * 4, (double)p0 + t, rope_freq);
    }
}

}  // namespace swa
