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
// Memory-bound design: the kernel must stream the window's K and V rows at
// HBM speed, so the arithmetic per key row has to stay a few instructions.
//  * grid (split, kv head, sequence); a block of 4 warps streams one split of
//    up to SPLIT keys in blocks of 16 keys, warp w taking blocks w, w+4, ...
//  * each warp keeps its own 3-deep ring of 16-key K and V blocks in shared
//    memory, filled by 16-byte cp.async copies (rows XOR-swizzled in 16-byte
//    chunks so the matrix loads below are free of bank conflicts).
//  * the G query heads of the group are the rows of a 16-row tensor-core
//    tile (mma.sync m16n8k16, bf16 in, fp32 out; rows G..15 are zero):
//    S = Q K^T for 16 keys is 2 x D/16 MMAs with K fed by ldmatrix, and
//    O += P V is D/8 MMAs with V fed by ldmatrix.trans.  The S accumulator
//    of a thread is exactly its A fragment of P (head = row, keys = columns),
//    so P never leaves registers.  About 23 warp instructions per key row
//    of one KV head, the copies and the split's merge included.
//  * online softmax per head in base 2, scale applied to S in fp32; the
//    exponent offset of a head is raised (exact maximum over the block,
//    rescale of l and o) only when a score exceeds it by more than 2^8, so
//    most blocks take no maximum.
//  * warps and splits are merged by log-sum-exp: in shared memory inside a
//    block, and across splits either by swa_decode_combine_kernel or, when a
//    window takes exactly 4 splits (W = 4096 at large batch), inside a
//    cluster of those 4 blocks through distributed shared memory (one
//    launch fewer per step: 146.7 vs 149.7 us per call at B=64, W=4096).
//  * the one-token sequences of a packed chunk batch (decode steps in a
//    mixed pre-fill call) take a third mode: the token's own K/V come from
//    its packed row (the buffer is written after the attention), and the 4
//    splits of a window are the blocks of one cluster, merged the same way,
//    so no workspace is needed.
#pragma once

#include "device_common.cuh"

namespace swa {

// keys per block: at most kDecodeSplit (1024 measured 0.5-2.5% faster than
// 512 at B=64), fewer (down to kDecodeMinSplit) for batches too small to fill
// the GPU; the host picks it per launch from the sizes alone
constexpr int kDecodeSplit = 1024;
constexpr int kDecodeMinSplit = 256;
constexpr int kDecodeWarps = 4;
constexpr int kDecodeBlk = 16;         // keys per tensor-core block
constexpr int kDecodeStages = 3;       // per-warp ring depth, in 16-key blocks
// MODE 2 and 3 (no workspace): the window of one (sequence, kv head) is split
// over a cluster of this many blocks, merged through distributed shared memory
constexpr int kDecodeClusterSplits = 4;

template <int D, int G>
struct DecodeCfg {
    static constexpr int CH = D / 8;                       // 16-byte chunks per key row
    static constexpr int ROW_BYTES = D * 2;
    static constexpr int BLK_BYTES = kDecodeBlk * ROW_BYTES;   // K (or V) rows of one block
    static constexpr int STAGE_BYTES = 2 * BLK_BYTES;          // K then V
    static constexpr int WARP_RING = kDecodeStages * STAGE_BYTES;
    static constexpr int RING_BYTES = kDecodeWarps * WARP_RING;
    static constexpr int CPL = kDecodeBlk * CH / 32;           // 16-byte copies per lane, K or V
    static constexpr int KSTEPS = D / 16;                      // MMA k-steps of S = Q K^T
    static constexpr int NB = D / 8;                           // 8-column blocks of O
    // the warp merge reuses the rings once every copy has landed: per warp
    // and head {o[D], m, l}, then the block's merged {o[D], m, l} per head
    // (read by the cluster merge)
    static constexpr int MERGE_BYTES = (kDecodeWarps + 1) * G * (D + 2) * 4;
    static constexpr int SMEM_BYTES = RING_BYTES > MERGE_BYTES ? RING_BYTES : MERGE_BYTES;
    static_assert(D == 64 || D == 128, "head_dim");
    static_assert(G >= 1 && G <= 8, "group size 1 to 8 (the rows 0..7 of the MMA tile)");
    static_assert(CPL * 32 == kDecodeBlk * CH, "copies per lane");
};

__device__ __forceinline__ void cp_async16(uint32_t dst, const void *src) {
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16;" ::"r"(dst), "l"(src) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() {
    asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory");
}

// Four 8x8 bf16 matrices from shared memory (each lane gives one row address:
// lanes 8i..8i+7 the rows of matrix i); register i of a lane holds two
// adjacent elements of row lane/4 of matrix i (transposed: of column lane/4).
__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
    asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(addr)
                 : "memory");
}

// D(16x8, fp32) += A(16x16, bf16) B(16x8, bf16), warp-wide.  Only rows 0..7
// of A are given (a0: columns 2t, 2t+1 and a2: columns 2t+8, 2t+9 of row
// lane/4, t = lane%4); rows 8..15 are zero, so only d0 = D[lane/4][2t] and
// d1 = D[lane/4][2t+1] are accumulated and returned.
__device__ __forceinline__ void mma_rows8(float &d0, float &d1, uint32_t a0, uint32_t a2, uint32_t b0,
                                          uint32_t b1) {
    [[maybe_unused]] float u2, u3;     // rows 8..15 of D: zero, not kept
    asm("mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, "
        "{%8, %9}, {%10, %11, %12, %13};"
        : "=f"(d0), "=f"(d1), "=f"(u2), "=f"(u3)
        : "r"(a0), "r"(0u), "r"(a2), "r"(0u), "r"(b0), "r"(b1), "f"(d0), "f"(d1), "f"(0.f), "f"(0.f));
}

// Shared-memory offset of 16-byte chunk `ch` of row `r` in a block of rows of
// `row_bytes`: chunks XOR-swizzled by the row's low three bits, so the eight
// rows of one 8x8 matrix load fall in eight different bank groups.
__device__ __forceinline__ uint32_t swz_off(int r, int ch, int row_bytes) {
    return (uint32_t)(r * row_bytes + ((ch ^ (r & 7)) << 4));
}

// Partial result of one (sequence, kv head, split): per head m (base-2 max),
// l (sum of 2^(s-m)) and o[D] (sum of 2^(s-m) v).  Layout in the workspace:
// ml[((b*Hkv + g)*nsplit_max + s)*G + h] = {m, l};  o[...*D + d].
// MODE 0: the window only.  MODE 1 (attention sinks): keys past the window's
// come from the sink buffer.  MODE 2 (the length-1 sequences of a packed
// chunk batch, attend before the buffer write): sequence b is decoded only if
// it holds exactly one of the `total` packed rows (cu[b+1] - cu[b] == 1); its
// q and out rows are row cu[b]; the buffer gives positions p-Lc .. p-1
// (Lc = min(p, W-1), slot = position mod W) and the token's own key and value
// are row cu[b] of the packed k and v, passed as ksink / vsink.  The window
// is split over a cluster of kDecodeClusterSplits blocks (grid x), merged
// through distributed shared memory (each block merges a quarter of the
// outputs from all blocks' partials), so no workspace is needed.  MODE 3: the
// window as in MODE 0, split and merged as in MODE 2.
constexpr int kDecodeWindow = 0, kDecodeSinks = 1, kDecodePackedRows = 2, kDecodeWindowCluster = 3;

template <int D, int G, int MODE>
__global__ void __launch_bounds__(kDecodeWarps * 32, 2)
swa_decode_kernel(const __nv_bfloat16 *__restrict__ q, const __nv_bfloat16 *__restrict__ kc,
                  const __nv_bfloat16 *__restrict__ vc, const int32_t *__restrict__ pos,
                  __nv_bfloat16 *__restrict__ out, float2 *__restrict__ ws_ml,
                  float *__restrict__ ws_o, int Hkv, int W, int nsplit_max, float scale_log2,
                  int rope, const RopeTable rope_freq, const __nv_bfloat16 *__restrict__ ksink,
                  const __nv_bfloat16 *__restrict__ vsink, int S, const int32_t *__restrict__ cu,
                  int total, int split_len, int kv_rep) {
    constexpr bool SINKS = MODE == kDecodeSinks;
    // the splits of a window are the blocks of one cluster (grid x)
    constexpr bool CLUSTER = MODE == kDecodePackedRows || MODE == kDecodeWindowCluster;
    using Cfg = DecodeCfg<D, G>;
    constexpr int CH = Cfg::CH, RB = Cfg::ROW_BYTES;
    extern __shared__ __align__(128) uint8_t smem[];

    const int split = blockIdx.x, g = blockIdx.y, b = blockIdx.z;
    const int Hq = Hkv * G;
    int qrow = b;                                   // row of q and out
    if (MODE == kDecodePackedRows) {
        const int c0 = __ldg(cu + b), c1 = __ldg(cu + b + 1);
        // not a single-row sequence (malformed offsets are recorded by the
        // attention kernel that handles the other rows)
        if (c1 - c0 != 1 || c0 < 0 || c1 > total) return;
        qrow = c0;
    }
    const int p = __ldg(pos + b);
    if (p < 0) {                                    // invalid position: record, write nothing
        if (threadIdx.x == 0 && split == 0 && g == 0) record_status(kStatusInvalid);
        return;
    }
    const int Lw = (p >= W - 1) ? W : p + 1;           // keys in the window
    // MODE 2: keys 0 .. Lc-1 are buffer slots from that of position p - Lc
    // on, key Lc the packed row
    const int Lc = Lw - 1;
    const int slot0 = (MODE == kDecodePackedRows) ? (int)((p - Lc) % W) : 0;
    // sink positions that left the window: slots 0 .. ns-1 of the sink buffer,
    // numbered after the window's keys
    const int ns = (SINKS && S > 0 && p >= W) ? min(S, p - W + 1) : 0;
    const int L = Lw + ns;
    constexpr int kClusterKeys = kDecodeClusterSplits * kDecodeBlk;
    const int split_keys =
        CLUSTER ? (L + kClusterKeys - 1) / kClusterKeys * kDecodeBlk : split_len;
    // a cluster block past the window's keys still takes part in the merge
    if (!CLUSTER && split * split_keys >= L) return;
    const int begin = min(split * split_keys, L);
    const int end = min(L, begin + split_keys);
    const int nsplit = (L + split_keys - 1) / split_keys;

    const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
    const int hr = lane >> 2;                // fragment row: head of the group (valid if < G)
    const int t4 = lane & 3;                 // fragment column pair
    const bool head_ok = hr < G;
    const uint32_t ring = smem_addr(smem) + warp * Cfg::WARP_RING;

    // A fragments of Q (row hr; columns kk*16 + 2*t4 + {0, 1} and + 8), bf16;
    // with rope, each pair (2i, 2i+1) rotated at position p in fp32 first
    uint32_t qa[Cfg::KSTEPS][2];
    {
        const __nv_bfloat16 *qp = q + ((size_t)qrow * Hq + g * G + (head_ok ? hr : 0)) * D;
#pragma unroll
        for (int kk = 0; kk < Cfg::KSTEPS; ++kk)
#pragma unroll
            for (int hf = 0; hf < 2; ++hf) {
                const int d = kk * 16 + hf * 8 + 2 * t4;
                uint32_t w = head_ok ? __ldg(reinterpret_cast<const uint32_t *>(qp + d)) : 0u;
                if (rope && head_ok) {
                    float c, sn;
                    rope_cos_sin((double)p, rope_freq.f[d >> 1], c, sn);
                    const float x0 = __uint_as_float(w << 16), x1 = __uint_as_float(w & 0xFFFF0000u);
                    w = pack_bf16x2(x0 * c - x1 * sn, x0 * sn + x1 * c);
                }
                qa[kk][hf] = w;
            }
    }

    // K/V heads in memory: a group of more than 8 query heads (or one with no
    // divisor up to 8 above 1) is taken as kv_rep groups of G heads, all
    // reading K/V head g / kv_rep (Hkv counts those groups)
    const int Hkv_mem = Hkv / kv_rep, gk = g / kv_rep;
    const size_t row_stride = (size_t)Hkv_mem * D;  // elements between consecutive slots
    const __nv_bfloat16 *kbase = kc + ((size_t)b * W * Hkv_mem + gk) * D;
    const __nv_bfloat16 *vbase = vc + ((size_t)b * W * Hkv_mem + gk) * D;
    const __nv_bfloat16 *ksbase = ns ? ksink + ((size_t)b * S * Hkv_mem + gk) * D : kbase;
    const __nv_bfloat16 *vsbase = ns ? vsink + ((size_t)b * S * Hkv_mem + gk) * D : vbase;
    const __nv_bfloat16 *knew = (MODE == kDecodePackedRows) ? ksink + ((size_t)qrow * Hkv_mem + gk) * D : kbase;
    const __nv_bfloat16 *vnew = (MODE == kDecodePackedRows) ? vsink + ((size_t)qrow * Hkv_mem + gk) * D : vbase;

    const int nblk = (end - begin + kDecodeBlk - 1) / kDecodeBlk;
    const int my_blocks = (nblk > warp) ? (nblk - warp + kDecodeWarps - 1) / kDecodeWarps : 0;

    // stage layout: K rows [16][D] then V rows [16][D], swizzled chunks
    auto issue = [&](int i_local, int stage) {
        const int blk = warp + i_local * kDecodeWarps;
        const uint32_t st = ring + stage * Cfg::STAGE_BYTES;
#pragma unroll
        for (int c = 0; c < Cfg::CPL; ++c) {
            const int id = c * 32 + lane;
            const int r = id / CH, ch = id % CH;
            const int key = min(begin + blk * kDecodeBlk + r, end - 1);     // clamp: always in bounds
            const uint32_t off = swz_off(r, ch, RB);
            if (SINKS && key >= Lw) {
                if (!in_bounds(key - Lw, S)) continue;
                const size_t rowi = (size_t)(key - Lw) * row_stride + ch * 8;
                cp_async16(st + off, ksbase + rowi);
                cp_async16(st + Cfg::BLK_BYTES + off, vsbase + rowi);
            } else if (MODE == kDecodePackedRows) {
                if (key == Lc) {
                    cp_async16(st + off, knew + ch * 8);
                    cp_async16(st + Cfg::BLK_BYTES + off, vnew + ch * 8);
                } else {
                    const long long sl = (long long)slot0 + key;
                    const int slot = (int)(sl >= W ? sl - W : sl);
                    if (!in_bounds(slot, W)) continue;
                    const size_t rowi = (size_t)slot * row_stride + ch * 8;
                    cp_async16(st + off, kbase + rowi);
                    cp_async16(st + Cfg::BLK_BYTES + off, vbase + rowi);
                }
            } else {
                if (!in_bounds(key, W)) continue;
                const size_t rowi = (size_t)key * row_stride + ch * 8;
                cp_async16(st + off, kbase + rowi);
                cp_async16(st + Cfg::BLK_BYTES + off, vbase + rowi);
            }
        }
    };

    // per thread: head hr's running offset (equal in the 4 lanes of a quad),
    // this lane's share of its sum, and O[hr][nb*8 + 2*t4 + {0, 1}]
    float m_run = -INFINITY, l_run = 0.f;
    float o[Cfg::NB][2];
#pragma unroll
    for (int nb = 0; nb < Cfg::NB; ++nb) o[nb][0] = o[nb][1] = 0.f;

#pragma unroll
    for (int s = 0; s < kDecodeStages - 1; ++s) {
        if (s < my_blocks) issue(s, s);
        cp_async_commit();
    }

    for (int i = 0; i < my_blocks; ++i) {
        const int stage = i % kDecodeStages;
        cp_async_wait<kDecodeStages - 2>();
        __syncwarp();
        {
            const int nxt = i + kDecodeStages - 1;
            if (nxt < my_blocks) issue(nxt, nxt % kDecodeStages);
            cp_async_commit();
        }
        const uint32_t sk = ring + stage * Cfg::STAGE_BYTES, sv = sk + Cfg::BLK_BYTES;
        const int key0 = begin + (warp + i * kDecodeWarps) * kDecodeBlk;

        // S = Q K^T: keys 0-7 and 8-15 of the block; ldmatrix x4 covers 32 d
        float s[2][2] = {{0.f, 0.f}, {0.f, 0.f}};
#pragma unroll
        for (int nb = 0; nb < 2; ++nb)
#pragma unroll
            for (int c4 = 0; c4 < CH / 4; ++c4) {
                const int r = nb * 8 + (lane & 7), ch = c4 * 4 + (lane >> 3);
                uint32_t kb[4];
                ldsm_x4(sk + swz_off(r, ch, RB), kb);
                mma_rows8(s[nb][0], s[nb][1], qa[2 * c4][0], qa[2 * c4][1], kb[0], kb[1]);
                mma_rows8(s[nb][0], s[nb][1], qa[2 * c4 + 1][0], qa[2 * c4 + 1][1], kb[2], kb[3]);
            }
        // this lane's scores of head hr: keys key0 + 2*t4 + {0, 1, 8, 9}
        float sc[4] = {s[0][0], s[0][1], s[1][0], s[1][1]};
        float mx = -INFINITY;
#pragma unroll
        for (int e = 0; e < 4; ++e) {
            const int key = key0 + 2 * t4 + (e & 1) + (e >> 1) * 8;
            sc[e] = (key < end) ? sc[e] * scale_log2 : -INFINITY;
            mx = fmaxf(mx, sc[e]);
        }
        // a score more than 2^8 above its head's offset (always on the first
        // block) makes the warp take the exact maximum over the block (the
        // quad of lanes holding the head) and rescale; otherwise the offset
        // stays (p = 2^(s - offset) <= 2^8, exact after normalisation)
        if (__any_sync(0xffffffffu, head_ok && mx > m_run + 8.0f)) {
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 1));
            mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, 2));
            if (mx > m_run) {                    // uniform across the quad
                const float alpha = ex2_approx(m_run - mx);      // 0 when m_run = -inf
                l_run *= alpha;
#pragma unroll
                for (int nb = 0; nb < Cfg::NB; ++nb) {
                    o[nb][0] *= alpha;
                    o[nb][1] *= alpha;
                }
                m_run = mx;
            }
        }
        float pw[4];
#pragma unroll
        for (int e = 0; e < 4; ++e) pw[e] = head_ok ? ex2_approx(sc[e] - m_run) : 0.f;
        // P as the A fragment of O += P V: columns (keys) 2*t4 + {0, 1} and + 8;
        // l sums P as rounded to bf16, the weights V is actually multiplied by
        const uint32_t pa0 = pack_bf16x2(pw[0], pw[1]), pa2 = pack_bf16x2(pw[2], pw[3]);
        {
            const float2 l2 = add_bf16x2(add_bf16x2(make_float2(0.f, 0.f), pa0), pa2);
            l_run += l2.x + l2.y;
        }
#pragma unroll
        for (int c2 = 0; c2 < CH / 2; ++c2) {
            const int mi = lane >> 3;
            const int r = (mi & 1) * 8 + (lane & 7), ch = c2 * 2 + (mi >> 1);
            uint32_t vb[4];
            ldsm_x4_trans(sv + swz_off(r, ch, RB), vb);
            mma_rows8(o[2 * c2][0], o[2 * c2][1], pa0, pa2, vb[0], vb[1]);
            mma_rows8(o[2 * c2 + 1][0], o[2 * c2 + 1][1], pa0, pa2, vb[2], vb[3]);
        }
        __syncwarp();
    }
    cp_async_wait<0>();

    // l over the quad (each lane summed its own keys)
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 1);
    l_run += __shfl_xor_sync(0xffffffffu, l_run, 2);

    // merge the warps of the block in shared memory (over the rings)
    __syncthreads();
    float *mg = reinterpret_cast<float *>(smem);    // [warp][G][D+2]
    if (head_ok) {
        float *dst = mg + (warp * G + hr) * (D + 2);
#pragma unroll
        for (int nb = 0; nb < Cfg::NB; ++nb) {
            dst[nb * 8 + 2 * t4] = o[nb][0];
            dst[nb * 8 + 2 * t4 + 1] = o[nb][1];
        }
        if (t4 == 0) {
            dst[D] = m_run;
            dst[D + 1] = l_run;
        }
    }
    __syncthreads();
    float *part = mg + kDecodeWarps * G * (D + 2);  // [G][D+2]: the block's merge (cluster modes)
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
        if (CLUSTER) {
            part[h * (D + 2) + d] = acc;
            if (d == 0) {
                part[h * (D + 2) + D] = m;
                part[h * (D + 2) + D + 1] = l;
            }
        } else if (nsplit == 1) {
            const size_t oi = ((size_t)qrow * Hq + g * G + h) * D + d;
            if (in_bounds((long long)oi, (long long)gridDim.z * Hq * D)) out[oi] = __float2bfloat16_rn(acc / l);
        } else {
            const size_t slot = ((size_t)(b * Hkv + g) * nsplit_max + split) * G + h;
            if (!in_bounds(split, nsplit_max)) continue;
            ws_o[slot * D + d] = acc;
            if (d == 0) ws_ml[slot] = make_float2(m, l);
        }
    }
    if constexpr (CLUSTER) {
        // every block of the cluster reaches both barriers: the only returns
        // above depend on (b) alone, which the cluster shares
        cluster_sync_all();
        {   // each block of the cluster merges and writes a quarter of the outputs
            static_assert((G * D) % kDecodeClusterSplits == 0, "outputs per block");
            constexpr int kPer = G * D / kDecodeClusterSplits;
            const int i0 = (int)cluster_rank() * kPer;
            for (int idx = i0 + threadIdx.x; idx < i0 + kPer; idx += blockDim.x) {
                const int h = idx / D, d = idx % D;
                const uint32_t row = smem_addr(part + h * (D + 2));
                float mr[kDecodeClusterSplits], lr[kDecodeClusterSplits], ar[kDecodeClusterSplits];
                float m = -INFINITY;
#pragma unroll
                for (int r = 0; r < kDecodeClusterSplits; ++r) {
                    mr[r] = ld_peer_f32(row + D * 4, r);
                    lr[r] = ld_peer_f32(row + (D + 1) * 4, r);
                    ar[r] = ld_peer_f32(row + d * 4, r);
                    m = fmaxf(m, mr[r]);
                }
                float l = 0.f, acc = 0.f;
#pragma unroll
                for (int r = 0; r < kDecodeClusterSplits; ++r) {
                    const float sc = (mr[r] == -INFINITY) ? 0.f : ex2_approx(mr[r] - m);
                    l += lr[r] * sc;
                    acc += ar[r] * sc;
                }
                const size_t oi = ((size_t)qrow * Hq + g * G + h) * D + d;
                if (in_bounds((long long)oi, (long long)total * Hq * D)) out[oi] = __float2bfloat16_rn(acc / l);
            }
        }
        cluster_sync_all();                          // peers' shared memory stays until read
    }
}

// Log-sum-exp merge of the splits of each (sequence, kv head) into bf16 out.
template <int D, int G>
__global__ void __launch_bounds__(1024)
swa_decode_combine_kernel(const int32_t *__restrict__ pos, const float2 *__restrict__ ws_ml,
                          const float *__restrict__ ws_o, __nv_bfloat16 *__restrict__ out,
                          int Hkv, int W, int nsplit_max, int S, int split_len) {
    const int g = blockIdx.x, b = blockIdx.y;
    const int Hq = Hkv * G;
    const int p = __ldg(pos + b);
    if (p < 0) return;
    const int ns = (S > 0 && p >= W) ? min(S, p - W + 1) : 0;
    const int L = ((p >= W - 1) ? W : p + 1) + ns;
    const int nsplit = (L + split_len - 1) / split_len;
    if (nsplit <= 1 || !in_bounds(nsplit - 1, nsplit_max)) return;
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
        if (!in_bounds(slot, W) || !in_bounds(b, B)) continue;
        const size_t dst = ((size_t)b * W + slot) * row_vec + c;
        uint4 kv = __ldg(k_new + i);
        if (rope) kv = rope_rotate8(kv, (c % head_vec) * 4, (double)p, rope_freq);
        const uint4 vv = __ldg(v_new + i);
        k_cache[dst] = kv;
        v_cache[dst] = vv;
        if (p < S && in_bounds(p, S)) {  // attention sinks: positions below S kept for good
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
        if (r < c0 || r >= c1 || c0 < 0 || c1 > total || s0 < 0) {   // malformed offsets or position
            record_status(kStatusInvalid);
            continue;
        }
        const int t = r - c0;
        if (t < (c1 - c0) - W) continue;              // overwritten later in this call
        const int slot = (int)(((long long)s0 + t) % W);
        if (!in_bounds(slot, W) || !in_bounds(lo, B)) continue;
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
