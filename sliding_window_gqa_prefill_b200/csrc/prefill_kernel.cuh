// prefill_kernel.cuh -- banded sliding-window GQA attention on tcgen05 / TMEM.
//
// Computes, for every query row i of a prompt (one-shot) or of a chunk that
// continues a prompt through a rolling-buffer cache (chunked pre-fill):
//     out[i] = sum_j softmax_j(scale * q_i . k_j) v_j
// over the keys j of the causal window i-W < j <= i.  Sources: the SWA mask
// of section "핵심 구성요소" of the "Mistral 7B -- Sliding Window Attention"
// summary, the SWA equation of section 2 of "Mistral 7B: Engineering Extreme
// Efficiency in LLMs", and for the chunked form "Pre-fill + Chunking" of the
// same summary and section 4.1 / Figure 3 of the manon006 review.
//
// Design (one persistent CTA per SM):
//  * Work unit = (sequence b, KV head g, pair of query heads of group g,
//    block of 128 query rows).  Both query heads of the pair share every K/V
//    tile, so one TMA load of a K/V tile feeds two 128x128 MMAs.
//  * Only key tiles that intersect the band [q0-W+1, q0+127] are visited, so
//    work is O(N*W).  Tiles strictly inside the band skip all masking.
//  * Warp roles (12 warps): warp 0 issues TMA loads (Q once per unit, K and V
//    through 2-deep rings); warp 1 issues tcgen05.mma from one thread;
//    warp 2 owns the tensor-memory allocation; warps 4-7 and 8-11 are the
//    softmax warpgroups of query head 0 and 1 of the pair.
//  * Tensor memory (512 columns): S0 | S1 | O0 | O1, 128 columns each.  The
//    softmax writes P (bf16, two per column) over the first half of its S
//    columns and the PV MMA reads A = P straight from tensor memory.
//  * Online softmax in fp32, base-2 exponent with the scale folded in.  The
//    running maximum used as exponent offset is raised only when the tile
//    maximum exceeds it by more than 8 (2^8 bound on P), so the O rescale
//    round trip through tensor memory is rare.  P is rounded to bf16 for the
//    PV MMA; l adds, per tile, the rounding of the tile's largest P (as its
//    element computed it), so a row dominated by one key keeps O / l exact.
//  * Chunked pre-fill: the key tiles of a unit are the cache slot tiles that
//    hold positions inside the window of the block (one or two runs of slots
//    modulo W), then the chunk's own tiles.  Slot s holds position
//    s0 - age(s), age(s) = (q - s) mod W in 1..W, q = s0 mod W, so masks are
//    computed per element only on tiles that need them.
//  * Every wait is bounded (SWA_ERR_TIMEOUT in the status word, then the
//    block drains its own in-flight copies / MMAs, frees tensor memory and
//    returns).
#pragma once

#include "prefill_plan.cuh"

namespace swa {


template <int D>
struct PrefillCfg {
    static constexpr int BM = 128;                 // query rows per tile
    static constexpr int BN = 128;                 // keys per tile
    static constexpr int NREG = D / 64;            // 64-column (128-byte) swizzle regions
    static constexpr int REGION_BYTES = 128 * 128; // 128 rows x 128 bytes
    static constexpr int TILE_BYTES = NREG * REGION_BYTES;
    // K ring depth: 2 measured 1-5% faster than 3; the 32 KB it frees leave
    // more of the SM's unified L1 / shared storage to L1, through which the
    // softmax warps' register spills go
    static constexpr int KST = 2;
    static constexpr int VST = 2;                  // V ring depth
    static constexpr int OFF_Q = 0;                // two Q tiles
    static constexpr int OFF_K = 2 * TILE_BYTES;
    static constexpr int OFF_V = OFF_K + KST * TILE_BYTES;
    static constexpr int OFF_BAR = OFF_V + VST * TILE_BYTES;
    // barriers: q_full, q_empty, k_full[KST], k_empty[KST], v_full[VST],
    // v_empty[VST], s_full[2], p_full[2], o_full[2], drain, p_half[2], q_rot[2],
    // q1_full (q_full covers Q tile 0, q1_full tile 1)
    static constexpr int NBAR = 2 + 2 * KST + 2 * VST + 2 + 2 + 2 + 1 + 2 + 2 + 1;
    static constexpr int OFF_MISC = OFF_BAR + NBAR * 8;    // tmem base, abort flag, unit count
    static constexpr int OFF_PRE = OFF_MISC + 16;           // varlen: query-block prefix sums
    static constexpr int SMEM_BYTES = OFF_PRE + (kMaxVarlenSeqs + 1) * 4;
    static constexpr int SMEM_ALLOC = SMEM_BYTES + 1024;   // slack for 1024-byte alignment
    static constexpr int THREADS = 384;
    // which of the 16 column pairs of each 32-column chunk take the polynomial
    // exponential instead of ex2.approx (bits 3, 7, 11, 15: one pair in four)
    static constexpr uint32_t kEmuPairs = 0x8888u;
    static_assert(kEmuPairs == (kEmuPairs & 0xFu) * 0x1111u, "the pattern repeats every four pairs");
    // PV in two halves of 64 keys: the first half starts while the softmax
    // still computes the second half of P
    static constexpr bool kSplitPV = true;
    // the MMA thread polls its barriers instead of suspending on them
    static constexpr bool kMmaSpin = false;
    static constexpr uint32_t TMEM_COLS = 512;
    static constexpr uint32_t IDESC_QK = make_idesc_bf16(128, 128, 0);
    static constexpr uint32_t IDESC_PV = make_idesc_bf16(128, D, 1);
    static_assert(D == 64 || D == 128, "head_dim 64 or 128");
    static_assert(SMEM_ALLOC <= 232448, "dynamic shared memory of one block (227 KB)");
};

// Which query rows and key tiles one work unit covers.
// Rotary embedding of row `row` of a K-major, 128-byte-swizzled bf16 tile in
// shared memory (the layout TMA writes): 16-byte chunk c of the row in a
// 64-column region sits at chunk c ^ (row mod 8).
template <int D>
__device__ __forceinline__ void rope_row_swizzled(uint8_t *tile, int row, double p, const RopeTable &tab) {
#pragma unroll
    for (int reg = 0; reg < D / 64; ++reg) {
#pragma unroll
        for (int c = 0; c < 8; ++c) {
            uint4 *ptr = reinterpret_cast<uint4 *>(tile + reg * 128 * 128 + row * 128 + ((c ^ (row & 7)) * 16));
            *ptr = rope_rotate8(*ptr, reg * 32 + c * 4, p, tab);
        }
    }
}

template <int D>
__global__ void __launch_bounds__(384, 1)
swa_prefill_kernel(const __grid_constant__ CUtensorMap tm_q,
                   const __grid_constant__ CUtensorMap tm_k,
                   const __grid_constant__ CUtensorMap tm_v,
                   const __grid_constant__ CUtensorMap tm_kc,
                   const __grid_constant__ CUtensorMap tm_vc,
                   const __grid_constant__ CUtensorMap tm_ks,
                   const __grid_constant__ CUtensorMap tm_vs,
                   const PrefillParams p) {
    using Cfg = PrefillCfg<D>;
    constexpr int BN = Cfg::BN, KST = Cfg::KST, VST = Cfg::VST;
    constexpr int NREG = Cfg::NREG, RB = Cfg::REGION_BYTES, TB = Cfg::TILE_BYTES;

    extern __shared__ uint8_t smem_raw[];
    uint8_t *smem = reinterpret_cast<uint8_t *>(
        (reinterpret_cast<uintptr_t>(smem_raw) + 1023) & ~static_cast<uintptr_t>(1023));
    const uint32_t sbase = smem_addr(smem);
    const uint32_t sQ = sbase + Cfg::OFF_Q;
    const uint32_t sK = sbase + Cfg::OFF_K;
    const uint32_t sV = sbase + Cfg::OFF_V;
    const uint32_t bar0 = sbase + Cfg::OFF_BAR;
    const uint32_t bar_q_full = bar0;
    const uint32_t bar_q_empty = bar0 + 8;
    const uint32_t bar_k_full = bar0 + 16;                   // + 8*slot
    const uint32_t bar_k_empty = bar_k_full + 8 * KST;
    const uint32_t bar_v_full = bar_k_empty + 8 * KST;
    const uint32_t bar_v_empty = bar_v_full + 8 * VST;
    const uint32_t bar_s_full = bar_v_empty + 8 * VST;       // + 8*t
    const uint32_t bar_p_full = bar_s_full + 16;
    const uint32_t bar_o_full = bar_p_full + 16;
    const uint32_t bar_drain = bar_o_full + 16;
    const uint32_t bar_p_half = bar_drain + 8;                // + 8*t
    const uint32_t bar_q_rot = bar_p_half + 16;               // + 8*t (RoPE on Q done)
    // Q tile 1 lands on a barrier of its own: it is loaded only in units whose
    // second head (or query block) exists, and each consumer counts the
    // phases of the barriers it waits on over exactly those units
    const uint32_t bar_q1_full = bar_q_rot + 16;
    uint32_t *tmem_slot = reinterpret_cast<uint32_t *>(smem + Cfg::OFF_MISC);
    volatile int *abort_flag = reinterpret_cast<volatile int *>(smem + Cfg::OFF_MISC + 4);
    int *unit_count = reinterpret_cast<int *>(smem + Cfg::OFF_MISC + 8);
    int *pre = reinterpret_cast<int *>(smem + Cfg::OFF_PRE);

    const int warp = threadIdx.x >> 5;
    const int lane = threadIdx.x & 31;
    const unsigned long long limit = g_wait_limit_ns;

    if (threadIdx.x == 0) {
        mbar_init(bar_q_full, 1);
        mbar_init(bar_q_empty, 1);
        for (int s = 0; s < KST; ++s) {
            mbar_init(bar_k_full + 8 * s, 1);
            mbar_init(bar_k_empty + 8 * s, 1);
        }
        for (int s = 0; s < VST; ++s) {
            mbar_init(bar_v_full + 8 * s, 1);
            mbar_init(bar_v_empty + 8 * s, 1);
        }
        for (int t = 0; t < 2; ++t) {
            mbar_init(bar_s_full + 8 * t, 1);
            mbar_init(bar_p_full + 8 * t, 4);
            mbar_init(bar_o_full + 8 * t, 1);
        }
        mbar_init(bar_drain, 1);
        mbar_init(bar_p_half, 4);
        mbar_init(bar_p_half + 8, 4);
        mbar_init(bar_q_rot, 4);
        mbar_init(bar_q_rot + 8, 4);
        mbar_init(bar_q1_full, 1);
        *abort_flag = 0;
        mbar_init_fence();
        if (p.cu_seqlens) {
            // query blocks per sequence, prefix-summed (malformed sequences
            // count as empty and are recorded)
            if (varlen_prefix(p, pre)) record_status(kStatusInvalid);
            *unit_count = pre[p.B] * p.Hkv * p.npairs;
        } else {
            *unit_count = p.num_units;
        }
    }
    if (warp == 0 && lane == 0) {
        prefetch_tensormap(&tm_q);
        prefetch_tensormap(&tm_k);
        prefetch_tensormap(&tm_v);
        if (p.chunk_mode) {
            prefetch_tensormap(&tm_kc);
            prefetch_tensormap(&tm_vc);
        }
        if (p.sink_buf > 0) {
            prefetch_tensormap(&tm_ks);
            prefetch_tensormap(&tm_vs);
        }
    }
    // a block with no unit (a packed launch whose sequences all went to the
    // decode kernel, or fewer units than blocks) leaves before it allocates
    // tensor memory; the test is uniform across the block
    __syncthreads();
    const int num_units = *unit_count;
    if ((int)blockIdx.x >= num_units) return;
    if (warp == 2) {
        tmem_alloc(smem_addr(tmem_slot), Cfg::TMEM_COLS);
        tmem_relinquish();
    }
    tc_fence_before();
    __syncthreads();
    tc_fence_after();
    const uint32_t tmem = *tmem_slot;

    if (warp == 0) {
        // ------------------------------------------------------------ TMA producer
        if (lane == 0) {
            uint32_t kc = 0, vc = 0, uc = 0;          // tiles / units issued
            uint32_t k_cnt[KST] = {}, v_cnt[VST] = {};
            uint32_t q_cnt = 0, q1_cnt = 0;
            bool ok = true;
            for (int k = 0, u; (u = unit_of(k, blockIdx.x, gridDim.x)) < num_units && ok; ++k, ++uc) {
                const UnitPlan P = plan_unit(p, u, pre);
                const int nact = 1 + P.act1;
                if (!mbar_wait_bounded(bar_q_empty, (uc & 1) ^ 1, abort_flag, limit)) { ok = false; break; }
                mbar_arrive_expect_tx(bar_q_full, TB);
                if (P.act1) mbar_arrive_expect_tx(bar_q1_full, TB);
                const int qrow = P.row0 + P.q0;
                const int qb = checked_coord(P.tb, p.cu_seqlens ? 1 : p.B);
                for (int t = 0; t < nact; ++t) {
                    // the pair's second head, or with qpair its second query block
                    const int h = checked_coord(p.qpair ? P.h0 : P.h0 + t, p.Hq);
                    const int qr = checked_coord(qrow + (p.qpair ? t * 128 : 0), p.Nq);
                    const uint32_t qbar = t ? bar_q1_full : bar_q_full;
                    for (int r = 0; r < NREG; ++r)
                        tma_load_4d(sQ + t * TB + r * RB, &tm_q, qbar, r * 64, h, qr, qb);
                }
                ++q_cnt;
                q1_cnt += P.act1;
                for (int j = 0; j < P.n; ++j) {
                    const TileRef T = tile_ref(p, P, j);
                    const CUtensorMap *mk = T.cache == 2 ? &tm_ks : T.cache ? &tm_kc : &tm_k;
                    const CUtensorMap *mv = T.cache == 2 ? &tm_vs : T.cache ? &tm_vc : &tm_v;
                    const uint32_t ks = kc % KST, kph = (kc / KST) & 1;
                    if (!mbar_wait_bounded(bar_k_empty + 8 * ks, kph ^ 1, abort_flag, limit)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar_k_full + 8 * ks, TB);
                    // cache tiles: [B, W] slots of sequence b; main tiles: rows of this sequence
                    int krow = T.cache ? T.row0 : P.row0 + T.row0, kb = T.cache ? P.b : P.tb;
                    if (kBoundsCheck) {
                        krow = checked_coord(krow, T.cache == 2 ? p.sink_buf : T.cache ? p.W : p.Nk);
                        kb = checked_coord(kb, (T.cache || !p.cu_seqlens) ? p.B : 1);
                        (void)checked_coord(P.g, p.Hkv);
                    }
                    for (int r = 0; r < NREG; ++r)
                        tma_load_4d(sK + ks * TB + r * RB, mk, bar_k_full + 8 * ks, r * 64, P.g, krow, kb);
                    ++k_cnt[ks];
                    ++kc;
                    const uint32_t vs = vc % VST, vph = (vc / VST) & 1;
                    if (!mbar_wait_bounded(bar_v_empty + 8 * vs, vph ^ 1, abort_flag, limit)) { ok = false; break; }
                    mbar_arrive_expect_tx(bar_v_full + 8 * vs, TB);
                    for (int r = 0; r < NREG; ++r)
                        tma_load_4d(sV + vs * TB + r * RB, mv, bar_v_full + 8 * vs, r * 64, P.g, krow, kb);
                    ++v_cnt[vs];
                    ++vc;
                }
            }
            if (!ok) {
                // let every copy this thread started land before the block exits
                if (q_cnt) mbar_drain_bounded(bar_q_full, (q_cnt - 1) & 1, kDrainLimitNs);
                if (q1_cnt) mbar_drain_bounded(bar_q1_full, (q1_cnt - 1) & 1, kDrainLimitNs);
                for (int s = 0; s < KST; ++s)
                    if (k_cnt[s]) mbar_drain_bounded(bar_k_full + 8 * s, (k_cnt[s] - 1) & 1, kDrainLimitNs);
                for (int s = 0; s < VST; ++s)
                    if (v_cnt[s]) mbar_drain_bounded(bar_v_full + 8 * s, (v_cnt[s] - 1) & 1, kDrainLimitNs);
            }
        }
        __syncwarp();
    } else if (warp == 1) {
        // ------------------------------------------------------------ MMA issuer
        if (lane == 0) {
            // K-major Q/K operands: leading offset 16 B (unused under the 128-byte
            // swizzle), 8-row groups 1024 B apart.  MN-major V: the two 64-wide
            // halves of D are one region (RB) apart, 8-key groups 1024 B apart.
            constexpr uint32_t kDescHiK = smem_desc_hi(1024), kDescHiV = smem_desc_hi(1024);
            const uint32_t qdesc_lo = smem_desc_lo(sQ, 16);
            const uint32_t kdesc_lo = smem_desc_lo(sK, 16);
            const uint32_t vdesc_lo = smem_desc_lo(sV, RB);
            uint32_t kc = 0, vc = 0, uc = 0;
            uint32_t pc[2] = {0, 0};
            uint32_t qr1 = 0;                      // units with a second query tile
            bool ok = true;
            for (int k = 0, u; (u = unit_of(k, blockIdx.x, gridDim.x)) < num_units && ok; ++k, ++uc) {
                const UnitPlan P = plan_unit(p, u, pre);
                const int n = P.n;
                if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_q_full, uc & 1, abort_flag, limit)) { ok = false; break; }
                // Q tile 1 is absent in some units (odd group size, ragged last
                // query-block pair): its barriers complete once per unit where it
                // is present
                if (P.act1 && !mbar_wait_bounded<Cfg::kMmaSpin>(bar_q1_full, qr1 & 1, abort_flag, limit)) {
                    ok = false;
                    break;
                }
                if (p.rope) {       // the softmax warpgroups rotate Q in place first
                    if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_q_rot, uc & 1, abort_flag, limit)) { ok = false; break; }
                    if (P.act1 && !mbar_wait_bounded<Cfg::kMmaSpin>(bar_q_rot + 8, qr1 & 1, abort_flag, limit)) {
                        ok = false;
                        break;
                    }
                }
                qr1 += P.act1;
                // S_t = Q_t K^T for key tile j, into tensor-memory columns [t*128, t*128+128).
                // Descriptors step along K by adding to their low word only.
                auto issue_s = [&](int t, uint32_t kslot) {
                    const uint32_t alo = qdesc_lo + t * (TB >> 4), blo = kdesc_lo + kslot * (TB >> 4);
                    const uint32_t d = tmem + t * 128;
#pragma unroll
                    for (int kk = 0; kk < D / 16; ++kk) {
                        const uint32_t off = ((kk >> 2) * RB + (kk & 3) * 32) >> 4;
                        mma_ss(d, smem_desc64(alo + off, kDescHiK), smem_desc64(blo + off, kDescHiK),
                               Cfg::IDESC_QK, kk > 0);
                    }
                };
                // O_t (+)= P_t V for keys [64*half, 64*half+64), P_t read from tensor
                // memory over S_t's columns
                auto issue_pv = [&](int t, uint32_t vslot, bool acc, int half) {
                    const uint32_t blo = vdesc_lo + vslot * (TB >> 4);
                    const uint32_t d = tmem + 256 + t * 128, a = tmem + t * 128;
#pragma unroll
                    for (int k4 = 0; k4 < BN / 32; ++k4) {
                        const int kk = half * (BN / 32) + k4;
                        mma_ts(d, a + kk * 8, smem_desc64(blo + ((kk * 16 * 128) >> 4), kDescHiV),
                               Cfg::IDESC_PV, (acc || kk > 0) ? 1u : 0u);
                    }
                };
                {   // prologue: S for tile 0
                    const uint32_t ks = kc % KST, kph = (kc / KST) & 1;
                    if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_k_full + 8 * ks, kph, abort_flag, limit)) { ok = false; break; }
                    tc_fence_after();
                    issue_s(0, ks);
                    mma_commit(bar_s_full);
                    if (P.act1) {
                        issue_s(1, ks);
                        mma_commit(bar_s_full + 8);
                    }
                    mma_commit(bar_k_empty + 8 * ks);
                    if (n == 1) mma_commit(bar_q_empty);
                    ++kc;
                }
                for (int j = 0; j < n && ok; ++j) {
                    const uint32_t vs = vc % VST, vph = (vc / VST) & 1;
                    if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_v_full + 8 * vs, vph, abort_flag, limit)) { ok = false; break; }
                    if (Cfg::kSplitPV) {
                        if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_p_half, pc[0] & 1, abort_flag, limit)) { ok = false; break; }
                        tc_fence_after();
                        issue_pv(0, vs, j > 0, 0);
                    }
                    if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_p_full, pc[0] & 1, abort_flag, limit)) { ok = false; break; }
                    ++pc[0];
                    tc_fence_after();
                    if (!Cfg::kSplitPV) issue_pv(0, vs, j > 0, 0);
                    issue_pv(0, vs, j > 0, 1);
                    if (j == n - 1) mma_commit(bar_o_full);
                    uint32_t ks = 0;
                    const bool more = (j + 1 < n);
                    if (more) {
                        ks = kc % KST;
                        const uint32_t kph = (kc / KST) & 1;
                        if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_k_full + 8 * ks, kph, abort_flag, limit)) { ok = false; break; }
                        tc_fence_after();
                        issue_s(0, ks);
                        mma_commit(bar_s_full);
                    }
                    if (P.act1) {
                        if (Cfg::kSplitPV) {
                            if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_p_half + 8, pc[1] & 1, abort_flag, limit)) { ok = false; break; }
                            tc_fence_after();
                            issue_pv(1, vs, j > 0, 0);
                        }
                        if (!mbar_wait_bounded<Cfg::kMmaSpin>(bar_p_full + 8, pc[1] & 1, abort_flag, limit)) { ok = false; break; }
                        ++pc[1];
                        tc_fence_after();
                        if (!Cfg::kSplitPV) issue_pv(1, vs, j > 0, 0);
                        issue_pv(1, vs, j > 0, 1);
                        if (j == n - 1) mma_commit(bar_o_full + 8);
                    }
                    mma_commit(bar_v_empty + 8 * vs);
                    ++vc;
                    if (more) {
                        if (P.act1) {
                            issue_s(1, ks);
                            mma_commit(bar_s_full + 8);
                        }
                        mma_commit(bar_k_empty + 8 * ks);
                        if (j + 1 == n - 1) mma_commit(bar_q_empty);
                        ++kc;
                    }
                }
            }
            if (!ok) {
                mma_commit(bar_drain);
                mbar_drain_bounded(bar_drain, 0, kDrainLimitNs);
            }
        }
        __syncwarp();
    } else if (warp >= 4) {
        // ------------------------------------------------------------ softmax warpgroups
        const int t = (warp - 4) >> 2;            // query head of the pair
        const int quarter = warp & 3;             // TMEM lane quarter of this warp
        const int row = quarter * 32 + lane;      // query row within the tile
        const uint32_t lane_off = (uint32_t)(quarter * 32) << 16;
        const uint32_t tS = tmem + lane_off + t * 128;
        const uint32_t tO = tmem + lane_off + 256 + t * 128;
        const float sl2 = p.scale_log2;
        uint32_t sc = 0, oc = 0, qc = 0;
        bool ok = true;
        for (int k = 0, u; (u = unit_of(k, blockIdx.x, gridDim.x)) < num_units && ok; ++k) {
            const UnitPlan P = plan_unit(p, u, pre);
            if (t == 1 && !P.act1) continue;
            const int i_rel = P.q0 + (p.qpair ? t * 128 : 0) + row;   // query row in the q tensor
            // phase of this warpgroup's Q barrier: it counts only the units where
            // the tile is loaded, like the producer's arming of it
            const uint32_t qph = qc++ & 1;
            if (p.rope) {
                // rotary embedding of this thread's Q row, in shared memory, at
                // position s0 + i_rel; then make it visible to the tensor core
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(t ? bar_q1_full : bar_q_full, qph, abort_flag, limit))) {
                    ok = false;
                    break;
                }
                rope_row_swizzled<D>(smem + Cfg::OFF_Q + t * TB, row, (double)P.s0 + i_rel, p.rope_freq);
                fence_proxy_async_smem();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_q_rot + 8 * t);
            }
            float m_use = -INFINITY, l = 0.f;
            for (int j = 0; j < P.n; ++j) {
                const TileRef T = tile_ref(p, P, j);
                // warp-uniform outcome, so the collective tensor-memory ops stay converged
                if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_s_full + 8 * t, sc & 1, abort_flag, limit))) {
                    ok = false;
                    break;
                }
                ++sc;
                tc_fence_after();
                float s[BN];
                {
                    uint32_t r[BN / 32][32];
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) tmem_ld32(tS + c * 32, r[c]);
                    tmem_wait_ld();
#pragma unroll
                    for (int c = 0; c < BN / 32; ++c) {
                        reg_fence32(r[c]);
#pragma unroll
                        for (int e = 0; e < 32; ++e) s[c * 32 + e] = __uint_as_float(r[c][e]);
                    }
                }
                if (T.masked) {
                    if (T.cache == 2) {
                        // sink slot j holds position j: visible iff outside the window
                        const long long lim = (long long)P.s0 + i_rel - p.W;   // 64-bit: rows past the chunk too
#pragma unroll
                        for (int c = 0; c < BN; ++c) {
                            const int slot = T.row0 + c;
                            if (slot >= p.sink_buf || slot > lim) s[c] = -INFINITY;
                        }
                    } else if (T.cache) {
                        // slot k0+c holds position s0 - age; valid iff age < W - t_rel, age <= s0
                        const int lim = min(p.W - i_rel - 1, P.s0);
#pragma unroll
                        for (int c = 0; c < BN; ++c) {
                            const int slot = T.row0 + c;
                            const int age = (slot < P.qs) ? (P.qs - slot) : (P.qs - slot + p.W);
                            if (slot >= p.W || age > lim) s[c] = -INFINITY;
                        }
                    } else {
#pragma unroll
                        for (int c = 0; c < BN; ++c) {
                            const int key = T.row0 + c;
                            if (key > i_rel || (key <= i_rel - p.W && key >= p.sinks)) s[c] = -INFINITY;
                        }
                    }
                }
                float mx[8];
#pragma unroll
                for (int e = 0; e < 8; ++e) mx[e] = s[e];
#pragma unroll
                for (int c = 8; c < BN; c += 8)
#pragma unroll
                    for (int e = 0; e < 8; ++e) mx[e] = fmaxf(mx[e], s[c + e]);
                // chain e of the tree holds the columns c with c mod 8 == e, i.e. column
                // pair (e / 2) of every group of four pairs; kEmuPairs repeats every
                // four pairs, so each chain holds columns of one exponential only:
                // the maximum over the polynomial columns and over the others
                float mpoly = -INFINITY, mmufu = -INFINITY;
#pragma unroll
                for (int e = 0; e < 8; ++e) {
                    if ((Cfg::kEmuPairs >> (e >> 1)) & 1u) mpoly = fmaxf(mpoly, mx[e]);
                    else mmufu = fmaxf(mmufu, mx[e]);
                }
                const float mt = fmaxf(mpoly, mmufu);
                const float m_tile = mt * sl2;
                const float m_cand = fmaxf(m_use, m_tile);
                if (j == 0) {
                    m_use = m_cand;
                } else {
                    const bool need = m_cand > m_use + 8.0f;
                    if (__any_sync(0xffffffffu, need)) {
                        const float alpha = need ? ex2_approx(m_use - m_cand) : 1.0f;
                        if (need) {
                            l *= alpha;
                            m_use = m_cand;
                        }
#pragma unroll 1
                        for (int c = 0; c < D / 16; ++c) {
                            uint32_t r[16];
                            tmem_ld16(tO + c * 16, r);
                            tmem_wait_ld();
#pragma unroll
                            for (int e = 0; e < 16; ++e)
                                r[e] = __float_as_uint(__uint_as_float(r[e]) * alpha);
                            tmem_st16(tO + c * 16, r);
                        }
                    }
                }
                const float mb = (m_use == -INFINITY) ? 0.f : m_use;
                const float2 sl2x2 = make_float2(sl2, sl2), nmb2 = make_float2(-mb, -mb);
                float2 acc[4] = {make_float2(0.f, 0.f), make_float2(0.f, 0.f), make_float2(0.f, 0.f),
                                 make_float2(0.f, 0.f)};
#pragma unroll
                for (int c = 0; c < BN / 32; ++c) {
                    uint32_t pk[16];
#pragma unroll
                    for (int e = 0; e < 16; ++e) {
                        const float2 x = ffma2(make_float2(s[c * 32 + 2 * e], s[c * 32 + 2 * e + 1]), sl2x2, nmb2);
                        // a share of the exponentials runs on the FMA pipe (kEmuPairs bit e)
                        const float2 pe = ((Cfg::kEmuPairs >> e) & 1u)
                                              ? exp2_poly2(x)
                                              : make_float2(ex2_approx(x.x), ex2_approx(x.y));
                        acc[e & 3] = fadd2(acc[e & 3], pe);
                        pk[e] = pack_bf16x2(pe.x, pe.y);
                    }
                    tmem_st16(tS + c * 16, pk);
                    if (Cfg::kSplitPV && c == BN / 64 - 1) {
                        // first half of P (keys 0..63) is in place: let its PV start
                        tmem_wait_st();
                        tc_fence_before();
                        __syncwarp();
                        if (lane == 0) mbar_arrive(bar_p_half + 8 * t);
                    }
                }
                const float2 a01 = fadd2(acc[0], acc[1]), a23 = fadd2(acc[2], acc[3]);
                const float2 asum = fadd2(a01, a23);
                // l must sum the weights V is multiplied by, i.e. P as rounded to
                // bf16.  Only the largest P matters (when one key dominates a row its
                // rounding would scale the whole output; the others' average out): it
                // is recomputed exactly as its element computed it, by the same
                // exponential, and its rounding added
                const float xm = fmaf(mt, sl2, -mb);
                const float pm = (mpoly >= mmufu) ? exp2_poly2(make_float2(xm, xm)).x : ex2_approx(xm);
                l += asum.x + asum.y + (__bfloat162float(__float2bfloat16_rn(pm)) - pm);
                tmem_wait_st();
                tc_fence_before();
                __syncwarp();
                if (lane == 0) mbar_arrive(bar_p_full + 8 * t);
            }
            if (!ok) break;
            if (!__all_sync(0xffffffffu, mbar_wait_bounded(bar_o_full + 8 * t, oc & 1, abort_flag, limit))) {
                ok = false;
                break;
            }
            ++oc;
            tc_fence_after();
            const int h = p.qpair ? P.h0 : P.h0 + t;
            bool valid_row = i_rel < P.nq;
            if (kBoundsCheck && valid_row)
                valid_row = in_bounds((long long)P.orow0 + i_rel, p.cu_seqlens ? p.Nq : (long long)p.B * p.Nq) &&
                            in_bounds(h, p.Hq);
            const float inv_l = (l > 0.f) ? 1.0f / l : 0.f;
            __nv_bfloat16 *orow = p.out + ((P.orow0 + i_rel) * p.Hq + h) * D;
#pragma unroll
            for (int c = 0; c < D / 32; ++c) {
                uint32_t r[32];
                tmem_ld32(tO + c * 32, r);
                tmem_wait_ld();
                uint32_t pk[16];
#pragma unroll
                for (int e = 0; e < 16; ++e)
                    pk[e] = pack_bf16x2(__uint_as_float(r[2 * e]) * inv_l,
                                        __uint_as_float(r[2 * e + 1]) * inv_l);
                // each thread writes its own row (rows are Hq*D*2 bytes apart), so
                // every store instruction touches 32 lines: wider stores mean fewer
                // of them, which shortens the epilogue between units
                if (valid_row && p.out_v8) {
                    st_global_v8(orow + c * 32, pk);
                    st_global_v8(orow + c * 32 + 16, pk + 8);
                } else if (valid_row) {
                    uint4 *dst = reinterpret_cast<uint4 *>(orow + c * 32);
#pragma unroll
                    for (int v4 = 0; v4 < 4; ++v4)
                        dst[v4] = make_uint4(pk[4 * v4], pk[4 * v4 + 1], pk[4 * v4 + 2], pk[4 * v4 + 3]);
                }
            }
            tc_fence_before();
        }
    }

    tc_fence_before();
    __syncthreads();
    if (warp == 2) {
        tc_fence_after();
        tmem_dealloc(tmem, Cfg::TMEM_COLS);
    }
}

}  // namespace swa
