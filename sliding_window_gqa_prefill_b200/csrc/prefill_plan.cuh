// prefill_plan.cuh -- work decomposition of the banded prefill: the launch
// parameters, the work units and the key tiles each unit visits.
//
// Shared by the kernel (every warp of a CTA derives its units from these
// functions) and by the host (which picks the decomposition of a launch);
// everything here also compiles for the host, so the schedule can be
// enumerated and checked on a CPU: every query row of every head computed
// by exactly one unit, and the tiles of a unit holding exactly the keys of
// each of its rows' windows (i-W < j <= i, sinks and the rolling buffer's
// slots included).  Sources: the SWA mask of "핵심 구성요소" of the
// "Mistral 7B -- Sliding Window Attention" summary (band of W keys), its
// "Pre-fill + Chunking" section and section 4.1 / Figure 3 of the manon006
// review (a chunk attends to the buffer and to itself).
#pragma once

#include "device_common.cuh"

namespace swa {

// Read-only int32 load (the read-only data path on the device).
__host__ __device__ __forceinline__ int32_t ld_i32(const int32_t *p) {
#ifdef __CUDA_ARCH__
    return __ldg(p);
#else
    return *p;
#endif
}

// Records a malformed device-side input in the status word (device only).
__host__ __device__ __forceinline__ void note_invalid() {
#ifdef __CUDA_ARCH__
    record_status(kStatusInvalid);
#endif
}

struct PrefillParams {
    int B;            // sequences
    int Nq;           // query rows per sequence (N, or C in chunk mode)
    int Nk;           // rows of the main k/v tensors (== Nq)
    int Hq, Hkv, G;   // heads, G = Hq / Hkv
    int W;            // window (keys i-W < j <= i)
    int npairs;       // ceil(G / 2)
    int nqb;          // ceil(Nq / 128)
    int num_units;    // B * Hkv * npairs * nqb, plus one per pair unit split in two
    // pair units with index >= split_from are split into two single-head units
    // (fills the last wave of CTAs; == the pair-unit count when nothing is split)
    int split_from;
    float scale_log2; // softmax scale * log2(e)
    int chunk_mode;   // 1: keys also come from the rolling-buffer cache
    const int32_t *start_pos;  // chunk mode: [B] first position of the chunk
    __nv_bfloat16 *out;        // [B, Nq, Hq, D]
    int out_v8;                // 1: out is 32-byte aligned (rows of 128 or 256 bytes): 32-byte stores
    int rope;                  // 1: rotate each Q tile in shared memory after its load
    RopeTable rope_freq;       // theta^(-2i/D), i < D/2
    // variable-length batch: q/k/v/out packed as [total, H, D]; sequence b is
    // rows cu_seqlens[b] .. cu_seqlens[b+1]-1 (null: fixed-length [B, N, H, D])
    const int32_t *cu_seqlens;
    // 1 (odd group of heads): the two head slots of a unit are two
    // consecutive 128-row query blocks of one head, which share the key tiles
    // of their bands, instead of two heads of the group; npairs is then G (one
    // head per unit) and nqb counts the 256-row pairs (a packed batch's
    // prefix sums count them per sequence)
    int qpair;
    // variable-length chunk batch: 1 leaves sequences of one row to the
    // decode kernel (no work units for them)
    int skip_len1;
    // 1 (odd group, a launch whose single-head units all fit in one wave):
    // every unit is one query head of the group (npairs = G) and one 128-row
    // block, so the SMs a pair launch would leave idle take the second heads
    int single;
    // attention sinks (one-shot prefill): positions j < sinks stay visible to
    // every query besides its window
    int sinks;
    // attention sinks (chunk mode): slots 0 .. sink_buf-1 of the sink buffer
    // hold positions 0 .. sink_buf-1; those outside a query's window are
    // visible to it (0: no sinks)
    int sink_buf;
};

constexpr int kMaxVarlenSeqs = 256;     // sequences per variable-length launch

struct UnitPlan {
    int b, g, pair, qb;
    int h0;          // query head of the unit's first head slot
    int q0;          // first query row (relative to the q tensor)
    int s0;          // absolute position of query row 0 of the sequence (chunk start, or 0)
    int qs;          // s0 mod W (slot the next position would take)
    int act1;        // second query head (or block) of the pair exists
    int nc1, c1;     // cache run 1: tiles c1 .. c1+nc1-1
    int nc2, c2;     // cache run 2
    int nm, m0;      // main tiles m0 .. m0+nm-1
    int sink_tile;   // sink tiles visited first: main tiles below the band (one-shot) or
                     // sink-buffer tiles (chunk mode)
    int n;           // total tiles
    int nq;          // query rows of this sequence (== rows of its main k/v)
    int row0;        // first packed row of this sequence in q/k/v (varlen), else 0
    int tb;          // TMA batch coordinate of q/k/v (0 when packed)
    size_t orow0;    // output row of query row 0 of this sequence
};

// Rows of sequence b of a packed batch: cu_seqlens[b+1] - cu_seqlens[b] when
// 0 <= cu[b] <= cu[b+1] <= total rows, else 0 (a malformed sequence is
// skipped, so no row outside the packed tensors is ever read or written).
__host__ __device__ __forceinline__ int varlen_rows(const PrefillParams &p, int b) {
    const int c0 = ld_i32(p.cu_seqlens + b), c1 = ld_i32(p.cu_seqlens + b + 1);
    return (c0 >= 0 && c0 <= c1 && c1 <= p.Nq) ? c1 - c0 : 0;
}

// Query rows whose key tiles a unit visits, from q0: 256 for a pair of query
// blocks whose second block exists, else 128 (a head pair, a split pair, or
// a pair whose second block lies past the sequence, whose rows all sit
// below q0 + 128).
__host__ __device__ __forceinline__ int unit_span(const PrefillParams &p, const UnitPlan &P) {
    return (p.qpair && P.act1) ? 256 : 128;
}

// pre: prefix sums of query blocks (pairs of blocks with qpair) per sequence
// (packed batches only; varlen_prefix).
__host__ __device__ __forceinline__ UnitPlan plan_unit(const PrefillParams &p, int u, const int *pre) {
    constexpr int BM = 128, BN = 128;
    UnitPlan P;
    int which = -1;
    if (p.cu_seqlens) {
        const int per = p.Hkv * p.npairs;
        const int qbi = pre[p.B] - 1 - u / per;        // later blocks first
        int r = u % per;
        P.pair = r % p.npairs;
        P.g = r / p.npairs;
        int lo = 0, hi = p.B - 1;                       // last b with pre[b] <= qbi
        while (lo < hi) {
            const int mid = (lo + hi + 1) >> 1;
            if (pre[mid] <= qbi) lo = mid; else hi = mid - 1;
        }
        P.b = lo;
        P.qb = qbi - pre[lo];
        const int c0 = ld_i32(p.cu_seqlens + lo);
        P.nq = varlen_rows(p, lo);
        P.row0 = P.nq > 0 ? c0 : 0;
        P.tb = 0;
        P.orow0 = (size_t)c0;
    } else {
        int pu = u;                          // pair unit; which: head (or block) of a split unit
        if (u >= p.split_from) {
            pu = p.split_from + (u - p.split_from) / 2;
            which = (u - p.split_from) & 1;
        }
        const int per = p.B * p.Hkv * p.npairs;
        P.qb = p.nqb - 1 - pu / per;         // latest (heaviest) query blocks first
        int r = pu % per;
        P.pair = r % p.npairs;
        r /= p.npairs;
        P.g = r % p.Hkv;
        P.b = r / p.Hkv;
        P.nq = p.Nq;
        P.row0 = 0;
        P.tb = P.b;
        P.orow0 = (size_t)P.b * p.Nq;
    }
    P.q0 = P.qb * (p.qpair ? 2 * BM : BM);
    if (p.qpair) {
        P.h0 = P.g * p.G + P.pair;                   // one head per unit (npairs = G)
        // a split pair is one of its two blocks; else the second block exists
        // unless the sequence ends in the first
        if (which > 0) P.q0 += BM;
        P.act1 = which < 0 && P.q0 + BM < P.nq;
    } else {
        // head pairs (a split pair: one of its heads); single: one head per
        // unit (npairs = G)
        P.act1 = !p.single && which < 0 && (2 * P.pair + 1) < p.G;
        P.h0 = P.g * p.G + (p.single ? P.pair : 2 * P.pair + (which > 0 ? 1 : 0));
    }
    const int span = unit_span(p, P);
    P.nc1 = P.nc2 = 0;
    P.c1 = P.c2 = 0;
    if (!p.chunk_mode) {
        P.s0 = 0;
        P.qs = 0;
        const int lo = max(0, P.q0 - p.W + 1);
        const int hi = min(P.nq - 1, P.q0 + span - 1);
        P.m0 = lo / BN;
        P.nm = hi / BN - P.m0 + 1;
        // sink positions below the band live in the first ceil(S/128) tiles
        P.sink_tile = min((p.sinks + BN - 1) / BN, P.m0);
    } else {
        P.s0 = ld_i32(p.start_pos + P.b);
        if (P.s0 < 0) {                       // invalid start: record it, attend as if 0
            note_invalid();
            P.s0 = 0;
        }
        // sink positions j <= i - W exist for some row i of the block
        P.sink_tile = (p.sink_buf > 0 && (long long)P.s0 + P.q0 + span - 1 >= p.W) ? (p.sink_buf + BN - 1) / BN : 0;
        P.qs = P.s0 % p.W;
        // oldest age any row of the block still needs: age < W - q0, age <= s0
        const int A = min(p.W - P.q0 - 1, P.s0);
        if (A >= 1) {
            int last1 = -1;
            if (P.qs >= 1) {                       // slots qs-A .. qs-1 (clipped at 0)
                const int lo1 = max(0, P.qs - A);
                P.c1 = lo1 / BN;
                last1 = (P.qs - 1) / BN;
                P.nc1 = last1 - P.c1 + 1;
            }
            if (A > P.qs) {                        // wrapped part: slots W-(A-qs) .. W-1
                int lo2t = (p.W - (A - P.qs)) / BN;
                if (lo2t <= last1) lo2t = last1 + 1;
                const int hi2t = (p.W - 1) / BN;
                if (lo2t <= hi2t) {
                    P.c2 = lo2t;
                    P.nc2 = hi2t - lo2t + 1;
                }
            }
        }
        const int lo = max(0, P.q0 - p.W + 1);          // chunks longer than W
        const int hi = min(P.nq - 1, P.q0 + span - 1);
        P.m0 = lo / BN;
        P.nm = hi / BN - P.m0 + 1;
    }
    P.n = P.sink_tile + P.nc1 + P.nc2 + P.nm;
    return P;
}

// Unit taken by CTA c of C in round k: rounds alternate direction, so the
// CTAs that drew the heavier units of one round draw the lighter ones of the
// next (units are ordered heaviest first), which evens out the per-CTA work;
// >= the unit count once the CTA has no more work.
__host__ __device__ __forceinline__ int unit_of(int k, int c, int C) {
    return k * C + ((k & 1) ? (C - 1 - c) : c);
}

// Key tile j of a unit: source (1 = cache), first row (slot or key index),
// and whether any element of the 128x128 tile may be masked.
struct TileRef {
    int cache;       // 0: main k/v, 1: rolling-buffer cache, 2: sink buffer (chunk mode)
    int row0;
    int masked;
};

__host__ __device__ __forceinline__ TileRef tile_ref(const PrefillParams &p, const UnitPlan &P, int j) {
    constexpr int BN = 128;
    // rows over which a tile is tested clean: both blocks of a pair, also
    // for a split pair (a superset of its rows, so the test stays exact)
    // -- a constant of the launch, so the softmax loop holds no extra state
    const int span = p.qpair ? 2 * BN : BN;
    TileRef t;
    if (j < P.sink_tile) {                  // only the sink positions of this tile count
        t.cache = p.chunk_mode ? 2 : 0;
        t.row0 = j * BN;
        t.masked = 1;
        return t;
    }
    j -= P.sink_tile;
    if (j < P.nc1 + P.nc2) {
        t.cache = 1;
        const int tile = (j < P.nc1) ? (P.c1 + j) : (P.c2 + (j - P.nc1));
        const int k0 = tile * BN;
        t.row0 = k0;
        const int t_last = min(P.q0 + span - 1, P.nq - 1);
        const bool has_qs = (k0 <= P.qs) && (P.qs < k0 + BN);
        const int max_age = (k0 + BN - 1 < P.qs) ? (P.qs - k0) : (p.W - (k0 - P.qs));
        const bool clean = !has_qs && (k0 + BN <= p.W) && (max_age < p.W - t_last) &&
                           (max_age <= P.s0);
        t.masked = !clean;
    } else {
        t.cache = 0;
        const int k0 = (P.m0 + (j - P.nc1 - P.nc2)) * BN;
        t.row0 = k0;
        const bool clean = (k0 + BN - 1 <= P.q0) && (k0 > P.q0 + span - 1 - p.W) && (k0 + BN <= P.nq);
        t.masked = !clean;
    }
    return t;
}

// Query blocks (pairs of blocks with qpair) per sequence of a packed batch,
// prefix-summed into pre[0..B] (empty or malformed sequences count as empty,
// as do sequences of one row with skip_len1).  Returns true if a malformed
// sequence was seen.
__host__ __device__ __forceinline__ bool varlen_prefix(const PrefillParams &p, int *pre) {
    const int rows = p.qpair ? 256 : 128;
    int acc = 0;
    bool bad = false;
    for (int b = 0; b < p.B; ++b) {
        pre[b] = acc;
        int n = varlen_rows(p, b);
        if (n == 0 && ld_i32(p.cu_seqlens + b + 1) != ld_i32(p.cu_seqlens + b)) bad = true;
        if (n == 1 && p.skip_len1) n = 0;
        acc += (n + rows - 1) / rows;
    }
    pre[p.B] = acc;
    return bad;
}

// ------------------------------------------------------------------ host side

// An odd group leaves the second head slot of its last pair unit empty (all
// of them for G = 1); with at least two waves of units (for a packed batch,
// by the host's upper bound), a unit takes two consecutive 128-row query
// blocks of one head
// instead (they share most key tiles), which keeps both softmax warpgroups
// busy (B=2, N=16K, W=4K: G=3 867 -> 1000, G=5 866 -> 995, G=7 854 -> 957
// TFLOP/s).  Even groups keep the pairs of heads, which also share each key
// tile between the two heads.
inline bool use_qpair(int G, long long units, int sms) {
    return G % 2 == 1 && units >= 2LL * sms;
}

// Chunk attention units (all about the same cost) fill whole waves of CTAs
// except the last; when that wave is at most half full, its pair units are
// split into two single-head units each, which fit in it and take about three
// quarters of a pair unit's time (all of them when the whole launch is at
// most half a wave).  Returns the first split pair unit and raises units by
// the number split.
inline int split_units(int &units, bool splittable, int sms) {
    if (!splittable || units > 0x7fffffff - sms) return units;
    if (2 * units <= sms) {           // a launch of at most half a wave: split every unit
        units *= 2;
        return 0;
    }
    if (units <= sms) return units;
    const int rem = units % sms;
    if (rem == 0 || 2 * rem > sms) return units;
    const int from = units - rem;
    units += rem;
    return from;
}

// Work decomposition of a launch over B sequences of Nq query rows (the
// chunk length in chunk mode), Hq / Hkv heads and a window of W keys: head
// pairs or, for odd groups, pairs of query blocks; the unit count (an upper
// bound for a packed batch, whose kernel counts them from cu_seqlens); the
// single-head split of a short last wave (chunk mode) or of a launch of at
// most half a wave (one-shot).  Fills the fields the planner reads that do
// not depend on device pointers.
inline void prefill_units(PrefillParams &p, int B, int Nq, int Hq, int Hkv, int W, bool varlen, bool chunk,
                          int sms) {
    const int G = Hq / Hkv;
    const long long nqb = (Nq + 127) / 128;
    const long long units = varlen ? (long long)Hkv * ((G + 1) / 2) * (nqb + B)
                                   : (long long)B * Hkv * ((G + 1) / 2) * nqb;
    p.B = B;
    p.Nq = Nq;
    p.Nk = Nq;
    p.Hq = Hq;
    p.Hkv = Hkv;
    p.G = G;
    p.W = W;
    p.npairs = (G + 1) / 2;
    p.nqb = (int)nqb;
    p.num_units = (int)units;
    p.qpair = 0;
    p.single = 0;
    if (use_qpair(G, units, sms)) {
        // pairs of query blocks: a packed sequence of n rows takes
        // ceil(n / 256) of them, at most N / 256 + 1
        p.qpair = 1;
        p.npairs = G;
        p.nqb = (int)((nqb + 1) / 2);
        p.num_units = (int)(varlen ? (long long)Hkv * G * (p.nqb + B) : (long long)B * Hkv * G * p.nqb);
    }
    p.chunk_mode = chunk ? 1 : 0;
    if (varlen) {
        p.split_from = 0x7fffffff;
    } else if (chunk) {
        // head pairs of an even group split into their two heads; pairs of
        // query blocks into their two blocks, unless a pair with one block
        // (the sequence's last, when Nq is not a multiple of 256) would be
        // among them
        int n = p.num_units;
        const int from = split_units(n, G % 2 == 0 || p.qpair, sms);
        const bool one_block_pair = p.qpair && Nq % 256 != 0 && from < B * Hkv * G;
        if (!one_block_pair) {
            p.split_from = from;
            p.num_units = n;
        } else {
            p.split_from = p.num_units;
        }
    } else {
        // the lightest blocks come last, so a full launch is not split; one of
        // at most half a wave runs as single-head units (an odd group's pairs
        // cannot be split in two, so its units are then the heads themselves)
        p.split_from = p.num_units;
        if (G % 2 == 0 && 2 * units <= sms) {
            p.split_from = 0;
            p.num_units = (int)units * 2;
        } else if (G % 2 == 1 && G > 1 && !p.qpair && (long long)B * Hkv * G * nqb <= sms) {
            p.single = 1;
            p.npairs = G;
            p.num_units = B * Hkv * G * (int)nqb;
            p.split_from = p.num_units;
        }
    }
}

}  // namespace swa
