// device_common.cuh -- sm_100a building blocks shared by the libswa kernels:
// shared-memory barriers with bounded waits, TMA tile loads, and the tcgen05
// tensor-core / tensor-memory instructions, each as a thin inline-PTX wrapper.
#pragma once

#include <cstdint>
#include <cuda.h>
#include <cuda_bf16.h>

namespace swa {

// ---------------------------------------------------------------------------
// Device status word and wait limit (one per device, per loaded library).
// ---------------------------------------------------------------------------
__device__ int g_status = 0;                               // swa_status_t
__device__ unsigned long long g_wait_limit_ns = 1000000000ull;

constexpr int kStatusInvalid = 1;                          // SWA_ERR_INVALID_ARG (bad device-side input)
constexpr int kStatusTimeout = 4;                          // SWA_ERR_TIMEOUT

__device__ __forceinline__ unsigned long long globaltimer_ns() {
    unsigned long long t;
    asm volatile("mov.u64 %0, %globaltimer;" : "=l"(t));
    return t;
}

__device__ __forceinline__ void record_status(int code) {
    atomicCAS(&g_status, 0, code);
}

// Index checks of the bounds-checked build (compiled with SWA_BOUNDS_CHECK):
// every global row, slot and TMA start coordinate a kernel computes is checked
// against the extent of its tensor before use.  A failed check records
// SWA_ERR_INVALID_ARG in the status word and the access is skipped (or, for a
// TMA load whose barrier must still complete, redirected to coordinate 0); no
// trap.  In the normal build the checks compile to nothing.
#ifdef SWA_BOUNDS_CHECK
constexpr bool kBoundsCheck = true;
#else
constexpr bool kBoundsCheck = false;
#endif

__device__ __forceinline__ bool in_bounds(long long idx, long long n) {
    if (!kBoundsCheck || (idx >= 0 && idx < n)) return true;
    record_status(kStatusInvalid);
    return false;
}

// A TMA start coordinate: itself when inside [0, n), else 0 (recorded).
__device__ __forceinline__ int checked_coord(int c, int n) { return in_bounds(c, n) ? c : 0; }

__device__ __forceinline__ uint32_t smem_addr(const void *p) {
    return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

// ---------------------------------------------------------------------------
// mbarrier
// ---------------------------------------------------------------------------
__device__ __forceinline__ void mbar_init(uint32_t bar, uint32_t count) {
    asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(bar), "r"(count) : "memory");
}

__device__ __forceinline__ void mbar_init_fence() {
    asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint32_t bar) {
    asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(bar) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint32_t bar, uint32_t bytes) {
    asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(bar), "r"(bytes)
                 : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Non-blocking probe of the same condition (no suspension of the thread).
__device__ __forceinline__ bool mbar_test_wait(uint32_t bar, uint32_t parity) {
    uint32_t ok;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.test_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(ok)
        : "r"(bar), "r"(parity)
        : "memory");
    return ok != 0;
}

// Wait until the phase of parity `parity` of barrier `bar` has completed.
// Bounded: gives up when *abort becomes non-zero (another thread of the block
// gave up) or after `limit_ns`; on running out it records SWA_ERR_TIMEOUT,
// raises *abort and returns false.  Never traps.
// kSpin: poll without suspending (for a latency-critical single thread).
template <bool kSpin = false>
__device__ __forceinline__ bool mbar_wait_bounded(uint32_t bar, uint32_t parity,
                                                  volatile int *abort,
                                                  unsigned long long limit_ns) {
    if (kSpin ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (kSpin ? mbar_test_wait(bar, parity) : mbar_try_wait(bar, parity)) return true;
        if ((spin & 31u) == 0u) {
            if (*abort) return false;
            if (globaltimer_ns() - t0 >= limit_ns) {
                *abort = 1;
                record_status(kStatusTimeout);
                return false;
            }
        }
    }
}

// Clean-up waits (copies and MMAs this thread already started) have their own
// bound, independent of the wait limit a caller may have shortened: work in
// flight completes in microseconds, and the block must not exit before it has.
constexpr unsigned long long kDrainLimitNs = 2000000000ull;

// Same, for the clean-up path: ignores *abort, only the time limit ends it.
__device__ __forceinline__ bool mbar_drain_bounded(uint32_t bar, uint32_t parity,
                                                   unsigned long long limit_ns) {
    if (mbar_try_wait(bar, parity)) return true;
    const unsigned long long t0 = globaltimer_ns();
    for (uint32_t spin = 1;; ++spin) {
        if (mbar_try_wait(bar, parity)) return true;
        if ((spin & 31u) == 0u && globaltimer_ns() - t0 >= limit_ns) {
            record_status(kStatusTimeout);
            return false;
        }
    }
}

// ---------------------------------------------------------------------------
// Thread-block clusters: rank, a barrier of all threads of all blocks, and
// loads from a peer block's shared memory (distributed shared memory).
// ---------------------------------------------------------------------------
__device__ __forceinline__ uint32_t cluster_rank() {
    uint32_t r;
    asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
    return r;
}

// Release / acquire: shared-memory writes before it are visible to every
// block of the cluster after it.  Every thread of every block must reach it.
__device__ __forceinline__ void cluster_sync_all() {
    asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;" ::: "memory");
}

// Address, in the cluster window, of the same shared-memory offset in block `rank`.
__device__ __forceinline__ uint32_t peer_addr(uint32_t local_addr, uint32_t rank) {
    uint32_t a;
    asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(a) : "r"(local_addr), "r"(rank));
    return a;
}

__device__ __forceinline__ float ld_peer_f32(uint32_t local_addr, uint32_t rank) {
    float v;
    asm volatile("ld.shared::cluster.f32 %0, [%1];" : "=f"(v) : "r"(peer_addr(local_addr, rank)) : "memory");
    return v;
}

// ---------------------------------------------------------------------------
// TMA: tiled 4-D tensor load into shared memory, completion on an mbarrier.
// Coordinates are element indices, innermost first.  No multicast.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tma_load_4d(uint32_t dst, const CUtensorMap *map, uint32_t bar,
                                            int c0, int c1, int c2, int c3) {
    asm volatile(
        "cp.async.bulk.tensor.4d.shared::cluster.global.mbarrier::complete_tx::bytes"
        " [%0], [%1, {%3, %4, %5, %6}], [%2];" ::"r"(dst),
        "l"(reinterpret_cast<uint64_t>(map)), "r"(bar), "r"(c0), "r"(c1), "r"(c2), "r"(c3)
        : "memory");
}

__device__ __forceinline__ void prefetch_tensormap(const CUtensorMap *map) {
    asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// ---------------------------------------------------------------------------
// tcgen05: tensor memory allocation, MMA, commit, loads/stores, fences.
// ---------------------------------------------------------------------------
__device__ __forceinline__ void tmem_alloc(uint32_t dst_smem, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(dst_smem),
                 "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
                 : "memory");
}

__device__ __forceinline__ void tc_fence_before() {
    asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

__device__ __forceinline__ void tc_fence_after() {
    asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}

// D[tmem] (+)= A[smem desc] * B[smem desc]^T, kind::f16 (bf16 in, fp32 acc).
__device__ __forceinline__ void mma_ss(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// D[tmem] (+)= A[tmem] * B[smem desc], kind::f16.
__device__ __forceinline__ void mma_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t b_desc,
                                       uint32_t idesc, uint32_t accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n\t}" ::"r"(d_tmem),
        "r"(a_tmem), "l"(b_desc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation issued so far by this
// thread has completed.
__device__ __forceinline__ void mma_commit(uint32_t bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     bar)
                 : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
    asm volatile("tcgen05.wait::st.sync.aligned;" ::: "memory");
}

// Warp-collective: thread t of the warp reads 32 consecutive 32-bit columns
// of TMEM lane (lane_base + t), starting at column `col` of `taddr`.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, "
        "%16, %17, %18, %19, %20, %21, %22, %23, %24, %25, %26, %27, %28, %29, %30, %31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
          "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
          "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
        "{%0, %1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
          "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
    asm volatile(
        "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
        "{%1, %2, %3, %4, %5, %6, %7, %8, %9, %10, %11, %12, %13, %14, %15, %16};" ::"r"(taddr),
        "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
        "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
        "r"(r[15])
        : "memory");
}

// ---------------------------------------------------------------------------
// UMMA shared-memory matrix descriptor (sm_100 format): start address, leading
// and stride byte offsets (16-byte units), descriptor version 1, swizzle mode.
// ---------------------------------------------------------------------------
constexpr uint64_t kSwizzle128B = 2;

// Built as two 32-bit words.  lo holds the start address and
// the leading byte offset, hi the stride byte offset, version and swizzle, so
// stepping a descriptor along K inside a 128-byte swizzle row, or from one
// tile slot to the next, is a single 32-bit add on lo (the 14-bit address
// field of shared memory below 256 KB never carries into the offset field).
__host__ __device__ constexpr uint32_t smem_desc_hi(uint32_t sbo_bytes) {
    return ((sbo_bytes >> 4) & 0x3FFFu) | (1u << 14) | ((uint32_t)kSwizzle128B << 29);
}
__device__ __forceinline__ uint32_t smem_desc_lo(uint32_t saddr, uint32_t lbo_bytes) {
    return ((saddr >> 4) & 0x3FFFu) | (((lbo_bytes >> 4) & 0x3FFFu) << 16);
}
__device__ __forceinline__ uint64_t smem_desc64(uint32_t lo, uint32_t hi) {
    return ((uint64_t)hi << 32) | lo;
}

// Instruction descriptor of tcgen05.mma kind::f16: fp32 accumulator, bf16 A
// and B, A K-major, B K-major (b_mn_major = 0) or MN-major (1), shape M x N.
__host__ __device__ constexpr uint32_t make_idesc_bf16(int M, int N, int b_mn_major) {
    return (1u << 4)                        // D format: f32
         | (1u << 7)                        // A format: bf16
         | (1u << 10)                       // B format: bf16
         | ((uint32_t)b_mn_major << 16)     // B major
         | ((uint32_t)(N >> 3) << 17)       // N / 8
         | ((uint32_t)(M >> 4) << 24);      // M / 16
}

// Ties the 32 registers of a tcgen05.ld to program order after the
// tcgen05.wait::ld that precedes it, so no use is scheduled above the wait.
__device__ __forceinline__ void reg_fence32(uint32_t (&r)[32]) {
    asm volatile(""
                 : "+r"(r[0]), "+r"(r[1]), "+r"(r[2]), "+r"(r[3]), "+r"(r[4]), "+r"(r[5]),
                   "+r"(r[6]), "+r"(r[7]), "+r"(r[8]), "+r"(r[9]), "+r"(r[10]), "+r"(r[11]),
                   "+r"(r[12]), "+r"(r[13]), "+r"(r[14]), "+r"(r[15]), "+r"(r[16]), "+r"(r[17]),
                   "+r"(r[18]), "+r"(r[19]), "+r"(r[20]), "+r"(r[21]), "+r"(r[22]), "+r"(r[23]),
                   "+r"(r[24]), "+r"(r[25]), "+r"(r[26]), "+r"(r[27]), "+r"(r[28]), "+r"(r[29]),
                   "+r"(r[30]), "+r"(r[31]));
}

// Packed two-lane fp32 arithmetic (sm_100): one instruction for two values.
__device__ __forceinline__ float2 ffma2(float2 a, float2 b, float2 c) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rc, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\tmov.b64 rc, {%6, %7};\n\t"
        "fma.rn.f32x2 rd, ra, rb, rc;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y), "f"(c.x), "f"(c.y));
    return d;
}

__device__ __forceinline__ float2 fadd2(float2 a, float2 b) {
    float2 d;
    asm("{\n\t.reg .b64 ra, rb, rd;\n\t"
        "mov.b64 ra, {%2, %3};\n\tmov.b64 rb, {%4, %5};\n\t"
        "add.rn.f32x2 rd, ra, rb;\n\tmov.b64 {%0, %1}, rd;\n\t}"
        : "=f"(d.x), "=f"(d.y)
        : "f"(a.x), "f"(a.y), "f"(b.x), "f"(b.y));
    return d;
}

// 2^x for two values on the FMA pipe (offloads the exponential unit).
// Range reduction in the Cody-Waite manner: x = n + f with n = round(x) taken
// from the low mantissa bits of x + 1.5*2^23, f = x - n in [-0.5, 0.5]; 2^f
// by a degree-3 polynomial fitted for this code (iteratively reweighted least
// squares on Chebyshev nodes toward minimax relative error: 7.5e-5 on
// [-0.5, 0.5]); 2^n is added into the exponent field.  x is clamped at -126
// so masked (-inf) inputs give a positive value below 2^-125.
__device__ __forceinline__ float2 exp2_poly2(float2 x) {
    constexpr float kShift = 12582912.0f;                       // 1.5 * 2^23
    constexpr float c0 = 0.99992806f, c1 = 0.69326097f, c2 = 0.24261113f, c3 = 0.05517165f;
    x.x = fmaxf(x.x, -126.0f);
    x.y = fmaxf(x.y, -126.0f);
    const float2 t = fadd2(x, make_float2(kShift, kShift));
    const float2 n = fadd2(t, make_float2(-kShift, -kShift));    // round(x), exact
    const float2 f = ffma2(n, make_float2(-1.0f, -1.0f), x);     // x - n, exact
    float2 p = ffma2(f, make_float2(c3, c3), make_float2(c2, c2));
    p = ffma2(p, f, make_float2(c1, c1));
    p = ffma2(p, f, make_float2(c0, c0));
    return make_float2(__uint_as_float(__float_as_uint(p.x) + (__float_as_uint(t.x) << 23)),
                       __uint_as_float(__float_as_uint(p.y) + (__float_as_uint(t.y) << 23)));
}


// One 32-byte global store of eight 32-bit words (address 32-byte aligned):
// a full sector per thread, half the store instructions of 16-byte stores.
__device__ __forceinline__ void st_global_v8(void *ptr, const uint32_t *w) {
    asm volatile("st.global.v8.b32 [%0], {%1, %2, %3, %4, %5, %6, %7, %8};" ::"l"(ptr), "r"(w[0]), "r"(w[1]),
                 "r"(w[2]), "r"(w[3]), "r"(w[4]), "r"(w[5]), "r"(w[6]), "r"(w[7])
                 : "memory");
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
    __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
    return *reinterpret_cast<uint32_t *>(&v);
}

// acc.x += low bf16 half of w, acc.y += high half (each widened exactly to
// fp32).  Lets a softmax sum the weights it actually multiplies V by, i.e. P
// after its rounding to bf16, so that O / l is a convex combination of the
// value rows: when one key dominates a row, its rounding cancels instead of
// showing as a relative error of the whole output.
__device__ __forceinline__ float2 add_bf16x2(float2 acc, uint32_t w) {
    asm("{\n\t.reg .b16 lo, hi;\n\tmov.b32 {lo, hi}, %2;\n\t"
        "add.rn.f32.bf16 %0, lo, %0;\n\tadd.rn.f32.bf16 %1, hi, %1;\n\t}"
        : "+f"(acc.x), "+f"(acc.y)
        : "r"(w));
    return acc;
}

// Rotary embedding frequencies theta^(-2i/D), i < D/2, computed on the host
// in double precision and passed by value.
struct RopeTable {
    double f[64];
};

// Generic-proxy writes to shared memory become visible to the async proxy
// (TMA, tensor core) after this fence.
__device__ __forceinline__ void fence_proxy_async_smem() {
    asm volatile("fence.proxy.async.shared::cta;" ::: "memory");
}

// cos and sin of p * f: the angle is formed and reduced to [-pi, pi] in
// double precision, then evaluated with the fast single-precision intrinsic
// (absolute error below 2^-21 on [-pi, pi], far below the bf16 step).
__device__ __forceinline__ void rope_cos_sin(double p, double f, float &c, float &s) {
    constexpr double kTwoPi = 6.283185307179586;
    const double a = p * f;
    const double r = fma(-rint(a * (1.0 / kTwoPi)), kTwoPi, a);
    __sincosf((float)r, &s, &c);
}

// Rotate four adjacent (even, odd) bf16 pairs held in a 16-byte word; pairs
// i0 .. i0+3 of the row, position p.
__device__ __forceinline__ uint4 rope_rotate8(uint4 w, int i0, double p, const RopeTable &tab) {
    uint32_t in[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
    for (int e = 0; e < 4; ++e) {
        float c, s;
        rope_cos_sin(p, tab.f[i0 + e], c, s);
        const float x0 = __uint_as_float(in[e] << 16), x1 = __uint_as_float(in[e] & 0xFFFF0000u);
        in[e] = pack_bf16x2(x0 * c - x1 * s, x0 * s + x1 * c);
    }
    return make_uint4(in[0], in[1], in[2], in[3]);
}

__device__ __forceinline__ float ex2_approx(float x) {
    float y;
    asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
    return y;
}


}  // namespace swa
