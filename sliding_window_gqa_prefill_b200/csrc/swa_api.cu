// swa_api.cu -- host side of libswa: argument checks, TMA descriptors, launch
// configuration and the device status word.  All kernels are in the headers
// included below, compiled into this one translation unit.
#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include <cuda.h>
#include <cuda_runtime.h>

#include "../../include/swa.h"
#include "decode_kernel.cuh"
#include "device_common.cuh"
#include "prefill_kernel.cuh"

namespace {

thread_local int t_last_cuda_error = 0;

swa_status_t cuda_fail(cudaError_t e) {
    t_last_cuda_error = static_cast<int>(e);
    return SWA_ERR_CUDA;
}

#define SWA_CUDA_TRY(expr)                       \
    do {                                         \
        cudaError_t e_ = (expr);                 \
        if (e_ != cudaSuccess) return cuda_fail(e_); \
    } while (0)

bool aligned16(const void *p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// ----------------------------------------------------------------- TMA descriptors
using EncodeTiledFn = CUresult (*)(CUtensorMap *, CUtensorMapDataType, cuuint32_t, void *,
                                   const cuuint64_t *, const cuuint64_t *, const cuuint32_t *,
                                   const cuuint32_t *, CUtensorMapInterleave, CUtensorMapSwizzle,
                                   CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
    static EncodeTiledFn fn = nullptr;
    static std::once_flag once;
    std::call_once(once, [] {
        void *p = nullptr;
        cudaDriverEntryPointQueryResult q;
        if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
                cudaSuccess &&
            q == cudaDriverEntryPointSuccess)
            fn = reinterpret_cast<EncodeTiledFn>(p);
    });
    return fn;
}

// bf16 tensor [d3, d2, d1, d0] (d0 innermost, contiguous) as a 4-D TMA map
// with a (64, 1, 128, 1) box and 128-byte swizzle: one 128-row x 128-byte
// region of a K-major UMMA operand per load.  Out-of-range rows read as zero.
swa_status_t make_operand_map(CUtensorMap *map, const void *base, uint64_t d0, uint64_t d1,
                              uint64_t d2, uint64_t d3) {
    EncodeTiledFn fn = encode_fn();
    if (!fn) return cuda_fail(cudaErrorNotSupported);
    const cuuint64_t dims[4] = {d0, d1, d2, d3};
    const cuuint64_t strides[3] = {d0 * 2, d0 * d1 * 2, d0 * d1 * d2 * 2};   // bytes, dims 1..3
    const cuuint32_t box[4] = {64, 1, 128, 1};
    const cuuint32_t estr[4] = {1, 1, 1, 1};
    CUresult r = fn(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 4, const_cast<void *>(base), dims,
                    strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                    CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
    if (r != CUDA_SUCCESS) {
        t_last_cuda_error = static_cast<int>(r);
        return SWA_ERR_CUDA;
    }
    return SWA_OK;
}

// ----------------------------------------------------------------- device info
constexpr int kMaxDevices = 64;

struct DeviceInfo {
    int sms = 0;
    bool attrs_set = false;
};
DeviceInfo g_dev[kMaxDevices];
std::mutex g_dev_mu;

swa_status_t device_info(DeviceInfo **out) {
    int dev = 0;
    SWA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return SWA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_dev_mu);
    DeviceInfo &d = g_dev[dev];
    if (!d.attrs_set) {
        SWA_CUDA_TRY(cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev));
        SWA_CUDA_TRY(cudaFuncSetAttribute(swa::swa_prefill_kernel<64>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          swa::PrefillCfg<64>::SMEM_ALLOC));
        SWA_CUDA_TRY(cudaFuncSetAttribute(swa::swa_prefill_kernel<128>,
                                          cudaFuncAttributeMaxDynamicSharedMemorySize,
                                          swa::PrefillCfg<128>::SMEM_ALLOC));
#define SWA_SET_DECODE_ATTR(DD, GG)                                                           \
    SWA_CUDA_TRY(cudaFuncSetAttribute(swa::swa_decode_kernel<DD, GG, swa::kDecodeWindow>,    \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                      swa::DecodeCfg<DD, GG>::SMEM_BYTES));                  \
    SWA_CUDA_TRY(cudaFuncSetAttribute(swa::swa_decode_kernel<DD, GG, swa::kDecodeSinks>,     \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                      swa::DecodeCfg<DD, GG>::SMEM_BYTES));                  \
    SWA_CUDA_TRY(cudaFuncSetAttribute(swa::swa_decode_kernel<DD, GG, swa::kDecodePackedRows>, \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                      swa::DecodeCfg<DD, GG>::SMEM_BYTES));                  \
    SWA_CUDA_TRY(cudaFuncSetAttribute(swa::swa_decode_kernel<DD, GG, swa::kDecodeWindowCluster>, \
                                      cudaFuncAttributeMaxDynamicSharedMemorySize,           \
                                      swa::DecodeCfg<DD, GG>::SMEM_BYTES));
        SWA_SET_DECODE_ATTR(64, 1) SWA_SET_DECODE_ATTR(64, 2) SWA_SET_DECODE_ATTR(64, 3)
        SWA_SET_DECODE_ATTR(64, 4) SWA_SET_DECODE_ATTR(64, 5) SWA_SET_DECODE_ATTR(64, 6)
        SWA_SET_DECODE_ATTR(64, 7) SWA_SET_DECODE_ATTR(64, 8)
        SWA_SET_DECODE_ATTR(128, 1) SWA_SET_DECODE_ATTR(128, 2) SWA_SET_DECODE_ATTR(128, 3)
        SWA_SET_DECODE_ATTR(128, 4) SWA_SET_DECODE_ATTR(128, 5) SWA_SET_DECODE_ATTR(128, 6)
        SWA_SET_DECODE_ATTR(128, 7) SWA_SET_DECODE_ATTR(128, 8)
#undef SWA_SET_DECODE_ATTR
        d.attrs_set = true;
    }
    *out = &d;
    return SWA_OK;
}

// ----------------------------------------------------------------- common checks
swa_status_t check_heads(int Hq, int Hkv, int D) {
    if (Hq < 1 || Hkv < 1 || Hq % Hkv != 0) return SWA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
    return SWA_OK;
}

bool bad_scale(float s) { return !(std::isfinite(s) && s > 0.f); }

constexpr float kLog2e = 1.4426950408889634f;

template <int D>
// mks / mvs: sink-buffer maps (chunk mode with sinks), else any valid map.
swa_status_t launch_prefill(const CUtensorMap &mq, const CUtensorMap &mk, const CUtensorMap &mv,
                            const CUtensorMap &mkc, const CUtensorMap &mvc, const CUtensorMap &mks,
                            const CUtensorMap &mvs, const swa::PrefillParams &p, int sms, cudaStream_t s) {
    const int grid = p.num_units < sms ? p.num_units : sms;
    swa::swa_prefill_kernel<D><<<grid, swa::PrefillCfg<D>::THREADS, swa::PrefillCfg<D>::SMEM_ALLOC, s>>>(
        mq, mk, mv, mkc, mvc, mks, mvs, p);
    SWA_CUDA_TRY(cudaGetLastError());
    return SWA_OK;
}

swa_status_t launch_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                           const int32_t *pos, int B, int T, int Hkv, int D, int W, int sms,
                           const swa::RopeTable *rope, cudaStream_t s, void *k_sink = nullptr,
                           void *v_sink = nullptr, int S = 0) {
    const int row_vec = Hkv * D * 2 / 16;
    const long long total = (long long)B * T * row_vec;
    long long blocks = (total + 255) / 256;
    const long long cap = (long long)sms * 8;
    if (blocks > cap) blocks = cap;
    if (blocks < 1) blocks = 1;
    swa::swa_append_kernel<<<(int)blocks, 256, 0, s>>>(
        static_cast<const uint4 *>(k_new), static_cast<const uint4 *>(v_new),
        static_cast<uint4 *>(k_cache), static_cast<uint4 *>(v_cache), pos, B, T, W, row_vec, D / 8,
        rope ? 1 : 0, rope ? *rope : swa::RopeTable{}, static_cast<uint4 *>(k_sink),
        static_cast<uint4 *>(v_sink), S);
    SWA_CUDA_TRY(cudaGetLastError());
    return SWA_OK;
}

// Keys per decode split for a launch over L = W (+ S) keys: kDecodeSplit, or
// fewer (multiples of 64, at least kDecodeMinSplit) when B * Hkv windows of
// kDecodeSplit keys would give fewer than ~256 blocks, so that a small batch
// still spreads over the GPU.  A function of the sizes only: the workspace
// size follows from it.
int decode_split_keys(int B, int Hkv, int L) {
    const long long pairs = (long long)B * Hkv;
    const long long want = (256 + pairs - 1) / pairs;       // splits per (sequence, kv head)
    long long split = ((L + want - 1) / want + 63) / 64 * 64;
    if (split < swa::kDecodeMinSplit) split = swa::kDecodeMinSplit;
    if (split > swa::kDecodeSplit) split = swa::kDecodeSplit;
    return (int)split;
}

// The decode kernel takes the Hq/Hkv query heads that share a K/V head as
// the rows of its MMA tile, at most 8 at a time: a group of G heads runs as
// rep = G / Gt groups of Gt heads, Gt the largest divisor of G up to 8 (each
// K/V head then read rep times).  Returns Gt.
int decode_group(int Hq, int Hkv, int *rep) {
    const int G = Hq / Hkv;
    int gt = G < 8 ? G : 8;
    while (G % gt != 0) --gt;
    *rep = G / gt;
    return gt;
}

int decode_nsplit_max(int B, int Hkv, int L) {
    const int split = decode_split_keys(B, Hkv, L);
    return (int)(((long long)L + split - 1) / split);
}

// Grid (kDecodeClusterSplits, Hkv, B) in clusters of kDecodeClusterSplits
// along x: the splits of each window are merged through distributed shared
// memory, with no workspace.  MODE kDecodeWindowCluster: the window of the
// cache (knew / vnew / cu unused, total = B); kDecodePackedRows: the
// one-row sequences of a packed batch.
template <int D, int G, int MODE>
swa_status_t launch_decode_cluster(const void *q, const void *kc, const void *vc, const int32_t *pos,
                                   void *out, int B, int Hkv, int W, float scale,
                                   const swa::RopeTable *rope, const void *knew, const void *vnew,
                                   const int32_t *cu, int total, int kv_rep, cudaStream_t s) {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = dim3(swa::kDecodeClusterSplits, Hkv, B);
    cfg.blockDim = dim3(swa::kDecodeWarps * 32);
    cfg.dynamicSmemBytes = swa::DecodeCfg<D, G>::SMEM_BYTES;
    cfg.stream = s;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = swa::kDecodeClusterSplits;
    attr[0].val.clusterDim.y = 1;
    attr[0].val.clusterDim.z = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    float2 *no_ml = nullptr;
    float *no_o = nullptr;
    SWA_CUDA_TRY(cudaLaunchKernelEx(&cfg, swa::swa_decode_kernel<D, G, MODE>,
                                    static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(kc),
                                    static_cast<const __nv_bfloat16 *>(vc), pos, static_cast<__nv_bfloat16 *>(out),
                                    no_ml, no_o, Hkv, W, 1, scale * kLog2e, rope ? 1 : 0,
                                    rope ? *rope : swa::RopeTable{}, static_cast<const __nv_bfloat16 *>(knew),
                                    static_cast<const __nv_bfloat16 *>(vnew), 0, cu, total, 0, kv_rep));
    return SWA_OK;
}

// Hkv: groups of G query heads (kv_rep groups per K/V head in memory).
template <int D, int G>
swa_status_t launch_decode_dg(const void *q, const void *kc, const void *vc, const int32_t *pos,
                              void *out, int B, int Hkv, int W, float scale, void *ws,
                              const swa::RopeTable *rope, cudaStream_t s, const void *ksink,
                              const void *vsink, int S, int kv_rep) {
    const int nsm = decode_nsplit_max(B, Hkv, W + S);
    const int split = decode_split_keys(B, Hkv, W + S);
    const size_t o_elems = (size_t)B * Hkv * nsm * G * D;
    float *ws_o = static_cast<float *>(ws);
    float2 *ws_ml = ws ? reinterpret_cast<float2 *>(static_cast<char *>(ws) + ((o_elems * 4 + 255) & ~size_t(255)))
                       : nullptr;
    // a window of exactly kDecodeClusterSplits splits: merged in its cluster
    if (S == 0 && nsm == swa::kDecodeClusterSplits)
        return launch_decode_cluster<D, G, swa::kDecodeWindowCluster>(q, kc, vc, pos, out, B, Hkv, W, scale, rope,
                                                                      nullptr, nullptr, nullptr, B, kv_rep, s);
    dim3 grid(nsm, Hkv, B);
    auto kernel = S > 0 ? swa::swa_decode_kernel<D, G, swa::kDecodeSinks>
                        : swa::swa_decode_kernel<D, G, swa::kDecodeWindow>;
    kernel<<<grid, swa::kDecodeWarps * 32, swa::DecodeCfg<D, G>::SMEM_BYTES, s>>>(
        static_cast<const __nv_bfloat16 *>(q), static_cast<const __nv_bfloat16 *>(kc),
        static_cast<const __nv_bfloat16 *>(vc), pos, static_cast<__nv_bfloat16 *>(out), ws_ml, ws_o,
        Hkv, W, nsm, scale * kLog2e, rope ? 1 : 0, rope ? *rope : swa::RopeTable{},
        static_cast<const __nv_bfloat16 *>(ksink), static_cast<const __nv_bfloat16 *>(vsink), S,
        nullptr, 0, split, kv_rep);
    SWA_CUDA_TRY(cudaGetLastError());
    if (nsm > 1) {
        swa::swa_decode_combine_kernel<D, G><<<dim3(Hkv, B), G * D, 0, s>>>(
            pos, ws_ml, ws_o, static_cast<__nv_bfloat16 *>(out), Hkv, W, nsm, S, split);
        SWA_CUDA_TRY(cudaGetLastError());
    }
    return SWA_OK;
}

template <int D>
swa_status_t launch_decode_d(int G, int kv_rep, const void *q, const void *kc, const void *vc,
                             const int32_t *pos, void *out, int B, int Hkv, int W, float scale,
                             void *ws, const swa::RopeTable *rope, cudaStream_t s,
                             const void *ksink = nullptr, const void *vsink = nullptr, int S = 0) {
    switch (G) {
        case 1: return launch_decode_dg<D, 1>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 2: return launch_decode_dg<D, 2>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 3: return launch_decode_dg<D, 3>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 4: return launch_decode_dg<D, 4>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 5: return launch_decode_dg<D, 5>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 6: return launch_decode_dg<D, 6>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 7: return launch_decode_dg<D, 7>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        case 8: return launch_decode_dg<D, 8>(q, kc, vc, pos, out, B, Hkv, W, scale, ws, rope, s, ksink, vsink, S, kv_rep);
        default: return SWA_ERR_UNSUPPORTED;
    }
}

// The length-1 sequences of a packed chunk batch (q/k/v/out [total, H, D]):
// a cluster of kDecodeClusterSplits blocks per (sequence, kv head), merged in
// distributed shared memory; the other sequences' blocks return at once.
template <int D, int G>
swa_status_t launch_decode_packed_dg(const void *q, const void *k, const void *v, const void *kc,
                                     const void *vc, const int32_t *start_pos, const int32_t *cu,
                                     void *out, int B, int total, int Hkv, int W, float scale,
                                     cudaStream_t s, int kv_rep) {
    return launch_decode_cluster<D, G, swa::kDecodePackedRows>(q, kc, vc, start_pos, out, B, Hkv, W, scale, nullptr,
                                                               k, v, cu, total, kv_rep, s);
}

// false when the decode kernel has no instance for this head group
template <int D>
bool launch_decode_packed_d(int G, int kv_rep, swa_status_t *e, const void *q, const void *k, const void *v,
                            const void *kc, const void *vc, const int32_t *start_pos, const int32_t *cu,
                            void *out, int B, int total, int Hkv, int W, float scale, cudaStream_t s) {
    switch (G) {
        case 1: *e = launch_decode_packed_dg<D, 1>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 2: *e = launch_decode_packed_dg<D, 2>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 3: *e = launch_decode_packed_dg<D, 3>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 4: *e = launch_decode_packed_dg<D, 4>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 5: *e = launch_decode_packed_dg<D, 5>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 6: *e = launch_decode_packed_dg<D, 6>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 7: *e = launch_decode_packed_dg<D, 7>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        case 8: *e = launch_decode_packed_dg<D, 8>(q, k, v, kc, vc, start_pos, cu, out, B, total, Hkv, W, scale, s, kv_rep); return true;
        default: return false;
    }
}

__global__ void swa_selftest_wait_kernel() {
    __shared__ alignas(8) uint64_t bar;
    __shared__ int abort_flag;
    if (threadIdx.x == 0) {
        swa::mbar_init(swa::smem_addr(&bar), 1);
        abort_flag = 0;
        swa::mbar_init_fence();
    }
    __syncthreads();
    // nothing ever arrives on `bar`: the wait must run out and record the status
    swa::mbar_wait_bounded(swa::smem_addr(&bar), 0, &abort_flag, swa::g_wait_limit_ns);
}

// Scratch of swa_decode_noalloc: reserved statically on every device that
// loads this library, shared by all its calls.  Host code must not pass the
// symbol itself to a kernel (on the host it names a host-side shadow); the
// device address is looked up once per device with cudaGetSymbolAddress.
constexpr size_t kNoallocScratchBytes = SWA_DECODE_NOALLOC_SCRATCH_BYTES;
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoallocScratchBytes];

void *g_noalloc_ptr[kMaxDevices] = {};
std::mutex g_noalloc_mu;

swa_status_t noalloc_scratch(void **out) {
    int dev = 0;
    SWA_CUDA_TRY(cudaGetDevice(&dev));
    if (dev < 0 || dev >= kMaxDevices) return SWA_ERR_UNSUPPORTED;
    std::lock_guard<std::mutex> lk(g_noalloc_mu);
    if (!g_noalloc_ptr[dev]) {
        void *p = nullptr;
        SWA_CUDA_TRY(cudaGetSymbolAddress(&p, g_noalloc_scratch));   // device `dev` is current
        g_noalloc_ptr[dev] = p;
    }
    *out = g_noalloc_ptr[dev];
    return SWA_OK;
}

__global__ void swa_selftest_exp2_kernel(const float *x, float *y, int n) {
    const int i = 2 * (blockIdx.x * blockDim.x + threadIdx.x);
    if (i + 1 < n) {
        const float2 r = swa::exp2_poly2(make_float2(x[i], x[i + 1]));
        y[i] = r.x;
        y[i + 1] = r.y;
    } else if (i < n) {
        y[i] = swa::exp2_poly2(make_float2(x[i], 0.f)).x;
    }
}

// ----------------------------------------------------------------- implementations
// `rope` null: no rotary embedding; otherwise the frequency table.

bool bad_theta(float theta) { return !(std::isfinite(theta) && theta > 1.f); }

swa::RopeTable make_rope_table(float theta, int D) {
    swa::RopeTable t{};
    for (int i = 0; i < D / 2 && i < 64; ++i) t.f[i] = std::pow((double)theta, -2.0 * i / D);
    return t;
}

// cu_seqlens non-null: variable-length batch, tensors packed [N = total rows, H, D].
swa_status_t prefill_impl(const void *q, const void *k, const void *v, void *out, int B, int N,
                          int Hq, int Hkv, int D, int W, int window_mode, float scale,
                          const swa::RopeTable *rope, const int32_t *cu_seqlens, cudaStream_t s,
                          int sinks = 0) {
    if (!q || !k || !v || !out) return SWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(out)) return SWA_ERR_INVALID_ARG;
    if (B < 1 || N < 1 || W < 1 || bad_scale(scale)) return SWA_ERR_INVALID_ARG;
    if (window_mode != SWA_WINDOW_EXCL_LEFT && window_mode != SWA_WINDOW_INCL_LEFT)
        return SWA_ERR_INVALID_ARG;
    if (swa_status_t e = check_heads(Hq, Hkv, D)) return e;
    long long Weff = (long long)W + (window_mode == SWA_WINDOW_INCL_LEFT ? 1 : 0);
    if (Weff > N) Weff = N;                       // the window never reaches before position 0
    const int G = Hq / Hkv;
    if (cu_seqlens && (B > swa::kMaxVarlenSeqs || (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)))
        return B > swa::kMaxVarlenSeqs ? SWA_ERR_UNSUPPORTED : SWA_ERR_INVALID_ARG;
    const long long nqb = (N + 127) / 128;
    // varlen: an upper bound (the kernel counts the real units from cu_seqlens)
    const long long units = cu_seqlens ? (long long)Hkv * ((G + 1) / 2) * (nqb + B)
                                       : (long long)B * Hkv * ((G + 1) / 2) * nqb;
    if (units > 0x7fffffffll) return SWA_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;

    const int mb = cu_seqlens ? 1 : B;              // packed tensors have one batch row
    CUtensorMap mq, mk, mv;
    if (swa_status_t e = make_operand_map(&mq, q, D, Hq, N, mb)) return e;
    if (swa_status_t e = make_operand_map(&mk, k, D, Hkv, N, mb)) return e;
    if (swa_status_t e = make_operand_map(&mv, v, D, Hkv, N, mb)) return e;

    swa::PrefillParams p{};
    swa::prefill_units(p, B, N, Hq, Hkv, (int)Weff, cu_seqlens != nullptr, false, dev->sms);
    p.scale_log2 = scale * kLog2e;
    p.start_pos = nullptr;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    p.rope = rope ? 1 : 0;
    if (rope) p.rope_freq = *rope;
    p.cu_seqlens = cu_seqlens;
    p.sinks = sinks;
    return D == 128 ? launch_prefill<128>(mq, mk, mv, mk, mv, mk, mv, p, dev->sms, s)
                    : launch_prefill<64>(mq, mk, mv, mk, mv, mk, mv, p, dev->sms, s);
}

// cu_seqlens non-null: variable-length batch; q/k/v/out packed [C = total rows,
// H, D], sequence b is rows cu[b]..cu[b+1]-1 (any length; one longer than W
// leaves its last W positions in the buffer).
// k_sink / v_sink, S > 0: S-slot sink buffers [B, S, Hkv, D] (fixed-length only).
swa_status_t prefill_chunk_impl(const void *q, const void *k, const void *v, void *k_cache,
                                void *v_cache, const int32_t *start_pos, void *out, int B, int C,
                                int Hq, int Hkv, int D, int W, float scale,
                                const swa::RopeTable *rope, const int32_t *cu_seqlens,
                                cudaStream_t s, void *k_sink = nullptr, void *v_sink = nullptr,
                                int S = 0) {
    if (!q || !k || !v || !k_cache || !v_cache || !start_pos || !out) return SWA_ERR_INVALID_ARG;
    if (S < 0 || (S > 0 && (!k_sink || !v_sink || !aligned16(k_sink) || !aligned16(v_sink) || cu_seqlens)))
        return SWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(k_cache) ||
        !aligned16(v_cache) || !aligned16(out) || (reinterpret_cast<uintptr_t>(start_pos) & 3u))
        return SWA_ERR_INVALID_ARG;
    if (B < 1 || C < 1 || W < 1 || bad_scale(scale)) return SWA_ERR_INVALID_ARG;
    if (!cu_seqlens && C > W) return SWA_ERR_INVALID_ARG;
    if (cu_seqlens && (reinterpret_cast<uintptr_t>(cu_seqlens) & 3u)) return SWA_ERR_INVALID_ARG;
    if (cu_seqlens && B > swa::kMaxVarlenSeqs) return SWA_ERR_UNSUPPORTED;
    if (swa_status_t e = check_heads(Hq, Hkv, D)) return e;
    const int G = Hq / Hkv;
    const long long nqb = (C + 127) / 128;
    const long long units = cu_seqlens ? (long long)Hkv * ((G + 1) / 2) * (nqb + B)
                                       : (long long)B * Hkv * ((G + 1) / 2) * nqb;
    if (units > 0x7fffffffll) return SWA_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;

    const int mb = cu_seqlens ? 1 : B;
    CUtensorMap mq, mk, mv, mkc, mvc;
    if (swa_status_t e = make_operand_map(&mq, q, D, Hq, C, mb)) return e;
    if (swa_status_t e = make_operand_map(&mk, k, D, Hkv, C, mb)) return e;
    if (swa_status_t e = make_operand_map(&mv, v, D, Hkv, C, mb)) return e;
    if (swa_status_t e = make_operand_map(&mkc, k_cache, D, Hkv, W, B)) return e;
    if (swa_status_t e = make_operand_map(&mvc, v_cache, D, Hkv, W, B)) return e;

    swa::PrefillParams p{};
    swa::prefill_units(p, B, C, Hq, Hkv, W, cu_seqlens != nullptr, true, dev->sms);
    p.scale_log2 = scale * kLog2e;
    p.start_pos = start_pos;
    p.out = static_cast<__nv_bfloat16 *>(out);
    p.out_v8 = (reinterpret_cast<uintptr_t>(out) & 31u) == 0;
    p.rope = rope ? 1 : 0;
    if (rope) p.rope_freq = *rope;
    p.cu_seqlens = cu_seqlens;
    CUtensorMap mks = mkc, mvs = mvc;
    if (S > 0) {
        if (swa_status_t e = make_operand_map(&mks, k_sink, D, Hkv, S, B)) return e;
        if (swa_status_t e = make_operand_map(&mvs, v_sink, D, Hkv, S, B)) return e;
    }
    p.sink_buf = S;
    if (cu_seqlens) {
        // length-1 sequences (decode tokens) go to the decode kernel, which
        // reads their windows at memory speed instead of as 128-row tiles
        swa_status_t ed = SWA_OK;
        int rep = 1;
        const int gt = decode_group(Hq, Hkv, &rep);
        const bool fits = (long long)Hkv * rep <= 65535;
        const bool dec = fits && (D == 128 ? launch_decode_packed_d<128>(gt, rep, &ed, q, k, v, k_cache, v_cache,
                                                                         start_pos, cu_seqlens, out, B, C, Hkv * rep,
                                                                         W, scale, s)
                                           : launch_decode_packed_d<64>(gt, rep, &ed, q, k, v, k_cache, v_cache,
                                                                        start_pos, cu_seqlens, out, B, C, Hkv * rep,
                                                                        W, scale, s));
        if (ed) return ed;
        p.skip_len1 = dec ? 1 : 0;
    }
    swa_status_t e = D == 128 ? launch_prefill<128>(mq, mk, mv, mkc, mvc, mks, mvs, p, dev->sms, s)
                              : launch_prefill<64>(mq, mk, mv, mkc, mvc, mks, mvs, p, dev->sms, s);
    if (e) return e;
    // attend first, then write the chunk (its keys already rotated) into the buffer
    if (!cu_seqlens)     // positions below S also go to the sink buffer
        return launch_append(k, v, k_cache, v_cache, start_pos, B, C, Hkv, D, W, dev->sms, nullptr, s,
                             k_sink, v_sink, S);
    const int row_vec = Hkv * D * 2 / 16;
    long long blocks = ((long long)C * row_vec + 255) / 256;
    if (blocks > (long long)dev->sms * 8) blocks = (long long)dev->sms * 8;
    swa::swa_append_varlen_kernel<<<(int)blocks, 256, 0, s>>>(
        static_cast<const uint4 *>(k), static_cast<const uint4 *>(v), static_cast<uint4 *>(k_cache),
        static_cast<uint4 *>(v_cache), start_pos, cu_seqlens, B, C, W, row_vec);
    SWA_CUDA_TRY(cudaGetLastError());
    return SWA_OK;
}

swa_status_t append_impl(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                         const int32_t *pos, int B, int T, int Hkv, int D, int W,
                         const swa::RopeTable *rope, cudaStream_t s) {
    if (!k_new || !v_new || !k_cache || !v_cache || !pos) return SWA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(pos) & 3u))
        return SWA_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || W < 1 || T > W || Hkv < 1) return SWA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;
    return launch_append(k_new, v_new, k_cache, v_cache, pos, B, T, Hkv, D, W, dev->sms, rope, s);
}

size_t decode_workspace_bytes(int B, int Hq, int Hkv, int D, int W) {
    if (B < 1 || W < 1 || check_heads(Hq, Hkv, D) != SWA_OK) return 0;
    int rep = 1;
    decode_group(Hq, Hkv, &rep);
    if ((long long)Hkv * rep > 65535) return 0;
    const size_t nsm = (size_t)decode_nsplit_max(B, Hkv * rep, W);
    const size_t rows = (size_t)B * Hq * nsm;        // (b, kv head, split, head in group)
    const size_t o_bytes = (rows * D * 4 + 255) & ~size_t(255);
    return o_bytes + rows * 8;
}

swa_status_t decode_checks(const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *pos, const void *out, int B, int Hq, int Hkv, int D,
                           int W, float scale) {
    if (!q || !k_cache || !v_cache || !pos || !out) return SWA_ERR_INVALID_ARG;
    if (!aligned16(q) || !aligned16(k_cache) || !aligned16(v_cache) || !aligned16(out) ||
        (reinterpret_cast<uintptr_t>(pos) & 3u))
        return SWA_ERR_INVALID_ARG;
    if (B < 1 || W < 1 || bad_scale(scale)) return SWA_ERR_INVALID_ARG;
    if (swa_status_t e = check_heads(Hq, Hkv, D)) return e;
    int rep = 1;
    decode_group(Hq, Hkv, &rep);
    if (B > 65535 || (long long)Hkv * rep > 65535) return SWA_ERR_UNSUPPORTED;
    return SWA_OK;
}

swa_status_t decode_launch(const void *q, const void *k_cache, const void *v_cache,
                           const int32_t *pos, void *out, int B, int Hq, int Hkv, int D, int W,
                           float scale, void *workspace, const swa::RopeTable *rope, cudaStream_t s) {
    int rep = 1;
    const int G = decode_group(Hq, Hkv, &rep);
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;
    return D == 128 ? launch_decode_d<128>(G, rep, q, k_cache, v_cache, pos, out, B, Hkv * rep, W, scale, workspace,
                                           rope, s)
                    : launch_decode_d<64>(G, rep, q, k_cache, v_cache, pos, out, B, Hkv * rep, W, scale, workspace,
                                          rope, s);
}

swa_status_t decode_impl(const void *q, const void *k_cache, const void *v_cache,
                         const int32_t *pos, void *out, int B, int Hq, int Hkv, int D, int W,
                         float scale, void *workspace, size_t workspace_bytes,
                         const swa::RopeTable *rope, cudaStream_t s) {
    if (swa_status_t e = decode_checks(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale)) return e;
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, D, W);
    int rep = 1;
    decode_group(Hq, Hkv, &rep);
    if (decode_nsplit_max(B, Hkv * rep, W) > 1) {
        if (!workspace || workspace_bytes < need) return SWA_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SWA_ERR_INVALID_ARG;
    }
    return decode_launch(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale, workspace, rope, s);
}

}  // namespace

extern "C" {

swa_status_t swa_prefill(const void *q, const void *k, const void *v, void *out, int B, int N,
                         int Hq, int Hkv, int D, int W, int window_mode, float scale,
                         swa_stream_t stream) {
    return prefill_impl(q, k, v, out, B, N, Hq, Hkv, D, W, window_mode, scale, nullptr, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_prefill_chunk(const void *q, const void *k, const void *v, void *k_cache,
                               void *v_cache, const int32_t *start_pos, void *out, int B, int C,
                               int Hq, int Hkv, int D, int W, float scale, swa_stream_t stream) {
    return prefill_chunk_impl(q, k, v, k_cache, v_cache, start_pos, out, B, C, Hq, Hkv, D, W, scale,
                              nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_cache_append(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                              const int32_t *pos, int B, int T, int Hkv, int D, int W,
                              swa_stream_t stream) {
    return append_impl(k_new, v_new, k_cache, v_cache, pos, B, T, Hkv, D, W, nullptr,
                       reinterpret_cast<cudaStream_t>(stream));
}

size_t swa_decode_workspace_size(int B, int Hq, int Hkv, int D, int W) {
    return decode_workspace_bytes(B, Hq, Hkv, D, W);
}

swa_status_t swa_decode(const void *q, const void *k_cache, const void *v_cache,
                        const int32_t *pos, void *out, int B, int Hq, int Hkv, int D, int W,
                        float scale, void *workspace, size_t workspace_bytes,
                        swa_stream_t stream) {
    return decode_impl(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale, workspace,
                       workspace_bytes, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_decode_noalloc(const void *q, const void *k_cache, const void *v_cache,
                                const int32_t *pos, void *out, int B, int Hq, int Hkv, int D,
                                int W, float scale, swa_stream_t stream) {
    if (swa_status_t e = decode_checks(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale)) return e;
    if (decode_workspace_bytes(B, Hq, Hkv, D, W) > kNoallocScratchBytes) return SWA_ERR_UNSUPPORTED;
    void *scratch = nullptr;
    if (swa_status_t e = noalloc_scratch(&scratch)) return e;
    return decode_launch(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale, scratch, nullptr,
                         reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_rope(void *x, const int32_t *pos, int B, int T, int H, int D, float theta,
                      swa_stream_t stream) {
    if (!x || !pos || !aligned16(x) || (reinterpret_cast<uintptr_t>(pos) & 3u)) return SWA_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || H < 1 || bad_theta(theta)) return SWA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;
    const swa::RopeTable tab = make_rope_table(theta, D);
    const int row_vec = H * D / 8, head_vec = D / 8;
    const long long total = (long long)B * T * row_vec;
    long long blocks = (total + 255) / 256;
    if (blocks > (long long)dev->sms * 16) blocks = (long long)dev->sms * 16;
    swa::swa_rope_kernel<<<(int)blocks, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(
        static_cast<uint4 *>(x), pos, B, T, row_vec, head_vec, tab);
    SWA_CUDA_TRY(cudaGetLastError());
    return SWA_OK;
}

swa_status_t swa_cache_append_rope(const void *k_new, const void *v_new, void *k_cache,
                                   void *v_cache, const int32_t *pos, int B, int T, int Hkv,
                                   int D, int W, float theta, swa_stream_t stream) {
    if (bad_theta(theta)) return SWA_ERR_INVALID_ARG;
    const swa::RopeTable tab = make_rope_table(theta, D);
    return append_impl(k_new, v_new, k_cache, v_cache, pos, B, T, Hkv, D, W, &tab,
                       reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_prefill_rope(const void *q, const void *k, const void *v, void *out, int B, int N,
                              int Hq, int Hkv, int D, int W, int window_mode, float scale,
                              float theta, swa_stream_t stream) {
    if (bad_theta(theta)) return SWA_ERR_INVALID_ARG;
    const swa::RopeTable tab = make_rope_table(theta, D);
    return prefill_impl(q, k, v, out, B, N, Hq, Hkv, D, W, window_mode, scale, &tab, nullptr,
                        reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_prefill_chunk_rope(const void *q, const void *k, const void *v, void *k_cache,
                                    void *v_cache, const int32_t *start_pos, void *out, int B,
                                    int C, int Hq, int Hkv, int D, int W, float scale, float theta,
                                    swa_stream_t stream) {
    if (bad_theta(theta)) return SWA_ERR_INVALID_ARG;
    const swa::RopeTable tab = make_rope_table(theta, D);
    return prefill_chunk_impl(q, k, v, k_cache, v_cache, start_pos, out, B, C, Hq, Hkv, D, W, scale,
                              &tab, nullptr, reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_decode_rope(const void *q, const void *k_cache, const void *v_cache,
                             const int32_t *pos, void *out, int B, int Hq, int Hkv, int D, int W,
                             float scale, float theta, void *workspace, size_t workspace_bytes,
                             swa_stream_t stream) {
    if (bad_theta(theta)) return SWA_ERR_INVALID_ARG;
    const swa::RopeTable tab = make_rope_table(theta, D);
    return decode_impl(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale, workspace,
                       workspace_bytes, &tab, reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_prefill_varlen(const void *q, const void *k, const void *v, void *out,
                                const int32_t *cu_seqlens, int B, int total, int Hq, int Hkv, int D,
                                int W, int window_mode, float scale, swa_stream_t stream) {
    if (!cu_seqlens) return SWA_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, out, B, total, Hq, Hkv, D, W, window_mode, scale, nullptr, cu_seqlens,
                        reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_prefill_chunk_varlen(const void *q, const void *k, const void *v, void *k_cache,
                                      void *v_cache, const int32_t *start_pos,
                                      const int32_t *cu_seqlens, void *out, int B, int total,
                                      int Hq, int Hkv, int D, int W, float scale,
                                      swa_stream_t stream) {
    if (!cu_seqlens) return SWA_ERR_INVALID_ARG;
    return prefill_chunk_impl(q, k, v, k_cache, v_cache, start_pos, out, B, total, Hq, Hkv, D, W, scale,
                              nullptr, cu_seqlens, reinterpret_cast<cudaStream_t>(stream));
}

swa_status_t swa_prefill_sinks(const void *q, const void *k, const void *v, void *out, int B, int N,
                               int Hq, int Hkv, int D, int W, int S, float scale, swa_stream_t stream) {
    if (S < 0) return SWA_ERR_INVALID_ARG;
    return prefill_impl(q, k, v, out, B, N, Hq, Hkv, D, W, SWA_WINDOW_EXCL_LEFT, scale, nullptr, nullptr,
                        reinterpret_cast<cudaStream_t>(stream), S);
}

swa_status_t swa_prefill_chunk_sinks(const void *q, const void *k, const void *v, void *k_cache,
                                     void *v_cache, void *k_sink, void *v_sink, const int32_t *start_pos,
                                     void *out, int B, int C, int Hq, int Hkv, int D, int W, int S,
                                     float scale, swa_stream_t stream) {
    return prefill_chunk_impl(q, k, v, k_cache, v_cache, start_pos, out, B, C, Hq, Hkv, D, W, scale,
                              nullptr, nullptr, reinterpret_cast<cudaStream_t>(stream), k_sink, v_sink, S);
}

swa_status_t swa_cache_append_sinks(const void *k_new, const void *v_new, void *k_cache, void *v_cache,
                                    void *k_sink, void *v_sink, const int32_t *pos, int B, int T,
                                    int Hkv, int D, int W, int S, swa_stream_t stream) {
    if (S < 0 || (S > 0 && (!k_sink || !v_sink || !aligned16(k_sink) || !aligned16(v_sink))))
        return SWA_ERR_INVALID_ARG;
    if (!k_new || !v_new || !k_cache || !v_cache || !pos) return SWA_ERR_INVALID_ARG;
    if (!aligned16(k_new) || !aligned16(v_new) || !aligned16(k_cache) || !aligned16(v_cache) ||
        (reinterpret_cast<uintptr_t>(pos) & 3u))
        return SWA_ERR_INVALID_ARG;
    if (B < 1 || T < 1 || W < 1 || T > W || Hkv < 1) return SWA_ERR_INVALID_ARG;
    if (D != 64 && D != 128) return SWA_ERR_UNSUPPORTED;
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;
    return launch_append(k_new, v_new, k_cache, v_cache, pos, B, T, Hkv, D, W, dev->sms, nullptr,
                         reinterpret_cast<cudaStream_t>(stream), k_sink, v_sink, S);
}

swa_status_t swa_decode_sinks(const void *q, const void *k_cache, const void *v_cache,
                              const void *k_sink, const void *v_sink, const int32_t *pos, void *out,
                              int B, int Hq, int Hkv, int D, int W, int S, float scale,
                              void *workspace, size_t workspace_bytes, swa_stream_t stream) {
    if (S < 0 || (S > 0 && (!k_sink || !v_sink || !aligned16(k_sink) || !aligned16(v_sink))))
        return SWA_ERR_INVALID_ARG;
    if (swa_status_t e = decode_checks(q, k_cache, v_cache, pos, out, B, Hq, Hkv, D, W, scale)) return e;
    if ((long long)W + S > 0x7fffffffll) return SWA_ERR_UNSUPPORTED;
    const size_t need = decode_workspace_bytes(B, Hq, Hkv, D, W + S);
    int rep = 1;
    const int G = decode_group(Hq, Hkv, &rep);
    if (decode_nsplit_max(B, Hkv * rep, W + S) > 1) {
        if (!workspace || workspace_bytes < need) return SWA_ERR_INVALID_ARG;
        if (reinterpret_cast<uintptr_t>(workspace) & 255u) return SWA_ERR_INVALID_ARG;
    }
    DeviceInfo *dev = nullptr;
    if (swa_status_t e = device_info(&dev)) return e;
    cudaStream_t s = reinterpret_cast<cudaStream_t>(stream);
    return D == 128 ? launch_decode_d<128>(G, rep, q, k_cache, v_cache, pos, out, B, Hkv * rep, W, scale, workspace,
                                           nullptr, s, k_sink, v_sink, S)
                    : launch_decode_d<64>(G, rep, q, k_cache, v_cache, pos, out, B, Hkv * rep, W, scale, workspace,
                                          nullptr, s, k_sink, v_sink, S);
}

swa_status_t swa_get_device_status(swa_stream_t stream) {
    SWA_CUDA_TRY(cudaStreamSynchronize(reinterpret_cast<cudaStream_t>(stream)));
    int v = 0;
    SWA_CUDA_TRY(cudaMemcpyFromSymbol(&v, swa::g_status, sizeof(int)));
    const int zero = 0;
    SWA_CUDA_TRY(cudaMemcpyToSymbol(swa::g_status, &zero, sizeof(int)));
    return static_cast<swa_status_t>(v);
}

swa_status_t swa_set_wait_limit_ns(unsigned long long limit_ns) {
    SWA_CUDA_TRY(cudaMemcpyToSymbol(swa::g_wait_limit_ns, &limit_ns, sizeof(limit_ns)));
    return SWA_OK;
}

swa_status_t swa_selftest_wait_timeout(swa_stream_t stream) {
    swa_selftest_wait_kernel<<<1, 32, 0, reinterpret_cast<cudaStream_t>(stream)>>>();
    SWA_CUDA_TRY(cudaGetLastError());
    return SWA_OK;
}

swa_status_t swa_selftest_exp2(const float *x, float *y, int n, swa_stream_t stream) {
    if (!x || !y || n < 1) return SWA_ERR_INVALID_ARG;
    const int pairs = (n + 1) / 2;
    swa_selftest_exp2_kernel<<<(pairs + 255) / 256, 256, 0, reinterpret_cast<cudaStream_t>(stream)>>>(x, y, n);
    SWA_CUDA_TRY(cudaGetLastError());
    return SWA_OK;
}

const char *swa_status_string(swa_status_t status) {
    switch (status) {
        case SWA_OK: return "SWA_OK";
        case SWA_ERR_INVALID_ARG: return "SWA_ERR_INVALID_ARG";
        case SWA_ERR_UNSUPPORTED: return "SWA_ERR_UNSUPPORTED";
        case SWA_ERR_CUDA: return "SWA_ERR_CUDA";
        case SWA_ERR_TIMEOUT: return "SWA_ERR_TIMEOUT";
        default: return "SWA_ERR_UNKNOWN";
    }
}

int swa_last_cuda_error(void) { return t_last_cuda_error; }

}  // extern "C"
