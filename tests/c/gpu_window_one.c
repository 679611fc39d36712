/*
 * A plain C program driving the CUDA path through the C ABI: device buffers
 * from cudaMalloc, inputs copied in, swa_prefill / swa_cache_append /
 * swa_decode called from C.  Checked against a closed form that needs no
 * oracle: with W = 1 each query sees only its own position, so the softmax
 * weight is 1 and out[b,i,h,:] equals v[b,i,h/G,:] bit for bit; decode after
 * appending position p equals the appended value row.  Values are
 * +-(1 + m/128) * 2^e, exact in bf16 and far from zero.
 * Exit status 0 and "ok" on success.
 */
#include <stdint.h>
#include <stdio.h>
#include <stdlib.h>
#include <string.h>

#include <cuda_runtime.h>

#include "swa.h"

#define CHECK(cond)                                                          \
    do {                                                                     \
        if (!(cond)) {                                                       \
            fprintf(stderr, "gpu_window_one.c:%d: %s\n", __LINE__, #cond);   \
            return 1;                                                        \
        }                                                                    \
    } while (0)

static uint32_t lcg(uint32_t *s) {
    *s = *s * 1664525u + 1013904223u;
    return *s >> 8;
}

/* sign | exponent 126 or 127 | 7-bit mantissa */
static uint16_t draw(uint32_t *s) {
    uint32_t r = lcg(s);
    return (uint16_t)(((r & 1u) << 15) | ((126u + ((r >> 1) & 1u)) << 7) | ((r >> 2) & 127u));
}

int main(void) {
    enum { B = 2, N = 300, HQ = 8, HKV = 2, D = 128, G = HQ / HKV };
    const size_t nq = (size_t)B * N * HQ * D, nkv = (size_t)B * N * HKV * D;
    uint16_t *hq = malloc(nq * 2), *hk = malloc(nkv * 2), *hv = malloc(nkv * 2), *ho = malloc(nq * 2);
    void *dq, *dk, *dv, *dout, *kc, *vc, *ws, *dqd, *dod;
    int32_t *dpos;
    uint32_t seed = 12345u;
    size_t i, need;
    int b, t, h, p;
    CHECK(hq && hk && hv && ho);
    for (i = 0; i < nq; ++i) hq[i] = draw(&seed);
    for (i = 0; i < nkv; ++i) hk[i] = draw(&seed);
    for (i = 0; i < nkv; ++i) hv[i] = draw(&seed);
    CHECK(cudaMalloc(&dq, nq * 2) == cudaSuccess && cudaMalloc(&dk, nkv * 2) == cudaSuccess);
    CHECK(cudaMalloc(&dv, nkv * 2) == cudaSuccess && cudaMalloc(&dout, nq * 2) == cudaSuccess);
    CHECK(cudaMemcpy(dq, hq, nq * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(dk, hk, nkv * 2, cudaMemcpyHostToDevice) == cudaSuccess);
    CHECK(cudaMemcpy(dv, hv, nkv * 2, cudaMemcpyHostToDevice) == cudaSuccess);

    /* one-shot prefill, W = 1 */
    CHECK(swa_prefill(dq, dk, dv, dout, B, N, HQ, HKV, D, 1, SWA_WINDOW_EXCL_LEFT, 0.088f, NULL) == SWA_OK);
    CHECK(cudaMemcpy(ho, dout, nq * 2, cudaMemcpyDeviceToHost) == cudaSuccess);
    for (b = 0; b < B; ++b)
        for (t = 0; t < N; ++t)
            for (h = 0; h < HQ; ++h)
                CHECK(memcmp(ho + (((size_t)b * N + t) * HQ + h) * D,
                             hv + (((size_t)b * N + t) * HKV + h / G) * D, D * 2) == 0);

    /* decode through a one-slot rolling buffer: append position p, attend */
    CHECK(cudaMalloc(&kc, (size_t)B * HKV * D * 2) == cudaSuccess);
    CHECK(cudaMalloc(&vc, (size_t)B * HKV * D * 2) == cudaSuccess);
    CHECK(cudaMalloc(&dqd, (size_t)B * HQ * D * 2) == cudaSuccess);
    CHECK(cudaMalloc(&dod, (size_t)B * HQ * D * 2) == cudaSuccess);
    CHECK(cudaMalloc((void **)&dpos, B * sizeof(int32_t)) == cudaSuccess);
    need = swa_decode_workspace_size(B, HQ, HKV, D, 1);
    CHECK(need > 0 && cudaMalloc(&ws, need) == cudaSuccess);
    for (p = 0; p < 5; ++p) {
        int32_t pos[B];
        uint16_t kn[B * HKV * D], vn[B * HKV * D], qn[B * HQ * D], on[B * HQ * D];
        for (b = 0; b < B; ++b) pos[b] = 7 * p + b;
        for (i = 0; i < (size_t)B * HKV * D; ++i) { kn[i] = draw(&seed); vn[i] = draw(&seed); }
        for (i = 0; i < (size_t)B * HQ * D; ++i) qn[i] = draw(&seed);
        CHECK(cudaMemcpy(dpos, pos, sizeof(pos), cudaMemcpyHostToDevice) == cudaSuccess);
        CHECK(cudaMemcpy(dk, kn, sizeof(kn), cudaMemcpyHostToDevice) == cudaSuccess);
        CHECK(cudaMemcpy(dv, vn, sizeof(vn), cudaMemcpyHostToDevice) == cudaSuccess);
        CHECK(cudaMemcpy(dqd, qn, sizeof(qn), cudaMemcpyHostToDevice) == cudaSuccess);
        CHECK(swa_cache_append(dk, dv, kc, vc, dpos, B, 1, HKV, D, 1, NULL) == SWA_OK);
        CHECK(swa_decode(dqd, kc, vc, dpos, dod, B, HQ, HKV, D, 1, 0.088f, ws, need, NULL) == SWA_OK);
        CHECK(cudaMemcpy(on, dod, sizeof(on), cudaMemcpyDeviceToHost) == cudaSuccess);
        for (b = 0; b < B; ++b)
            for (h = 0; h < HQ; ++h)
                CHECK(memcmp(on + ((size_t)b * HQ + h) * D, vn + ((size_t)b * HKV + h / G) * D, D * 2) == 0);
    }
    CHECK(swa_get_device_status(NULL) == SWA_OK);
    printf("ok\n");
    return 0;
}
