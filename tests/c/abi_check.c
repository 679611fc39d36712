/*
 * A plain C client of libswa.  It shows that include/swa.h is a C header
 * (it compiles as C11 and as C++ with every warning turned into an error) and
 * that calls from C reach the library: host-side argument checks answer with
 * status codes before anything touches a device, so this runs without a GPU.
 * Exit status 0 and "ok" on success.
 */
#include <stdio.h>
#include <string.h>

#include "swa.h"

#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "abi_check.c:%d: %s\n", __LINE__, #cond); \
            return 1;                                                 \
        }                                                             \
    } while (0)

int main(void) {
    /* aligned addresses that are never dereferenced: every call below fails
       its argument checks first */
    void *p = (void *)(uintptr_t)0x1000;
    const int32_t *ip = (const int32_t *)(uintptr_t)0x1000;
    size_t need;

    CHECK(swa_prefill(NULL, p, p, p, 1, 16, 4, 2, 128, 8, SWA_WINDOW_EXCL_LEFT, 0.1f, NULL) ==
          SWA_ERR_INVALID_ARG);
    CHECK(swa_prefill(p, p, p, (char *)p + 8, 1, 16, 4, 2, 128, 8, SWA_WINDOW_EXCL_LEFT, 0.1f, NULL) ==
          SWA_ERR_INVALID_ARG);                                   /* out not 16-byte aligned */
    CHECK(swa_prefill(p, p, p, p, 1, 16, 4, 2, 80, 8, SWA_WINDOW_EXCL_LEFT, 0.1f, NULL) ==
          SWA_ERR_UNSUPPORTED);                                   /* head dim outside {64, 128} */
    CHECK(swa_prefill(p, p, p, p, 1, 16, 3, 2, 128, 8, SWA_WINDOW_INCL_LEFT, 0.1f, NULL) ==
          SWA_ERR_INVALID_ARG);                                   /* Hq not a multiple of Hkv */
    CHECK(swa_prefill_chunk(p, p, p, p, p, ip, p, 1, 65, 4, 2, 128, 64, 0.1f, NULL) ==
          SWA_ERR_INVALID_ARG);                                   /* chunk longer than the window */
    CHECK(swa_cache_append(p, p, p, p, NULL, 1, 1, 2, 128, 64, NULL) == SWA_ERR_INVALID_ARG);
    CHECK(swa_prefill_sinks(p, p, p, p, 1, 16, 4, 2, 128, 8, -1, 0.1f, NULL) == SWA_ERR_INVALID_ARG);

    need = swa_decode_workspace_size(64, 32, 8, 128, 4096);
    CHECK(need > 0 && swa_decode_workspace_size(0, 32, 8, 128, 4096) == 0);
    CHECK(swa_decode(p, p, p, ip, p, 64, 32, 8, 128, 4096, 0.1f, p, need - 1, NULL) ==
          SWA_ERR_INVALID_ARG);                                   /* workspace one byte short */
    CHECK(need <= SWA_DECODE_NOALLOC_SCRATCH_BYTES);

    CHECK(strcmp(swa_status_string(SWA_OK), "SWA_OK") == 0);
    CHECK(strcmp(swa_status_string(SWA_ERR_TIMEOUT), "SWA_ERR_TIMEOUT") == 0);
    CHECK(strcmp(swa_status_string((swa_status_t)99), "SWA_ERR_UNKNOWN") == 0);
    printf("ok\n");
    return 0;
}
