/* A plain C99 caller of the library: it includes the public header, links against libcobs.so
 * and exercises the host-side part of the ABI (sizing, version, status strings, argument
 * validation), none of which touches a GPU. Exit status 0 on success, else the failing check. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "cobs.h"

#define CHECK(cond)                                                     \
    do {                                                                \
        if (!(cond)) {                                                  \
            fprintf(stderr, "check failed: %s (line %d)\n", #cond, __LINE__); \
            return __LINE__;                                            \
        }                                                               \
    } while (0)

int main(void) {
    cobs_params p;
    memset(&p, 0, sizeof p);
    p.B = 8; p.Hq = 32; p.Hkv = 8; p.d = 128; p.T = 32768;
    p.block = 64; p.cmp_block = 32; p.cmp_stride = 16; p.topk = 16; p.window = 512;
    p.alpha = 1.0f; p.dtype = COBS_BF16; p.variance = COBS_VAR_CHANNEL; p.rank = 0;
    p.sub = 0; p.basis = NULL;

    CHECK(cobs_version() == 102);
    CHECK(strcmp(cobs_status_string(COBS_OK), "ok") == 0);
    /* 64 units x 16 groups of 32 blocks x (means + variances) */
    CHECK(cobs_summaries_elems(&p) == (size_t)64 * 16 * 2 * 128 * 32);
    CHECK(cobs_workspace_bytes(&p, COBS_WS_SELECT) > 0);
    CHECK(cobs_workspace_bytes(&p, COBS_WS_DECODE) > 0);

    /* the query-subspace form: 32 (d + r s + r) floats per group; sizing needs no basis */
    p.variance = COBS_VAR_SUBSPACE; p.rank = 4; p.sub = 84;
    CHECK(cobs_summaries_elems(&p) == (size_t)64 * 16 * 32 * (128 + 4 * 84 + 4));

    /* invalid arguments are rejected on the host, before anything is launched */
    void* fake = (void*)(uintptr_t)256;
    p.variance = COBS_VAR_CHANNEL;
    p.d = 96;
    CHECK(cobs_build_summaries(&p, fake, fake, NULL, NULL, 0, (float*)fake, fake, fake, NULL) == COBS_ERR_UNSUPPORTED);
    CHECK(strlen(cobs_last_error()) > 0);
    p.d = 128;
    CHECK(cobs_select(&p, NULL, (const float*)fake, 0, (int32_t*)fake, fake, 1u << 20, NULL) == COBS_ERR_INVALID_ARG);
    p.variance = COBS_VAR_SUBSPACE; p.sub = 84; p.basis = NULL;
    CHECK(cobs_select(&p, fake, (const float*)fake, 0, (int32_t*)fake, fake, (size_t)1 << 30, NULL) ==
          COBS_ERR_INVALID_ARG);
    printf("ok\n");
    return 0;
}
