/*
 * abi_check.c -- a plain C99 client of libomni, built and run by
 * tests/test_abi_c.py on the CPU.  It includes include/omni.h as C, links
 * the library and calls every entry point with arguments the host-side
 * checks reject, so no call reaches the GPU.  Exit status 0 means every
 * expectation held; each failure is printed.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "omni.h"

static int failures = 0;

#define EXPECT(cond)                                                        \
    do {                                                                    \
        if (!(cond)) {                                                      \
            fprintf(stderr, "abi_check.c:%d: expected %s\n", __LINE__, #cond); \
            ++failures;                                                     \
        }                                                                   \
    } while (0)

int main(void) {
    /* never dereferenced: every call below is refused before any launch */
    void *fake = (void *)(uintptr_t)(1u << 20);
    const omni_bf16 *fb = (const omni_bf16 *)fake;
    float *ff = (float *)fake;
    int32_t *fi = (int32_t *)fake;
    const int L = 4, d = 256, Nr = 4, Nc = 4, K = 2, B = 2;
    size_t ws;
    int st = 7;

    EXPECT(omni_version() == 1);
    EXPECT(strcmp(omni_status_string(OMNI_ERR_WORKSPACE), "OMNI_ERR_WORKSPACE") == 0);
    EXPECT(strcmp(omni_device_status_string(OMNI_DEV_WAIT_TIMEOUT), "OMNI_DEV_WAIT_TIMEOUT") == 0);

    ws = omni_workspace_size(L, d, Nr, Nc, K, B);
    EXPECT(ws > 0 && ws % 256 == 0);
    EXPECT(omni_workspace_size(0, d, Nr, Nc, K, B) == 0);
    EXPECT(omni_router_workspace_size(L, Nr, Nc, K) > 0);
    EXPECT(omni_schedule_workspace_size(L, K, Nr * Nc, B) > 0);
    EXPECT(omni_expert_workspace_size(L, d, K, Nr * Nc, B) > 0);
    EXPECT(omni_shared_mlp_workspace_size(L, d, 128) == 256 + 2 * (size_t)L * 128);
    EXPECT(omni_routed_bwd_workspace_size(L, d, Nr, Nc, K) == 256 + 2 * 256 + 256 + 8 * (size_t)(Nr + Nc) * 256);
    EXPECT(omni_routed_bwd_workspace_size(L, d, Nr, Nc, 0) == 0);

    /* null input */
    EXPECT(omni_router_topk(NULL, fb, fb, L, d, Nr, Nc, K, ff, ff, fi, ff, ff, 0, fake, ws, NULL) ==
           OMNI_ERR_INVALID_ARG);
    /* K > N */
    EXPECT(omni_routed_fwd(fb, fb, fb, fb, fb, L, d, Nr, Nc, 17, B, ff, NULL, NULL, 0, fake, ws,
                           NULL) == OMNI_ERR_INVALID_ARG);
    /* workspace too small */
    EXPECT(omni_routed_fwd(fb, fb, fb, fb, fb, L, d, Nr, Nc, K, B, ff, NULL, NULL, 0, fake, 256,
                           NULL) == OMNI_ERR_WORKSPACE);
    /* d off the expert stage's grid */
    EXPECT(omni_grouped_expert_fwd(fb, fb, fb, L, 264, K, Nr * Nc, B, fi, fi, ff, fi, fi, fi, ff,
                                   0, fake, ws, NULL) == OMNI_ERR_UNSUPPORTED);
    /* misaligned workspace */
    EXPECT(omni_schedule(fi, ff, L, K, Nr * Nc, B, fi, fi, ff, fi, fi, fi, fi, fi,
                         (char *)fake + 64, ws, NULL) == OMNI_ERR_INVALID_ARG);
    /* backward: flags must be 0 */
    EXPECT(omni_routed_bwd(fb, fb, fb, fb, fb, L, d, Nr, Nc, K, fi, ff, ff, ff, ff, ff, ff, ff, 1,
                           fake, 256, NULL) == OMNI_ERR_INVALID_ARG);
    /* backward: every gradient buffer is required */
    EXPECT(omni_routed_bwd(fb, fb, fb, fb, fb, L, d, Nr, Nc, K, fi, ff, ff, ff, ff, ff, ff, NULL, 0,
                           fake, 256, NULL) == OMNI_ERR_INVALID_ARG);
    /* backward: d off its 256 grid */
    EXPECT(omni_routed_bwd(fb, fb, fb, fb, fb, L, 384, Nr, Nc, K, fi, ff, ff, ff, ff, ff, ff, ff, 0,
                           fake, 256, NULL) == OMNI_ERR_UNSUPPORTED);
    /* backward: below the 256-byte minimum workspace, or a misaligned one */
    EXPECT(omni_routed_bwd(fb, fb, fb, fb, fb, L, d, Nr, Nc, K, fi, ff, ff, ff, ff, ff, ff, ff, 0,
                           fake, 128, NULL) == OMNI_ERR_WORKSPACE);
    EXPECT(omni_routed_bwd(fb, fb, fb, fb, fb, L, d, Nr, Nc, K, fi, ff, ff, ff, ff, ff, ff, ff, 0,
                           (char *)fake + 64, 4096, NULL) == OMNI_ERR_WORKSPACE);
    EXPECT(omni_routed_bwd_workspace_size(0, d, Nr, Nc, K) == 0);
    /* shared MLP: F off the 64 grid */
    EXPECT(omni_shared_mlp_fwd(fb, fb, fb, fb, L, d, 96, ff, 0, fake, 1u << 20, NULL) ==
           OMNI_ERR_UNSUPPORTED);
    /* allocation-free expert stage: above its token limit */
    EXPECT(omni_grouped_expert_fwd_noalloc(fb, fb, fb, 20000, d, 1, Nr * Nc, B, fi, fi, ff, fi, fi,
                                           fi, ff, 0, NULL) == OMNI_ERR_UNSUPPORTED);
    /* diagnostics need a workspace */
    EXPECT(omni_selftest_wait_timeout(NULL, 256, 10, NULL) == OMNI_ERR_INVALID_ARG);
    EXPECT(omni_get_device_status(NULL, 0, NULL, &st) == OMNI_ERR_INVALID_ARG);
    EXPECT(omni_noalloc_get_device_status(NULL, NULL) == OMNI_ERR_INVALID_ARG);

    if (failures == 0) printf("abi_check: all expectations held\n");
    return failures == 0 ? 0 : 1;
}
