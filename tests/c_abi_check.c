/* A plain C99 caller of include/fa.h: the header must compile as C and every
 * entry point must link and reject bad arguments before touching a GPU.
 * Built and run by tests/test_c_abi.py (gcc, no CUDA headers needed).
 * Exit status 0 when every check holds; otherwise the number of the first
 * failed check. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa.h"

#define CHECK(n, cond)                                   \
    do {                                                 \
        if (!(cond)) {                                   \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                    \
        }                                                \
    } while (0)

int main(void) {
    /* a 16-byte aligned address that is never dereferenced: every call below
     * fails its argument checks first */
    void* p = (void*)(uintptr_t)0x10000;
    void* odd = (void*)(uintptr_t)0x10008;
    fa_shape good = {1, 4, 2, 128, 128, 0.125f, 1};
    fa_shape bad_d = good;
    fa_shape bad_heads = good;
    fa_kv_shape kv = {1, 4, 2, 3, 700, 128, 0.125f, 1};
    fa_kv_shape kv_bad = kv;
    bad_d.D = 96;
    bad_heads.Hkv = 3;
    kv_bad.Nq = 701;

    CHECK(1, fa_fwd(NULL, p, p, p, p, (float*)p, NULL) == FA_ERR_INVALID_ARG);
    CHECK(2, fa_fwd(&bad_d, p, p, p, p, (float*)p, NULL) == FA_ERR_UNSUPPORTED);
    CHECK(3, fa_fwd(&bad_heads, p, p, p, p, (float*)p, NULL) == FA_ERR_INVALID_ARG);
    CHECK(4, fa_fwd(&good, odd, p, p, p, (float*)p, NULL) == FA_ERR_INVALID_ARG);
    CHECK(5, fa_fwd_fp8(&bad_d, p, p, p, 1.0f, 1.0f, 1.0f, p, (float*)p, NULL) == FA_ERR_UNSUPPORTED);
    CHECK(6, fa_fwd_fp8(&good, p, p, p, 0.0f, 1.0f, 1.0f, p, (float*)p, NULL) == FA_ERR_INVALID_ARG);
    CHECK(7, fa_bwd_workspace_bytes(&good) > 0 && fa_bwd_workspace_bytes(&bad_heads) == 0);
    CHECK(8, fa_bwd(&good, p, p, p, p, p, (float*)p, p, p, p, p, 0, NULL) == FA_ERR_INVALID_ARG);
    CHECK(9, fa_bwd_noalloc(&bad_d, p, p, p, p, p, (float*)p, p, p, p, NULL) == FA_ERR_UNSUPPORTED);
    CHECK(10, fa_decode_workspace_bytes(&kv) > 0 && fa_decode_workspace_bytes(&kv_bad) == 0);
    CHECK(11, fa_decode(&kv_bad, p, p, p, p, (float*)p, p, 1u << 30, NULL) == FA_ERR_INVALID_ARG);
    CHECK(12, fa_lse_merge(-1, 128, p, (float*)p, (float*)p, (float*)p, NULL, 0, NULL) == FA_ERR_INVALID_ARG);
    CHECK(13, fa_lse_merge(0, 128, NULL, NULL, NULL, NULL, NULL, 0, NULL) == FA_OK);
    CHECK(14, fa_accumulate(12, p, (float*)p, NULL, 0, NULL) == FA_ERR_INVALID_ARG);
    CHECK(15, fa_accumulate(0, NULL, NULL, NULL, 1, NULL) == FA_OK);
    CHECK(16, strcmp(fa_status_str(FA_OK), "ok") == 0 && fa_status_str((fa_status)99) != NULL);
    CHECK(17, fa_debug_timeout_sites() == 0u);
    CHECK(18, FA_PROFILE_KINDS == 14 && FA_NOALLOC_SCRATCH_BYTES == (32u << 20));
    CHECK(19, fa_selftest_wait_timeout(3, 3, NULL) == FA_ERR_INVALID_ARG);
    printf("c abi ok\n");
    return 0;
}
