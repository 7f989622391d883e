/* Uses include/fa.h from plain C99 and calls the library's host-side paths: argument
 * validation, status strings and the version (no device work, so it runs without a GPU). */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fa.h"

static int fails = 0;

static void expect(int got, int want, const char *what) {
    if (got != want) {
        printf("%s: got %d, want %d\n", what, got, want);
        ++fails;
    }
}

int main(void) {
    /* a 16-byte aligned non-null address that is never dereferenced */
    void *f = (void *)(uintptr_t)(1u << 20);
    const int32_t *cu = (const int32_t *)f;
    const float *lse = (const float *)f;

    expect(fa_fwd(NULL, f, f, f, NULL, 1, 1, 128, 64, 0.f, 0, FA_FP16, NULL), FA_ERR_NULL, "fa_fwd null q");
    expect(fa_fwd(f, f, f, f, NULL, 1, 1, 128, 96, 0.f, 0, FA_FP16, NULL), FA_ERR_HEADDIM, "fa_fwd D=96");
    expect(fa_fwd(f, f, f, f, NULL, 1, 1, 128, 64, 0.f, 0, (fa_dtype)7, NULL), FA_ERR_DTYPE, "fa_fwd dtype");
    expect(fa_varlen_fwd(NULL, NULL, NULL, NULL, 0, 0, 0, NULL, NULL, 4, 64, 0.f, 0, FA_BF16, NULL), FA_OK,
           "fa_varlen_fwd empty");
    expect(fa_varlen_fwd_padded(f, f, f, (const int64_t *)f, cu, 2, 8, 10, 5, f, NULL, 2, 64, 0.f, 0, FA_BF16,
                                NULL),
           FA_ERR_SHAPE, "fa_varlen_fwd_padded total > padded_rows");
    expect(fa_fwd_paged(f, f, f, cu, 3, 24, 10, f, NULL, 2, 4, 130, 128, 0.f, 0, FA_BF16, NULL), FA_ERR_SHAPE,
           "fa_fwd_paged page 24");
    expect(fa_bwd(f, f, f, f, f, lse, f, f, f, (float *)f, 1, 2, 128, 96, 0.f, 1, FA_BF16, NULL), FA_ERR_HEADDIM,
           "fa_bwd D=96");
    expect(fa_varlen_bwd(f, f, f, f, f, lse, cu, 3, 64, 0, f, f, f, (float *)f, 2, 64, 0.f, 1, FA_BF16, NULL), FA_OK,
           "fa_varlen_bwd empty");
    expect(fa_bwd_noalloc(f, f, f, f, f, lse, f, f, f, 1, 128, 131073, 128, 0.f, 1, FA_BF16, NULL), FA_ERR_SHAPE,
           "fa_bwd_noalloc oversize");
    expect(fa_unpad(NULL, NULL, 0, 10, 64, NULL, NULL), FA_OK, "fa_unpad empty");
    expect(fa_pad(f, (const int64_t *)f, 11, 10, 64, f, NULL), FA_ERR_SHAPE, "fa_pad nnz > rows");
    expect(fa_selftest_bounded_wait(0, NULL), FA_ERR_SHAPE, "fa_selftest_bounded_wait 0");
    if (strncmp(fa_status_string(FA_ERR_TIMEOUT), "FA_ERR_TIMEOUT", 14) != 0) {
        printf("status string: %s\n", fa_status_string(FA_ERR_TIMEOUT));
        ++fails;
    }
    if (!strstr(fa_version(), "sm_100a")) {
        printf("version: %s\n", fa_version());
        ++fails;
    }
    printf("%s\n", fails ? "FAIL" : "ok");
    return fails ? 1 : 0;
}
