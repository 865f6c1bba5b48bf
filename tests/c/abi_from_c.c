/* A plain C99 caller of libattnqat: the header compiles as C, the library
 * links, and the host-side checks answer without touching a GPU (every call
 * below fails validation before any device work).  Prints one line per
 * check and exits non-zero on the first mismatch. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "attnqat.h"

static int fails = 0;

static void expect(const char *what, long long got, long long want)
{
    printf("%-48s %lld (want %lld)\n", what, got, want);
    if (got != want)
        fails++;
}

int main(void)
{
    /* 256-byte aligned, never dereferenced: validation fails first */
    void *fake = (void *)(uintptr_t)0x10000;
    float *ffake = (float *)fake;
    const size_t ws = attnqat_workspace_size(1, 6, 31200, 31200, 128, ATTNQAT_QUANT_ALL);
    expect("workspace bytes > 0 (H6 L31200 D128)", ws > 0, 1);
    expect("workspace for D = 96", (long long)attnqat_workspace_size(1, 1, 16, 16, 96, 0), 0);
    expect("causal needs Lq == Lk",
           (long long)attnqat_workspace_size(1, 1, 128, 256, 128, ATTNQAT_QUANT_ALL | ATTNQAT_CAUSAL), 0);
    expect("sparse workspace > dense workspace",
           attnqat_sparse_workspace_size(1, 6, 31200, 31200, 128, ATTNQAT_QUANT_ALL) > ws, 1);
    expect("fwd: null q", attnqat_fwd(NULL, fake, fake, 1, 1, 128, 128, 128, 0.125f, ATTNQAT_QUANT_ALL, fake,
                                      ffake, ffake, fake, (size_t)1 << 30, NULL), ATTNQAT_EINVAL);
    expect("fwd: workspace too small", attnqat_fwd(fake, fake, fake, 1, 1, 128, 128, 128, 0.125f,
                                                   ATTNQAT_QUANT_ALL, fake, ffake, ffake, fake, 16, NULL),
           ATTNQAT_ENOSPC);
    expect("bwd: sm_scale 0", attnqat_bwd(fake, fake, fake, ffake, ffake, fake, 1, 1, 128, 128, 128, 0.0f,
                                          ATTNQAT_QUANT_ALL, fake, fake, fake, fake, (size_t)1 << 30, NULL),
           ATTNQAT_EINVAL);
    expect("sparse fwd: null mask", attnqat_sparse_fwd(fake, fake, fake, 1, 1, 128, 128, 128, 0.125f,
                                                       ATTNQAT_QUANT_ALL, NULL, fake, ffake, ffake, fake,
                                                       (size_t)1 << 30, NULL), ATTNQAT_EINVAL);
    expect("select: topk 0", attnqat_vsa_select(fake, fake, 1, 1, 128, 128, 128, 0, (uint8_t *)fake, fake,
                                                (size_t)1 << 30, NULL), ATTNQAT_EINVAL);
    expect("quantize: cols 24", attnqat_quantize(fake, 1, 4, 24, 0, 24, 1, (uint8_t *)fake, (uint8_t *)fake,
                                                 NULL, NULL), ATTNQAT_EINVAL);
    expect("strerror(EINVAL) non-empty", strlen(attnqat_strerror(ATTNQAT_EINVAL)) > 0, 1);
    return fails ? 1 : 0;
}
