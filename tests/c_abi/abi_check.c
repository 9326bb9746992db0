/* Calls libfg8.so through its C header only (no Python, no CUDA headers) and
 * checks the host-side contract: argument validation, no-op sizes and the
 * helpers.  Needs no GPU; prints one line per failed check and returns the
 * number of failures. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fg8.h"

static int failures = 0;

static void expect(const char* what, long got, long want) {
    if (got != want) {
        printf("FAIL %s: got %ld, want %ld\n", what, got, want);
        ++failures;
    }
}

int main(void) {
    /* 16-byte aligned, never dereferenced: every call below fails its checks first. */
    void* fake = (void*)(uintptr_t)0x100000;
    const float* ff = (const float*)fake;
    expect("K not a multiple of 128", fg_fp8_gemm_nt(fake, ff, fake, ff, fake, 64, 128, 130, 0), FG_ERR_UNSUPPORTED);
    expect("N not a multiple of 16", fg_fp8_gemm_nt(fake, ff, fake, ff, fake, 64, 120, 256, 0), FG_ERR_UNSUPPORTED);
    expect("negative M", fg_fp8_gemm_nt(fake, ff, fake, ff, fake, -1, 128, 256, 0), FG_ERR_INVALID_ARG);
    expect("null A", fg_fp8_gemm_nt(NULL, ff, fake, ff, fake, 64, 128, 256, 0), FG_ERR_INVALID_ARG);
    expect("misaligned A", fg_fp8_gemm_nt((char*)fake + 8, ff, fake, ff, fake, 64, 128, 256, 0), FG_ERR_ALIGNMENT);
    expect("empty GEMM", fg_fp8_gemm_nt(NULL, NULL, NULL, NULL, NULL, 0, 128, 256, 0), FG_OK);
    expect("contiguous M_tot % 128", fg_m_grouped_fp8_gemm_nt_contiguous(fake, ff, fake, ff, fake, (const int*)fake,
                                                                         200, 128, 256, 2, 0), FG_ERR_INVALID_ARG);
    expect("masked no groups", fg_m_grouped_fp8_gemm_nt_masked(NULL, NULL, NULL, NULL, NULL, NULL, 0, 256, 128,
                                                                256, 0, 0), FG_OK);
    expect("no-alloc M above its limit", fg_fp8_gemm_nt_small_m_no_alloc(fake, ff, fake, ff, fake,
                                                                          FG_NO_ALLOC_MAX_M + 1, 128, 256, 0),
           FG_ERR_UNSUPPORTED);
    expect("quantiser K % 128", fg_quantize_fp8_activations(fake, 0, fake, (float*)fake, 4, 100, 0),
           FG_ERR_UNSUPPORTED);
    expect("alignment helper", (long)fg_get_tma_aligned_size(5, 4), 8);
    expect("alignment helper bytes", (long)fg_get_tma_aligned_size(17, 1), 32);
    expect("contiguous alignment", fg_get_m_alignment_for_contiguous_layout(), 128);
    expect("set_num_sms(0)", fg_set_num_sms(0), FG_ERR_INVALID_ARG);
    expect("wait limit too small", fg_set_wait_limit_ns(10), FG_ERR_INVALID_ARG);
    expect("status string", strcmp(fg_status_string(FG_ERR_TIMEOUT), "FG_ERR_TIMEOUT"), 0);
    expect("version prefix", strncmp(fg_version(), "fg8 ", 4), 0);
    return failures;
}
