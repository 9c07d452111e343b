/*
 * abi_from_c.c -- the C ABI of libsq.so used from plain C (C11, no CUDA
 * headers): the header compiles as C, every entry point links, and calls
 * whose arguments fail validation return the documented status without
 * touching a GPU. Prints "ok" and exits 0 on success.
 *
 * Built and run by tests/test_abi.py (gcc, no GPU needed).
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "sq.h"

static int failures = 0;

static void expect(int cond, const char* what) {
    if (!cond) {
        fprintf(stderr, "FAILED: %s\n", what);
        ++failures;
    }
}

int main(void) {
    /* a 16-byte aligned address that is never dereferenced */
    void* A = (void*)(uintptr_t)0x7F0000000000ull;
    float* F = (float*)A;

    expect(sq_abi_version() == SQ_ABI_VERSION, "sq_abi_version matches the header");
    expect(strncmp(sq_status_string(SQ_OK), "SQ_OK", 5) == 0, "status string of SQ_OK");
    expect(strstr(sq_status_string(SQ_ERR_TIMEOUT), "TIMEOUT") != NULL, "status string of a timeout");

    /* every call below fails validation on the host */
    expect(sq_calibrate_amax(NULL, SQ_BF16, 4, 64, SQ_AMAX_PER_COLUMN, F, 0, NULL) ==
               SQ_ERR_INVALID_ARG, "calibrate: NULL input");
    expect(sq_smooth_factors(F, F, 64, 1.5, F, NULL, NULL) == SQ_ERR_INVALID_ARG,
           "smooth factors: alpha outside [0,1]");
    expect(sq_quantize_weight(A, SQ_BF16, 40, 64, NULL, SQ_I8, A, F, NULL) == SQ_ERR_INVALID_ARG,
           "quantize weight: K not a multiple of 16");
    expect(sq_quantize_act(A, SQ_BF16, 4, 64, NULL, NULL, SQ_I8, (char*)A + 1, F, 0u, NULL) ==
               SQ_ERR_MISALIGNED, "quantize act: misaligned codes");
    expect(sq_quantize_act(NULL, SQ_BF16, 0, 64, NULL, NULL, SQ_I8, NULL, NULL, SQ_OVERLAP_PREVIOUS, NULL) == SQ_OK,
           "quantize act: empty batch is a no-op");
    expect(sq_quantize_act_tensor(A, SQ_BF16, 4, 64, NULL, NULL, SQ_E4M3, NULL, A, F, NULL, NULL) ==
               SQ_ERR_INVALID_ARG, "per-tensor: the tensor max output is required");
    expect(sq_gemm_w8a8((const int8_t*)A, F, (const int8_t*)A, F, NULL, 16, 64, 133152, A, SQ_BF16,
                        NULL, NULL, 0, NULL) == SQ_ERR_UNSUPPORTED,
           "INT8 GEMM: K beyond the int32 accumulator bound");
    expect(sq_gemm_fp8((const uint8_t*)A, F, (const uint8_t*)A, F, NULL, 16, 12, 64, A, SQ_BF16,
                       NULL, 0, NULL) == SQ_ERR_INVALID_ARG, "FP8 GEMM: N not a multiple of 8");
    expect(sq_linear(A, SQ_BF16, NULL, NULL, A, F, NULL, SQ_F32, 16, 64, 64, A, F, A, SQ_BF16, NULL,
                     0, NULL) == SQ_ERR_INVALID_ARG, "linear: code type must be I8 or E4M3");
    expect(sq_gemm_w8a8_noalloc((const int8_t*)A, F, (const int8_t*)A, F, NULL, 0, 64, 64, A,
                                SQ_BF16, NULL) == SQ_OK, "no-alloc GEMM: empty batch");
    expect(sq_fold_smoothing(A, SQ_F32, 3, 40, F, SQ_AMAX_PER_COLUMN, (float*)A, NULL) ==
               SQ_ERR_INVALID_ARG, "fold: output aliasing the input");
    expect(sq_fold_smoothing(NULL, SQ_F32, 0, 40, NULL, SQ_AMAX_PER_COLUMN, NULL, NULL) == SQ_OK,
           "fold: nothing to fold");
    expect(sq_rmsnorm_quantize_act(A, F, 1e-6f, 4, 16392, SQ_I8, (char*)A + 0x100000, F, NULL, 0u, NULL) ==
               SQ_ERR_UNSUPPORTED, "norm + quantization: K beyond one row on chip");
    expect(sq_rmsnorm_quantize_act(A, F, 0.0f, 4, 64, SQ_I8, (char*)A + 0x100000, F, NULL, 0u, NULL) ==
               SQ_ERR_INVALID_ARG, "norm + quantization: eps must be positive");
    expect(sq_rmsnorm_quantize_act(NULL, NULL, 1e-6f, 0, 64, SQ_E4M3, NULL, NULL, NULL, 0u, NULL) == SQ_OK,
           "norm + quantization: empty batch");
    expect(sq_quantize_act(A, SQ_BF16, 4, 64, NULL, NULL, SQ_I8, (char*)A + 0x100000, F, 2u, NULL) ==
               SQ_ERR_INVALID_ARG, "quantize act: unknown flag bit");
    expect(sq_probe_wait_timeout(10, NULL) == SQ_ERR_INVALID_ARG, "probe: timeout below 1 ms");
    expect(sq_selftest_fast_division(NULL, NULL) == SQ_ERR_INVALID_ARG, "self-test: NULL result");
    (void)sq_gemm_workspace_bytes;  /* links; the size depends on the GPU */
    (void)sq_get_device_status;  /* links; calling it would need a GPU */

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
