/*
 * A plain C99 client of libfp8bs.so that sees only include/fp8bs.h.  It runs
 * the host-side paths that need no GPU: version and status names, argument
 * errors returned before any launch, and empty problems as no-ops.  Prints
 * "abi c client ok" and exits 0 when every check holds.
 */
#include <stdio.h>
#include <string.h>

#include "fp8bs.h"

static int failures = 0;

static void check(int cond, const char *what) {
    if (!cond) {
        fprintf(stderr, "FAILED: %s (last error: %s)\n", what, fp8bs_last_error_message());
        ++failures;
    }
}

int main(void) {
    /* Operand pointers that are never dereferenced: validation fails first. */
    const uint8_t *codes = (const uint8_t *)(uintptr_t)4096;
    const float *scales = (const float *)(uintptr_t)4096;
    uint16_t *y = (uint16_t *)(uintptr_t)4096;
    fp8bs_status st;

    check(fp8bs_version() >= 100, "version");
    check(strcmp(fp8bs_status_string(FP8BS_OK), "FP8BS_OK") == 0, "status string OK");
    check(strcmp(fp8bs_status_string(FP8BS_ERR_INVALID_ARG), "FP8BS_ERR_INVALID_ARG") == 0,
          "status string INVALID_ARG");

    /* K must be a positive multiple of 128. */
    st = fp8bs_fp8_gemm(codes, scales, codes, scales, 8, 256, 100, y, NULL, 0, NULL);
    check(st == FP8BS_ERR_INVALID_ARG, "fp8_gemm K=100 refused");
    check(strstr(fp8bs_last_error_message(), "K=100") != NULL, "fp8_gemm K=100 message");

    /* Block sizes other than 32, 64, 128 and 256 are not implemented. */
    st = fp8bs_act_quant(codes, FP8BS_DTYPE_BF16, 4, 96, 48, FP8BS_SCALE_FMT_NONE, NULL, NULL,
                         NULL);
    check(st == FP8BS_ERR_UNSUPPORTED, "act_quant block=48 unsupported");

    /* Empty problems succeed without touching a device. */
    st = fp8bs_act_quant(NULL, FP8BS_DTYPE_BF16, 0, 256, 128, FP8BS_SCALE_FMT_UE8M0, NULL, NULL,
                         NULL);
    check(st == FP8BS_OK, "act_quant rows=0");
    st = fp8bs_fp8_gemm(codes, scales, codes, scales, 0, 256, 128, y, NULL, 0, NULL);
    check(st == FP8BS_OK, "fp8_gemm M=0");
    st = fp8bs_weight_dequant(NULL, NULL, 0, 16, 128, NULL, FP8BS_DTYPE_BF16, NULL);
    check(st == FP8BS_OK, "weight_dequant M=0");

    if (failures) return 1;
    printf("abi c client ok\n");
    return 0;
}
