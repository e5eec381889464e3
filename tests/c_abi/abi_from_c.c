/* A C (not C++) client of the library: the header must compile as C99, the library must link
 * and load, and calls that break a rule must return a status before any CUDA call (this program
 * runs without a GPU).  Prints one line per check; exits 0 when all pass. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "nvfp4lora.h"

static int failures = 0;

static void expect(int cond, const char* what) {
    printf("%s %s\n", cond ? "ok" : "FAIL", what);
    if (!cond) ++failures;
}

int main(void) {
    const char* v = nvfp4lora_version();
    expect(v != NULL && strstr(v, "sm_100a") != NULL, "version names sm_100a");

    /* K not a multiple of 256: rejected before CUDA, and the message names K */
    uint8_t* a = (uint8_t*)(uintptr_t)0x10000;
    uint8_t* b = (uint8_t*)(uintptr_t)0x20000;
    uint8_t* sf = (uint8_t*)(uintptr_t)0x30000;
    float* alpha = (float*)(uintptr_t)0x40000;
    uint16_t* out = (uint16_t*)(uintptr_t)0x50000;
    nvfp4lora_status st = nvfp4lora_mm(a, b, sf, 1 << 20, sf, 1 << 20, alpha, NULL, NULL, NULL, 0, NULL, out,
                                       128, 256, 200, NULL);
    expect(st == NVFP4LORA_ERR_INVALID_ARG, "K = 200 is INVALID_ARG");
    expect(strstr(nvfp4lora_last_error(), "K") != NULL, "the message names K");

    /* a null operand */
    st = nvfp4lora_mm(NULL, b, sf, 1 << 20, sf, 1 << 20, alpha, NULL, NULL, NULL, 0, NULL, out, 128, 256, 256, NULL);
    expect(st == NVFP4LORA_ERR_INVALID_ARG, "null a is INVALID_ARG");

    /* the LoRA delta's rank rule */
    st = nvfp4lora_bgmv_moe_gemm2_lora_delta(a, 16, 64, (const int32_t*)sf, (const int64_t*)sf, 0,
                                             (const int64_t*)sf, 0, (const int32_t*)sf, (const float*)sf,
                                             (const int32_t*)sf, 4, 2, 2, 12, 64, NVFP4LORA_DTYPE_BF16, 1.0f,
                                             NVFP4LORA_DTYPE_BF16, out, NULL);
    expect(st == NVFP4LORA_ERR_INVALID_ARG, "rank 12 is INVALID_ARG");

    /* no tokens: nothing to do, nothing enqueued */
    st = nvfp4lora_bgmv_moe_gemm2_lora_delta(NULL, 0, 64, NULL, NULL, 0, NULL, 0, NULL, NULL, NULL, 0, 2, 2, 16, 64,
                                             NVFP4LORA_DTYPE_BF16, 1.0f, NVFP4LORA_DTYPE_FP16, NULL, NULL);
    expect(st == NVFP4LORA_OK, "zero tokens is OK");

    /* the bounded-wait self-test refuses a limit out of range before CUDA */
    st = nvfp4lora_selftest_wait_timeout(0, NULL);
    expect(st == NVFP4LORA_ERR_INVALID_ARG, "self-test limit 0 is INVALID_ARG");
    return failures == 0 ? 0 : 1;
}
