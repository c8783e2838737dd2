/* The boundary used from plain C: this program includes only include/fp8vit.h,
 * links libfp8vit.so and exercises the calls that need no GPU (status strings,
 * the descale rule, the scale-file reader and writer, and the host-side
 * argument checks of the device entry points, which return before any CUDA
 * call).  Built and run by tests/test_abi.py; exit status 0 means every check
 * held, otherwise it is the number of the first failed check. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "fp8vit.h"

#define CHECK(n, cond)                                      \
    do {                                                    \
        if (!(cond)) {                                      \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                       \
        }                                                   \
    } while (0)

int main(int argc, char** argv) {
    if (argc != 3) return 100;
    const char* golden = argv[1];  /* the pages' printed scale-file example */
    const char* scratch = argv[2]; /* a writable path */
    CHECK(1, fp8vit_version() >= 100);
    CHECK(2, strcmp(fp8vit_status_string(FP8VIT_OK), "ok") == 0);
    CHECK(3, fp8_descale_from_amax(224.0f) == 0.5f);
    CHECK(4, fp8_descale_from_amax(0.0f) == 1e-10f);
    CHECK(41, fp8_descale_from_amax_margin(224.0f, 1.5f) == 0.75f);

    float v[3] = {0, 0, 0};
    CHECK(5, fp8_static_scales_load(golden, "visual.blocks.0.attn.attn", v) == FP8VIT_OK);
    CHECK(6, v[0] == 224.0f && v[1] == 198.0f && v[2] == 210.0f);
    CHECK(7, fp8_static_scales_load(golden, "no.such.layer", v) == FP8VIT_ENOTFOUND);

    const char* layers[2] = {"blocks.0", "blocks.1"};
    const float amax[6] = {1.0f, 2.0f, 3.0f, 10.0f, 20.0f, 30.0f};
    CHECK(8, fp8_static_scales_save(scratch, 2, layers, amax, 1.5f) == FP8VIT_OK);
    CHECK(9, fp8_static_scales_load(scratch, "blocks.1", v) == FP8VIT_OK);
    CHECK(10, v[0] == 15.0f && v[1] == 30.0f && v[2] == 45.0f);
    CHECK(11, fp8_static_scales_save(scratch, 2, layers, amax, -1.0f) == FP8VIT_EINVAL);

    /* host-side checks: null context / pointers come back before any CUDA call */
    CHECK(12, fp8vit_check(NULL, NULL, NULL) == FP8VIT_EINVAL);
    CHECK(13, fp8vit_set_attn_p_terms(NULL, 2) == FP8VIT_EINVAL);
    CHECK(14, fp8_amax_ring_update(NULL, NULL, NULL, NULL, 8, NULL, NULL, NULL) ==
                  FP8VIT_EINVAL);
    CHECK(15, fp8_varlen_attn_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 1, 64, 64, 16,
                                  128, 0.088f, NULL, 0, NULL, NULL) == FP8VIT_EINVAL);
    CHECK(16, per_token_group_quant_fp8(NULL, NULL, 1, 128, 128, NULL, NULL, NULL) ==
                  FP8VIT_EINVAL);
    CHECK(17, fp8_varlen_attn_fwd_bf16_group_quant(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL,
                                                   1, 64, 64, 16, 72, 0.118f, NULL, NULL, NULL,
                                                   NULL, NULL) == FP8VIT_EINVAL);
    printf("ok\n");
    return 0;
}
