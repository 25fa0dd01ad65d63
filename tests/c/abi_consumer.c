/*
 * A plain C99 consumer of libw4: include/w4.h must compile as C without
 * warnings, and the host-side paths of the ABI (status strings, layout
 * version, workspace queries, argument rejection) must work from C with no
 * Python and no GPU.  Every compute call below is malformed on purpose and
 * must be refused before anything is launched; the pointers are never
 * dereferenced.  Exit status 0 means every check held.
 */
#include <stdio.h>
#include <string.h>

#include "w4.h"

static int failures = 0;

#define CHECK(cond)                                                          \
    do {                                                                     \
        if (!(cond)) {                                                       \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++failures;                                                      \
        }                                                                    \
    } while (0)

int main(void)
{
    /* 16-byte aligned fake device addresses: refused calls never touch them */
    void *const fake = (void *)(uintptr_t)(1u << 20);
    uint32_t *const fake_u32 = (uint32_t *)fake;
    uint8_t *const fake_u8 = (uint8_t *)fake;
    const w4_stream_t stream = NULL;
    int s;

    CHECK(w4_layout_version() == W4_LAYOUT_VERSION);
    for (s = W4_OK; s <= W4_ERR_CUDA; ++s)
        CHECK(strncmp(w4_status_string(s), "W4_", 3) == 0);
    CHECK(w4_status_string(12345) != NULL);

    /* workspace queries are pure host arithmetic */
    CHECK(w4a16_workspace_bytes(1, 4096, 4096, 128) == 0);        /* the GEMV needs none */
    CHECK(w4_awq_workspace_bytes(128, 4096, 4096, 128, W4_ASYM, 20) > 0);
    CHECK(w4_awq_workspace_bytes(128, 4096, 4096, 128, W4_ASYM, 1) == 0);

    /* malformed requests are refused on the host */
    CHECK(w4_quant_pack(NULL, 16, 256, 128, W4_SYM, NULL, fake_u32, fake, NULL, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_quant_pack(fake, 16, 256, 96, W4_SYM, NULL, fake_u32, fake, NULL, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_quant_pack(fake, 16, 256, 128, W4_ASYM, NULL, fake_u32, fake, NULL, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_quant_pack(fake, 0, 256, 128, W4_SYM, NULL, fake_u32, fake, NULL, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4a16_gemm(fake, 1, 16, 300, fake_u32, fake, NULL, 128, W4_SYM, fake, NULL, 0, stream) ==
          W4_ERR_INVALID_ARG);
    CHECK(w4a16_gemm(fake, 0, 16, 256, fake_u32, fake, NULL, 128, W4_SYM, fake, NULL, 0, stream) ==
          W4_ERR_INVALID_ARG);
    CHECK(w4a16_gemm_noalloc(fake, 1, 16, 256, fake_u32, fake, NULL, 128, 7, fake, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_fp4_quant(fake, 4, 48, W4_MXFP4, fake_u8, fake_u8, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_fp4_quant(fake, 4, 64, 9, fake_u8, fake_u8, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_awq_search(fake, fake, 16, 256, 8, 128, W4_SYM, 1, (double *)fake, (int *)fake, (float *)fake, fake,
                        1u << 20, stream) == W4_ERR_INVALID_ARG);

    /* the offline repack: sizes by host arithmetic, K % 256 != 0 unsupported */
    CHECK(w4_repacked_words(16, 256) == 16 * 32);
    CHECK(w4_repacked_words(17, 256) == 32 * 32);                 /* N padded to whole 16-channel tiles */
    CHECK(w4_repacked_words(16, 320) == 0);
    CHECK(w4_repack(NULL, 16, 256, fake_u32, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_repack(fake_u32, 16, 320, fake_u32, stream) == W4_ERR_UNSUPPORTED);

    /* GPTQ: workspace query, then a group size the quantizer does not take */
    CHECK(w4_gptq_workspace_bytes(64, 256, 128) > 0);
    CHECK(w4_gptq_workspace_bytes(64, 320, 128) == 0);            /* K not a multiple of the group */
    CHECK(w4_gptq(fake, fake, 16, 256, 8, 96, W4_SYM, fake_u32, fake, NULL, fake, 1u << 20, stream) ==
          W4_ERR_INVALID_ARG);

    /* the bf16 rounding of fp32 partial sums */
    CHECK(w4_f32_to_bf16(NULL, 4, fake, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_f32_to_bf16((const float *)fake, 0, fake, stream) == W4_ERR_INVALID_ARG);

    /* the MX path: block sizes, the tensor-core scale layout's K % 128, flags */
    CHECK(w4_mxfp8_quant(fake, 1, 48, fake_u8, fake_u8, W4_MX_SCALES_ROWS, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_mxfp8_quant(fake, 1, 96, fake_u8, fake_u8, W4_MX_SCALES_MMA, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_mxfp8_quant(fake, 1, 128, fake_u8, fake_u8, 5, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_mx_scale_layout(fake_u8, 1, 96, fake_u8, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_mx_gemm(fake_u8, fake_u8, 1, 16, 96, fake_u8, fake_u8, fake, 0, stream) == W4_ERR_INVALID_ARG);
    CHECK(w4_mx_gemm(fake_u8, fake_u8, 1, 16, 128, fake_u8, fake_u8, fake, 3, stream) == W4_ERR_INVALID_ARG);

    /* the failure-path test controls are host settings */
    w4_set_wait_limit_ns(0);
    w4_test_stall_first_wait(0);

    if (failures == 0) printf("c consumer: all checks held\n");
    return failures == 0 ? 0 : 1;
}
