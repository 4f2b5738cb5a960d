/*
 * Plain-C client of the block-attention library: compiled with a C compiler
 * against include/ba.h and linked against libba.so. It checks that the
 * header is valid C99 and exercises only calls that never reach the device:
 * status strings, the version, workspace-size arithmetic and argument
 * errors that are returned before anything is launched.
 * Exit status 0 = every check passed; otherwise the number of failures.
 */
#include "ba.h"

#include <stdint.h>
#include <stdio.h>
#include <string.h>

static int failures = 0;

#define CHECK(cond)                                                                 \
    do {                                                                            \
        if (!(cond)) {                                                              \
            fprintf(stderr, "%s:%d: check failed: %s\n", __FILE__, __LINE__, #cond); \
            ++failures;                                                             \
        }                                                                           \
    } while (0)

static size_t align256(size_t x) { return (x + 255) & ~(size_t)255; }

int main(void)
{
    /* a never-dereferenced, 256-byte-aligned address: every call below fails its checks first */
    void *fake = (void *)(uintptr_t)(1u << 20);
    ba_problem p;
    ba_rope rope;
    size_t f, b, rf, rb, staged;

    CHECK(strcmp(ba_status_string(BA_OK), "ok") == 0);
    CHECK(strcmp(ba_status_string(BA_ERR_TIMEOUT), "device wait timed out") == 0);
    CHECK(ba_version() >= 100);

    p.batch = 3;
    p.total_tokens = 1000;
    p.heads = 2;
    p.head_dim = 128;
    p.dtype = BA_BF16;
    f = ba_fwd_workspace_size(&p, 128, 2);
    b = ba_bwd_workspace_size(&p, 128, 2);
    CHECK(f > 0 && f % 256 == 0 && b > f);
    /* the backward adds two float per-row buffers [heads, total_tokens] and
       (bf16) 128 staged rows of q and of dout per example */
    staged = 2 * align256((size_t)3 * 128 * 2 * 128 * 2);
    CHECK(b == f + 2 * align256(4u * 2 * 1000) + staged);
    /* the rotary forms add two rotated copies of a [T, H, D] bf16 tensor */
    rf = ba_rope_fwd_workspace_size(&p, 128, 2);
    rb = ba_rope_bwd_workspace_size(&p, 128, 2);
    CHECK(rf == f + 2 * align256((size_t)1000 * 2 * 128 * 2));
    CHECK(rb == b + 2 * align256((size_t)1000 * 2 * 128 * 2));
    /* sliding window = block 1 */
    CHECK(ba_swa_fwd_workspace_size(&p, 64) == ba_fwd_workspace_size(&p, 1, 64));
    /* invalid problems size to 0 */
    CHECK(ba_fwd_workspace_size(&p, 0, 2) == 0);
    CHECK(ba_fwd_workspace_size(NULL, 128, 2) == 0);

    /* argument errors come back before any launch */
    CHECK(ba_fwd(NULL, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, f, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_fwd(&p, fake, fake, fake, fake, 0, 2, NULL, fake, fake, fake, f, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_fwd(&p, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, f - 1, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_bwd(&p, fake, fake, fake, fake, fake, fake, fake, 128, 2, NULL, fake, fake, NULL, fake, b, NULL) ==
          BA_ERR_INVALID_ARG);
    p.head_dim = 96;
    CHECK(ba_fwd(&p, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, 1u << 30, NULL) == BA_ERR_UNSUPPORTED);
    p.head_dim = 128;

    memset(&rope, 0, sizeof(rope));
    CHECK(ba_rope_fwd(&p, NULL, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, rf, NULL) ==
          BA_ERR_INVALID_ARG);
    CHECK(ba_rope_fwd(&p, &rope, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, rf, NULL) ==
          BA_ERR_INVALID_ARG); /* no tables */
    rope.cos = (const float *)fake;
    rope.sin = (const float *)fake;
    rope.rows = 1000;
    rope.q_rot = fake; /* k_rot missing */
    CHECK(ba_rope_bwd(&p, &rope, fake, fake, fake, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, fake, rb,
                      NULL) == BA_ERR_INVALID_ARG);
    rope.q_rot = NULL;
    CHECK(ba_rope_fwd(&p, &rope, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, f, NULL) ==
          BA_ERR_INVALID_ARG); /* the plain workspace has no room for the rotated copies */

    CHECK(ba_selftest_wait_timeout(NULL, 256, 1000, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_gdpa_workspace_size(&p, 128, 2) == f + staged);
    CHECK(ba_gdpa_fwd(&p, (ba_activation)7, fake, fake, fake, fake, 128, 2, fake, fake, f, NULL) ==
          BA_ERR_INVALID_ARG); /* not an activation */
    CHECK(ba_gdpa_fwd(&p, BA_ACT_GELU, fake, fake, fake, fake, 128, 2, fake, fake, 16, NULL) ==
          BA_ERR_INVALID_ARG); /* workspace too small */
    CHECK(ba_gdpa_bwd(&p, BA_ACT_SILU, fake, fake, fake, NULL, fake, 128, 2, fake, fake, fake, fake, f, NULL) ==
          BA_ERR_INVALID_ARG); /* no dout */
    CHECK(ba_gdpa_cross_workspace_size(&p, 5000) >= ba_gdpa_cross_workspace_size(&p, 10));
    CHECK(ba_gdpa_cross_workspace_size(&p, -1) == 0);
    CHECK(ba_gdpa_cross_fwd(&p, 500, BA_ACT_GELU, fake, fake, fake, fake, NULL, fake, fake, f, NULL) ==
          BA_ERR_INVALID_ARG); /* no key/value offsets */
    CHECK(ba_gdpa_cross_bwd(&p, -3, BA_ACT_SILU, fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, f,
                            NULL) == BA_ERR_INVALID_ARG); /* negative key/value count */
    CHECK(ba_mx_quantize(NULL, 10, 2, 128, NULL, NULL, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_mx_quantize(fake, 10, 2, 100, fake, fake, NULL) == BA_ERR_INVALID_ARG); /* head_dim not a multiple of 32 */
    CHECK(ba_mx_fwd_workspace_size(&p, 128, 2) > f);
    CHECK(ba_mx_fwd(&p, fake, fake, fake, fake, 128, 2, NULL, fake, fake, fake, f, NULL) ==
          BA_ERR_INVALID_ARG); /* the plain workspace has no room for the MXFP8 operands */
    /* the MXFP8 backward: the backward's workspace plus two bf16 round-trip copies of q and k */
    CHECK(ba_mx_bwd_workspace_size(&p, 128, 2) == b + 2 * align256((size_t)1000 * 2 * 128 * 2));
    CHECK(ba_mx_bwd(&p, fake, fake, fake, fake, (const float *)fake, fake, fake, 128, 2, NULL, fake, fake, fake,
                    fake, b, NULL) == BA_ERR_INVALID_ARG); /* the plain backward's workspace is too small */
    CHECK(ba_mx_bwd(&p, fake, fake, fake, fake, NULL, fake, fake, 128, 2, NULL, fake, fake, fake, fake, 1u << 30,
                    NULL) == BA_ERR_INVALID_ARG); /* no lse */
    CHECK(ba_selftest_exp2(NULL, NULL, 5, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_selftest_exp2((const float *)fake, (float *)fake, -1, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_selftest_exp2(NULL, NULL, 0, NULL) == BA_OK); /* nothing to do, nothing launched */
    CHECK(ba_selftest_activation((ba_activation)0, (const float *)fake, (float *)fake, (float *)fake, 4, NULL) ==
          BA_ERR_INVALID_ARG); /* not an activation */
    CHECK(ba_selftest_activation(BA_ACT_GELU, NULL, NULL, NULL, 4, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_selftest_activation(BA_ACT_SILU, NULL, NULL, NULL, 0, NULL) == BA_OK); /* nothing launched */
    CHECK(ba_set_profile_events(3, NULL, NULL) == BA_ERR_INVALID_ARG);
    CHECK(ba_device_status(NULL, NULL) == BA_ERR_INVALID_ARG);

    if (failures == 0) printf("abi_check: all checks passed\n");
    return failures;
}
