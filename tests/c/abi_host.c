/* Plain C99 use of the library's C ABI (include/h3attn.h): host-only calls
 * and the argument checks that return before any CUDA call. Built and run by
 * tests/test_c_abi.py; exits 0 when every check holds. */
#include <math.h>
#include <stdio.h>
#include <string.h>

#include "h3attn.h"

static int failures = 0;
#define CHECK(cond)                                                        \
    do {                                                                   \
        if (!(cond)) {                                                     \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++failures;                                                    \
        }                                                                  \
    } while (0)

int main(void) {
    /* one segment: 1 image ref (2x3), 1 audio ref of 4 at rate 2, a 2x2x2 grid, 4 audio */
    h3_segment_layout seg;
    memset(&seg, 0, sizeof(seg));
    seg.image_refs = 1; seg.image_h = 2; seg.image_w = 3;
    seg.audio_refs = 1; seg.audio_ref_len = 4; seg.audio_rate = 2;
    seg.video_t = 2; seg.video_h = 2; seg.video_w = 2;
    seg.audio_tail = 4;
    CHECK(h3_segment_tokens(&seg) == 6 + 4 + 8 + 4);

    float pos[22 * 3];
    int32_t cu[2];
    CHECK(h3_build_positions(&seg, 1, pos, 22, cu) == H3_OK);
    CHECK(cu[0] == 0 && cu[1] == 22);
    /* image ref at t = 0, then the audio ref from t = 1 in steps of 1/2 */
    CHECK(pos[0] == 0.0f && pos[5 * 3 + 1] == 1.0f && pos[5 * 3 + 2] == 2.0f);
    CHECK(pos[6 * 3] == 1.0f && pos[7 * 3] == 1.5f && pos[9 * 3] == 2.5f);
    /* the video grid starts at t = 1 + 4/2 = 3, the tail spreads over its 2 frames */
    CHECK(pos[10 * 3] == 3.0f && pos[14 * 3] == 4.0f && pos[18 * 3] == 3.0f && pos[19 * 3] == 3.5f);

    /* the same segment on a clock that starts at 100 */
    double origin = 100.0;
    float pos2[22 * 3];
    CHECK(h3_build_positions_at(&seg, 1, &origin, pos2, 22, NULL) == H3_OK);
    for (int i = 0; i < 22; ++i) {
        CHECK(pos2[3 * i] == pos[3 * i] + 100.0f);
        CHECK(pos2[3 * i + 1] == pos[3 * i + 1] && pos2[3 * i + 2] == pos[3 * i + 2]);
    }
    origin = NAN;
    CHECK(h3_build_positions_at(&seg, 1, &origin, pos2, 22, NULL) == H3_ERR_INVALID_ARG);
    CHECK(h3_build_positions(&seg, 1, pos, 21, cu) == H3_ERR_INVALID_ARG);  /* capacity */

    /* argument checks of the device calls return before any CUDA call */
    h3_rope_cfg rope = {32, 48, 48, 10000.0f};
    void *fake = (void *)(uintptr_t)0x10000;
    void *ws = (void *)(uintptr_t)0x70000;
    CHECK(h3_rope_apply(fake, fake, (const float *)fake, 8, 2, 96, rope, NULL) == H3_ERR_UNSUPPORTED);
    CHECK(h3_varlen_attn_fwd(fake, fake, fake, fake, NULL, (const int32_t *)fake, 1, 8, NULL, rope,
                             8, 2, 128, -1.0f, ws, 1 << 20, NULL) == H3_ERR_INVALID_ARG);
    CHECK(h3_varlen_attn_fwd_sage(fake, fake, fake, fake, NULL, (const int32_t *)fake, 1, 8, NULL,
                                  rope, 8, 2, 64, 0.1f, ws, 1 << 20, NULL) == H3_ERR_UNSUPPORTED);
    CHECK(h3_qkv_rope_gemm(fake, fake, fake, fake, fake, NULL, rope, 8, 100, 2, 128, ws, 256,
                           NULL) == H3_ERR_INVALID_ARG);
    CHECK(h3_workspace_size(0, 1, 64, 1) == 256);
    CHECK(h3_sage_workspace_size(10, 2, 64, 1) == 0);
    CHECK(strcmp(h3_status_string(H3_ERR_BAD_SEQLENS), "invalid cu_seqlens") == 0);
    CHECK(h3_last_cuda_error() == 0);

    if (failures == 0) printf("c abi ok\n");
    return failures == 0 ? 0 : 1;
}
