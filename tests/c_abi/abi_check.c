/* Plain C caller of the library: compiles against include/fa.h alone and
 * exercises the host-side argument checks (nothing reaches a GPU). */
#include <stdio.h>
#include <string.h>
#include "fa.h"

#define CHECK(expr, want)                                                        \
    do {                                                                         \
        int got_ = (expr);                                                       \
        if (got_ != (want)) {                                                    \
            printf("FAIL %s: got %d want %d\n", #expr, got_, (want));            \
            return 1;                                                            \
        }                                                                        \
    } while (0)

int main(void) {
    char buf[64];
    void* p = (void*)(size_t)0x10000;          /* never dereferenced */
    float* f = (float*)p;
    CHECK(fa_fwd(NULL, p, p, p, f, 1, 1, 128, 128, 0.1f, 0, 0, NULL, 0), FA_ERR_NULLPTR);
    CHECK(fa_fwd(p, p, p, p, f, 1, 1, 128, 96, 0.1f, 0, 0, NULL, 0), FA_ERR_UNSUPPORTED_D);
    CHECK(fa_fwd(p, p, p, p, f, 1, 1, 128, 128, 0.1f, 0, 7, NULL, 0), FA_ERR_BAD_MASK);
    CHECK(fa_fwd(p, p, p, p, f, 1, 1, 128, 128, -1.0f, 0, 0, NULL, 0), FA_ERR_BAD_SCALE);
    CHECK(fa_fwd(p, p, p, p, f, 0, 1, 128, 128, 0.1f, 0, 0, NULL, 0), FA_OK);
    CHECK(fa_fwd_kv(p, p, p, p, f, 1, 1, 128, 512, 128, 0.1f, 1, 0, (const int*)p, NULL, 0),
          FA_ERR_BAD_SHAPE);
    CHECK(fa_fwd_kv(p, p, p, p, f, 2, 1, 0, 512, 128, 0.1f, 1, 0, NULL, NULL, 0), FA_OK);
    CHECK(fa_fwd_kvcache(p, p, p, p, f, 2, 2, 1, 512, 128, 0.1f, 1, 0, NULL, 33, NULL, 0, 0),
          FA_ERR_BAD_SHAPE);
    CHECK(fa_fwd_kvcache(p, p, p, p, f, 2, 2, 1, 512, 128, 0.1f, 1, 0, NULL, 4, NULL, 0, 0),
          FA_ERR_WORKSPACE);
    CHECK(fa_fwd_kvcache(p, p, p, p, f, 2, 2, 0, 512, 128, 0.1f, 1, 0, NULL, 1, NULL, 0, 0), FA_OK);
    if (fa_fwd_kvcache_workspace_size(16, 16, 1, 128, 8) != (size_t)8 * 16 * 16 * 129 * 4) {
        printf("FAIL kvcache workspace size\n");
        return 1;
    }
    CHECK(fa_quantize_fp8(p, p, f, 1, 128, 1, 64, 0, NULL, 0), FA_ERR_UNSUPPORTED_D);
    CHECK(fa_quantize_fp8(p, p, f, 1, 128, 1, 128, 1, f, 0), FA_ERR_BAD_SHAPE);
    CHECK(fa_fwd_fp8(p, p, p, f, f, f, p, f, 1, 1, 128, 128, 0.1f, 0, 9, 0), FA_ERR_BAD_MASK);
    if (fa_fp8_vt_bytes(2, 3, 200, 128) != (size_t)2 * 3 * 128 * 208) {
        printf("FAIL fp8 V bytes\n");
        return 1;
    }
    CHECK(fa_bwd(p, p, p, p, f, p, p, p, p, 1, 1, 128, 128, 0.1f, 0, 0, NULL, NULL, 0, 0),
          FA_ERR_WORKSPACE);
    CHECK(fa_bwd_noalloc(p, p, p, p, f, p, p, p, p, 1, 16, 65537, 128, 0.1f, 0, 0, NULL, 0),
          FA_ERR_SCRATCH_LIMIT);
    if (fa_bwd_workspace_size(2, 16, 4096, 128, 0) != (size_t)2 * 16 * 4096 * 8) {
        printf("FAIL workspace size\n");
        return 1;
    }
    snprintf(buf, sizeof buf, "%s", fa_status_string(FA_ERR_MISALIGNED));
    if (strstr(buf, "aligned") == NULL) {
        printf("FAIL status string '%s'\n", buf);
        return 1;
    }
    printf("ok\n");
    return 0;
}
