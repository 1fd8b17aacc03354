/* Calls libmla through include/mla.h from plain C99: workspace sizes, host
 * argument checks and status strings (nothing here launches a kernel, so it
 * runs without a GPU).  Prints one line per check; exits non-zero on the
 * first mismatch. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "mla.h"

#define CHECK(cond, what)                                   \
    do {                                                    \
        if (!(cond)) {                                      \
            printf("FAIL %s\n", what);                      \
            return 1;                                       \
        }                                                   \
        printf("ok %s\n", what);                            \
    } while (0)

int main(void) {
    mla_dims d = {128, 512, 64, 128, 128, MLA_BF16, 0.07216878f, 10000.0f};
    void* fake = (void*)(uintptr_t)0x10000;   /* never dereferenced: every call below fails its checks first */

    size_t ws = mla_decode_workspace_bytes(&d, 64, 1, 4096, 0);
    CHECK(ws > (size_t)64 * 128 * 576 * 2, "decode workspace covers the absorbed queries");
    mla_ws_layout L;
    CHECK(mla_decode_workspace_layout(&d, 64, 1, 4096, 0, &L) == MLA_OK && L.total == ws, "layout total");
    CHECK(mla_prefill_workspace_bytes(&d, 1, 4096, 4096) >= (size_t)2 * 128 * 4096 * 128 * 2,
          "prefill workspace covers the expanded keys and values");

    /* host-checkable errors return before anything is enqueued */
    CHECK(mla_decode(&d, 2, 1, NULL, fake, fake, fake, fake, 100, fake, 100, fake, fake, ws, 0, fake, NULL) ==
              MLA_ERR_ARG, "decode: null query");
    CHECK(mla_decode(&d, 2, 1, fake, fake, fake, fake, fake, 100, fake, 100, fake, fake, 0, 0, fake, NULL) ==
              MLA_ERR_WORKSPACE, "decode: workspace too small");
    CHECK(mla_decode(&d, 0, 1, NULL, NULL, NULL, NULL, NULL, 100, NULL, 100, NULL, NULL, 0, 0, NULL, NULL) ==
              MLA_OK, "decode: empty batch is a no-op");
    CHECK(mla_output_projection(&d, -1, 7168, fake, fake, fake, fake, NULL) == MLA_ERR_ARG,
          "output projection: negative token count");
    mla_dims f32 = d;
    f32.dtype = MLA_FP32;
    CHECK(mla_prefill(&f32, 1, 4, fake, fake, fake, fake, fake, 100, fake, 100, fake, fake, (size_t)1 << 30, fake,
                      NULL) == MLA_ERR_UNSUPPORTED, "prefill: fp32 is not implemented");
    mla_dims odd = d;
    odd.d_rope = 63;
    CHECK(mla_decode_workspace_bytes(&odd, 1, 1, 10, 0) == 0, "odd rope width rejected");

    CHECK(strcmp(mla_status_string(MLA_ERR_LEN), "MLA_ERR_LEN") == 0, "status string");
    CHECK(strcmp(mla_status_string(MLA_ERR_INDEX), "MLA_ERR_INDEX") == 0, "status string (index)");
    return 0;
}
