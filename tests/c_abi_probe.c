/* A plain C99 caller of the library: the header compiles as C, the library
 * links and loads without Python, and argument errors come back as status
 * codes before any device work (so this runs without a GPU). */
#include <stdio.h>
#include <string.h>

#include "qlora_nf4.h"

#define EXPECT(cond)                                                   \
    do {                                                               \
        if (!(cond)) {                                                 \
            fprintf(stderr, "failed: %s (line %d)\n", #cond, __LINE__); \
            return 1;                                                  \
        }                                                              \
    } while (0)

int main(void) {
    /* aligned stand-ins that are never dereferenced: every call below is
     * refused by its argument checks first */
    void *fake = (void *)(size_t)0x10000;
    nf4_weight w;
    memset(&w, 0, sizeof w);
    w.n = 64;
    w.k = 128;
    w.block_size = 64;
    w.double_quant = 0;
    w.codes = (uint8_t *)fake;
    w.absmax = (float *)fake;

    EXPECT(strcmp(nf4_status_string(NF4_OK), "unknown status") != 0);
    EXPECT(qlora_fwd_workspace_bytes(16, 1024, 1024, 8) >= 256);
    EXPECT(qlora_bwd_workspace_bytes(2048, 5120, 5120, 16) >= 2u * 2048u * 16u * 2u);
    EXPECT(nf4_quantize(NULL, &w, NULL) == NF4_ERR_INVALID_ARG);
    w.block_size = 96;
    EXPECT(nf4_quantize((const float *)fake, &w, NULL) == NF4_ERR_INVALID_ARG);
    w.block_size = 128;
    w.k = 192;
    EXPECT(nf4_quantize((const float *)fake, &w, NULL) == NF4_ERR_UNSUPPORTED_SHAPE);
    w.k = 128;
    EXPECT(qlora_linear_fwd(&w, fake, 4, fake, fake, 7, 16.0f, fake, NULL, fake, 1u << 20, NULL) ==
           NF4_ERR_UNSUPPORTED_SHAPE);
    EXPECT(qlora_linear_fwd(&w, fake, 0, fake, fake, 8, 16.0f, fake, NULL, fake, 1u << 20, NULL) == NF4_OK);
    puts("ok");
    return 0;
}
