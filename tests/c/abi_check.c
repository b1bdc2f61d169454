/* A plain C99 caller of the C ABI in include/attn.h: it checks that the
 * header compiles as C, that the library links, and that argument checks
 * answer before any CUDA work (no GPU is needed). Exit status 0 on success;
 * the first failing check's line number otherwise. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "attn.h"

#define CHECK(cond)                                              \
    do {                                                         \
        if (!(cond)) {                                           \
            fprintf(stderr, "abi_check: failed at line %d: %s\n", \
                    __LINE__, #cond);                            \
            return __LINE__;                                     \
        }                                                        \
    } while (0)

int main(void) {
    void* p = (void*)(uintptr_t)0x10000;       /* aligned, never dereferenced */
    void* mis = (void*)(uintptr_t)0x10008;
    const int* kl_mis = (const int*)(uintptr_t)0x10002;

    /* status strings */
    CHECK(strcmp(attn_status_string(ATTN_OK), "unknown status") != 0);
    CHECK(strcmp(attn_status_string((attn_status_t)99), "unknown status") == 0);

    /* workspace: 2 x (B*H*n_pad*4 rounded to 256) + (B*H*n*d*4 rounded to 256)
       + (256 + 4 per (batch, head), rounded to 256) */
    CHECK(attn_bwd_workspace_size(1, 1, 64, 64, 64, 64, ATTN_BF16) ==
          2 * 512 + 64 * 64 * 4 + 512);
    CHECK(attn_bwd_workspace_size(0, 1, 1, 1, 1, 1, ATTN_BF16) == 0);

    /* argument checks, before any launch */
    CHECK(attn_fwd(NULL, p, p, p, p, 1, 1, 64, 64, 64, 64, ATTN_BF16, 0, 0.125f, NULL) ==
          ATTN_ERR_NULL);
    CHECK(attn_fwd(p, p, p, p, p, 1, 1, 64, 65, 64, 64, ATTN_BF16, 1, 0.125f, NULL) ==
          ATTN_ERR_SHAPE);
    CHECK(attn_fwd(mis, p, p, p, p, 1, 1, 64, 64, 64, 64, ATTN_BF16, 0, 0.125f, NULL) ==
          ATTN_ERR_ALIGN);
    CHECK(attn_fwd(p, p, p, p, p, 1, 1, 64, 64, 64, 64, (attn_dtype_t)7, 0, 0.125f, NULL) ==
          ATTN_ERR_DTYPE);
    CHECK(attn_fwd_masked(p, p, p, p, p, kl_mis, 1, 1, 64, 64, 64, 64, ATTN_BF16, 0, 0.125f,
                          NULL) == ATTN_ERR_ALIGN);
    CHECK(attn_bwd(p, p, p, p, p, p, p, p, p, NULL, 0, 1, 1, 64, 64, 64, 64, ATTN_BF16, 0,
                   0.125f, NULL) == ATTN_ERR_WORKSPACE);
    CHECK(attn_set_path((attn_path_t)9) == ATTN_ERR_UNSUPPORTED);
    CHECK(attn_proj_bwd_workspace_size(2, 64, 64, 2, 64, 64, ATTN_F32) == 0);
    printf("abi_check ok\n");
    return 0;
}
