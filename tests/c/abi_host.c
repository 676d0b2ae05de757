/* Plain C client of the Gated Delta Rule-2 library: includes only gdr2.h and
 * links libgdr2.so. It exercises the host-side part of the boundary that needs
 * no GPU (version, status strings, workspace queries, argument validation)
 * and prints "ok" when every check holds. */
#include <stdio.h>
#include <string.h>

#include "gdr2.h"

static int failures = 0;
#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            ++failures;                                               \
        }                                                             \
    } while (0)

int main(void)
{
    CHECK(gdr2_version() >= 100);
    CHECK(strcmp(gdr2_status_string(GDR2_OK), "ok") == 0);
    CHECK(strcmp(gdr2_status_string(GDR2_ERR_WORKSPACE), "ok") != 0);

    size_t bytes = 1;
    CHECK(gdr2_chunk_fwd_workspace_size(4, 2048, 16, 128, 128, 4, GDR2_BF16, &bytes) == GDR2_OK);
    CHECK(bytes == 0);   /* a full fixed-length batch needs no scratch */
    CHECK(gdr2_chunk_fwd_workspace_size(1, 1000, 4, 128, 128, 3, GDR2_BF16, &bytes) == GDR2_OK);
    CHECK(bytes > 0 && bytes % 256 == 0);
    CHECK(gdr2_chunk_fwd_workspace_size(1, 64, 1, 96, 96, 1, GDR2_FP32, &bytes) == GDR2_ERR_UNSUPPORTED);

    CHECK(gdr2_chunk_bwd_workspace_size(4, 2048, 16, 128, 128, 4, GDR2_BF16, &bytes) == GDR2_OK);
    {
        const size_t slots = 4 * 2048 / 64 + 4;
        const size_t expect = 2 * slots * 16 * 128 * 128 * 4 + 2 * (size_t)4 * 2048 * 16 * 128 * 4;
        CHECK(bytes >= expect && bytes < expect + 256);
    }

    /* validation happens before any launch: null pointers, bad sizes */
    CHECK(gdr2_chunk_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 2, 64, 4, 128, 128, 2,
                         GDR2_BF16, NULL, NULL, NULL, 0, NULL) == GDR2_ERR_INVALID_ARG);
    CHECK(gdr2_recurrent_step(NULL, NULL, NULL, NULL, NULL, NULL, NULL, 4, 0, 64, 64, GDR2_FP32,
                              NULL, NULL) == GDR2_ERR_INVALID_ARG);
    CHECK(gdr2_chunk_bwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 2, 64, 4, 64,
                         64, 2, GDR2_FP32, NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0,
                         NULL) == GDR2_ERR_INVALID_ARG);
    /* empty problems are valid and launch nothing */
    CHECK(gdr2_chunk_fwd(NULL, NULL, NULL, NULL, NULL, NULL, NULL, NULL, 0, 64, 4, 128, 128, 0,
                         GDR2_BF16, NULL, NULL, NULL, 0, NULL) == GDR2_OK);

    if (failures == 0) printf("ok\n");
    return failures == 0 ? 0 : 1;
}
