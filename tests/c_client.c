/* A plain C11 client of include/ft.h: the boundary is usable from C with no
 * C++ or CUDA headers.  Exercises only entry points and validation paths
 * that run on the host (no GPU needed); exits 0 and prints "ok" when every
 * check holds, else prints the first failing check and exits 1. */
#include <stdio.h>
#include <string.h>

#include "ft.h"

#define CHECK(c)                                                   \
    do {                                                           \
        if (!(c)) {                                                \
            printf("failed: %s (line %d)\n", #c, __LINE__);       \
            return 1;                                              \
        }                                                          \
    } while (0)

int main(void) {
    /* status names */
    CHECK(strcmp(ft_status_str(FT_OK), "FT_OK") == 0);
    CHECK(strcmp(ft_status_str(FT_ERR_SHAPE), "FT_ERR_SHAPE") == 0);

    /* workspace sizes: positive, deterministic, growing with the batch */
    const size_t w1 = ft_workspace_bytes(128, 256, 256, 16, 16);
    const size_t w2 = ft_workspace_bytes(4608, 3072, 3072, 32, 16);
    CHECK(w1 > 0 && w2 > w1);
    CHECK(w2 == ft_workspace_bytes(4608, 3072, 3072, 32, 16));
    CHECK(ft_quantize_workspace_bytes() > 0);
    CHECK(ft_weight_operand_bytes(3072, 3072) >= (size_t)3072 * 3072 / 2);

    /* where Q(X) lands inside the workspace */
    size_t co = 0, so = 0, go = 0;
    CHECK(ft_workspace_qact(4608, 3072, 3072, 32, 16, &co, &so, &go) == FT_OK);
    CHECK(co + (size_t)4608 * 3072 / 2 <= w2 && so + (size_t)4608 * 3072 / 16 <= w2 && go + 4 <= w2);
    CHECK(ft_workspace_qact(4608, 3072, 3072, 32, 16, NULL, &so, &go) == FT_ERR_INVALID_ARG);

    /* host validation returns before any launch */
    ft_fp4 out;
    memset(&out, 0, sizeof(out));
    CHECK(ft_quantize(NULL, 128, 256, 256, FT_BLK_1x16, NULL, &out, NULL, 0, NULL) == FT_ERR_INVALID_ARG);
    CHECK(ft_linear_fwd(NULL, NULL, 128, NULL, NULL, FT_BF16, NULL, NULL, NULL, 0, NULL) == FT_ERR_INVALID_ARG);

    /* the quantizer's launch mode switch is host-only */
    CHECK(ft_set_cooperative_quantizer(1) == FT_OK);
    CHECK(ft_set_cooperative_quantizer(0) == FT_OK);

    printf("ok\n");
    return 0;
}
