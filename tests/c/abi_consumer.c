/* A plain C program against include/w4a16.h and libw4a16.so: the boundary is usable without
 * Python or PyTorch.  It only calls what needs no GPU (size queries, argument validation, status
 * strings) and prints one line per check; the test that builds it compares the output. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "w4a16.h"

static int fails = 0;
#define CHECK(cond, what)                                  \
    do {                                                   \
        if (cond) {                                        \
            printf("ok %s\n", what);                       \
        } else {                                           \
            printf("FAIL %s\n", what);                     \
            ++fails;                                       \
        }                                                  \
    } while (0)

int main(void) {
    size_t bytes = 1;
    CHECK(w4_gemm_workspace_size(1, 4096, 4096, 128, &bytes) == W4_OK, "gemm workspace query");
    CHECK(w4_gemm_workspace_size(1, 4096, 4000, 128, &bytes) == W4_ERR_SHAPE, "K not a multiple of 128");
    CHECK(w4_gemm_workspace_size(1, 4096, 4096, 64, &bytes) == W4_ERR_UNSUPPORTED, "group 64 for INT4 GEMM");
    CHECK(awq_workspace_size(65536, 4096, 4096, 128, 20, &bytes) == W4_OK && bytes > 4096u * 4096u * 2u,
          "awq workspace holds E");
    CHECK(awq_gram_workspace_size(65536, 4096, 4096, 128, 20, &bytes) == W4_OK, "gram workspace query");
    CHECK(gptq_workspace_size(4096, 4096, 4096, 128, &bytes) == W4_OK &&
              bytes >= (size_t)16 * 4096 * 4096 + (size_t)8 * 4096 * 4096,
          "gptq workspace holds H, its factors and W");
    CHECK(wb_gemm_workspace_size(1, 4096, 4096, 3, 128, &bytes) == W4_OK && bytes == (size_t)4096 * 4096 * 2,
          "wb_gemm workspace is the fp16 weights");
    CHECK(w4_quantize_pack(NULL, 64, 512, 128, NULL, NULL, NULL, NULL, NULL) == W4_ERR_NULL, "NULL weights");
    CHECK(w4_quantize_pack_bits(NULL, 64, 512, 5, 128, NULL, NULL, NULL, NULL, NULL) == W4_ERR_UNSUPPORTED,
          "5-bit codes rejected");
    CHECK(w4_gemm(NULL, 1, 64, 512, NULL, NULL, NULL, 128, NULL, NULL, 0, NULL) == W4_ERR_NULL, "NULL GEMM operands");
    CHECK(w4_selftest_bounded_wait(10000000000ull, NULL) == W4_ERR_UNSUPPORTED, "self-test limit above 5 s");
    CHECK(strcmp(w4_status_string(W4_OK), "ok") == 0, "status string ok");
    CHECK(strlen(w4_status_string(W4_ERR_NUMERIC)) > 0, "status string for a non-positive-definite Hessian");
    printf("%d failed\n", fails);
    return fails != 0;
}
