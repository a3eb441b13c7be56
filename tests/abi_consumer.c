/* A plain C99 consumer of the C ABI (include/fastmamba.h), built and run by
 * tests/test_abi_host.py with gcc against the in-tree libfastmamba.so.  It
 * calls only entry points that need no GPU: status names, the version, the
 * exponent-table layout, workspace sizes and argument validation (every
 * rejected call returns before any launch).  Exit status 0 when every check
 * holds; otherwise the number of the first failed check. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "fastmamba.h"

#define CHECK(n, cond)                                   \
    do {                                                 \
        if (!(cond)) {                                   \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                    \
        }                                                \
    } while (0)

int main(void) {
    const fm_shape s130 = {768, 1536, 64, 128, 1, 4};
    const fm_shape bad = {768, 1536, 32, 128, 1, 4};
    fm_exp_layout X;
    size_t one, pipe;

    CHECK(1, strcmp(fm_status_string(FM_OK), "FM_OK") == 0);
    CHECK(2, strcmp(fm_status_string(FM_ERR_WORKSPACE), "FM_ERR_WORKSPACE") == 0);
    CHECK(3, fm_version() >= 100);

    /* the exponent table of the 130M shape: conv_ch = 1792, nheads = 24 */
    X = fm_exp_table_layout(&s130);
    CHECK(4, X.e_u == 0 && X.e_w == 1792 && X.e_o == 2 * 1792 && X.e_x == 3 * 1792);
    CHECK(5, X.size == 3 * 1792 + 4 * 24 + 3);

    /* workspace sizes: the stack's plain loop needs a layer's; pipelined more */
    one = fm_workspace_bytes(&s130, 1, 2048);
    CHECK(6, one > 0);
    CHECK(7, fm_stack_workspace_bytes(&s130, 24, 1, 2048, 1) == one);
    pipe = fm_stack_workspace_bytes(&s130, 24, 1, 2048, 4);
    CHECK(8, pipe > one);
    CHECK(9, fm_stack_workspace_bytes(&s130, 24, 1, 2048, 0) == 0);
    CHECK(10, fm_workspace_bytes(&bad, 1, 16) == 0);

    /* validation before any launch */
    CHECK(11, fm_hadamard_quant(NULL, 4, 768, NULL, 1, FM_DYNAMIC, NULL, NULL, NULL, NULL, NULL) ==
                  FM_ERR_INVALID_ARG);
    CHECK(12, fm_w8a8_gemm(NULL, NULL, 4, NULL, NULL, 8, 100, NULL, NULL, NULL, NULL) ==
                  FM_ERR_SHAPE);
    CHECK(13, fm_decode_step(NULL, NULL, 1, 0, NULL, NULL, NULL, NULL, 0, NULL) ==
                  FM_ERR_INVALID_ARG);
    CHECK(14, fm_stack_prefill(NULL, 2, (float *)(uintptr_t)0x7000000, 1, 64, NULL, NULL, 0, NULL, 0,
                               NULL) == FM_ERR_INVALID_ARG);
    CHECK(15, strlen(fm_last_error()) > 0);
    CHECK(16, fm_set_state_spec(16, 3) == FM_ERR_INVALID_ARG);
    CHECK(17, fm_set_scan_tile(4, 3, 32) == FM_ERR_INVALID_ARG);
    printf("abi_consumer: 17 checks passed\n");
    return 0;
}
