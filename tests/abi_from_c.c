/* Calls the library through its header from plain C (test infrastructure):
 * checks that the header is valid C11 and that the entry points link and run.
 * Only host-side paths are exercised (no device is needed): the version,
 * status strings, workspace queries and argument validation.  Prints one
 * line per check; exits non-zero on the first failure. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "xlstm_mlstm.h"

#define CHECK(cond, what)                                   \
    do {                                                    \
        if (!(cond)) {                                      \
            printf("FAIL %s\n", what);                      \
            return 1;                                       \
        }                                                   \
        printf("ok %s\n", what);                            \
    } while (0)

int main(void) {
    size_t bytes = 0;
    void *fake = (void *)(uintptr_t)((uint64_t)1 << 40);   /* aligned, never dereferenced */
    CHECK(xlstm_abi_version() == XLSTM_ABI_VERSION, "abi version");
    CHECK(strcmp(xlstm_status_string(XLSTM_OK), "ok") == 0, "status string");
    CHECK(xlstm_mlstm_fwd_workspace_size(1, 8, 16384, 256, 64, XLSTM_BF16, &bytes) == XLSTM_OK &&
              bytes > 0, "forward workspace size");
    CHECK(xlstm_mlstm_fwd_workspace_size(1, 8, 16384, 256, 32, XLSTM_BF16, &bytes) ==
              XLSTM_ERR_CHUNK, "bf16 chunk rule");
    CHECK(xlstm_mlstm_bwd_workspace_size(1, 2, 10, 16, 4, XLSTM_F32, &bytes) == XLSTM_OK &&
              bytes > 0, "backward workspace size");
    CHECK(xlstm_mlstm_fwd(NULL, fake, fake, fake, fake, fake, fake, NULL, NULL, NULL, NULL, NULL,
                          NULL, 1, 1, 64, 64, 64, XLSTM_F32, XLSTM_FGATE_SIGMOID, fake, 0,
                          NULL) == XLSTM_ERR_NULL, "forward rejects a NULL q");
    CHECK(xlstm_mlstm_step(fake, fake, fake, fake, fake, fake, fake, fake, fake, fake, 1, 1, 24,
                           XLSTM_BF16, XLSTM_FGATE_EXP, NULL) == XLSTM_ERR_SHAPE,
          "step rejects DH 24");
    CHECK(xlstm_mlstm_headnorm_gate(fake, fake, fake, NULL, NULL, fake, fake, 1, 2, 8, 64, 0.0f,
                                    XLSTM_BF16, XLSTM_OGATE_SILU, NULL) == XLSTM_ERR_UNSUPPORTED,
          "epilogue rejects eps 0");
    CHECK(xlstm_slstm_fwd(fake, fake, fake, fake, fake, fake, NULL, NULL, NULL, NULL, NULL, NULL,
                          NULL, NULL, 1, 1, 4, 16, (xlstm_fgate)7, NULL) == XLSTM_ERR_DTYPE,
          "sLSTM rejects a bad gate kind");
    CHECK(xlstm_selftest_wait_timeout(0, NULL) == XLSTM_ERR_SHAPE, "self-test limit range");
    return 0;
}
