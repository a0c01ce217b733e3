/* The C ABI from plain C99: the header compiles as C and the host-only calls behave as
 * documented on a machine without a GPU (no call here launches device work). */
#include <stdio.h>
#include <string.h>

#include "kda_decode.h"

static int fails = 0;
#define CHECK(c)                                                  \
    do {                                                          \
        if (!(c)) {                                               \
            fprintf(stderr, "check failed: %s (line %d)\n", #c, __LINE__); \
            ++fails;                                              \
        }                                                         \
    } while (0)

int main(void)
{
    kda_config cfg;
    size_t bytes = 0;
    kda_handle h = NULL;
    kda_weights w;
    memset(&cfg, 0, sizeof cfg);
    memset(&w, 0, sizeof w);
    cfg.hidden = 4096;
    cfg.num_heads = 32;
    cfg.head_dk = 128;
    cfg.head_dv = 128;
    cfg.alpha_rank = 64;
    cfg.max_batch = 8;
    cfg.out_dtype = KDA_OUT_F32;
    cfg.engine = KDA_ENGINE_AUTO;

    CHECK(kda_decode_abi_version() == KDA_DECODE_ABI_VERSION);
    CHECK(strcmp(kda_status_string(KDA_OK), "KDA_OK") == 0);
    CHECK(strcmp(kda_status_string(KDA_ERR_DEVICE_TIMEOUT), "KDA_ERR_DEVICE_TIMEOUT") == 0);
    CHECK(kda_decode_scratch_bytes(&cfg, &bytes) == KDA_OK && bytes > 0);
    cfg.hidden = 100;
    CHECK(kda_decode_scratch_bytes(&cfg, &bytes) == KDA_ERR_UNSUPPORTED_SHAPE);
    cfg.hidden = 4096;
    CHECK(kda_decode_init(NULL, &h) == KDA_ERR_INVALID_ARG);
    CHECK(kda_decode_step(NULL, NULL, NULL, NULL, NULL, 1) == KDA_ERR_INVALID_ARG);
    CHECK(kda_decode_step_tokens(NULL, NULL, NULL, NULL, NULL, 1, 2) == KDA_ERR_INVALID_ARG);
    CHECK(kda_state_checkpoint(NULL, NULL, 0, 1, NULL) == KDA_ERR_INVALID_ARG);
    CHECK(kda_decode_destroy(NULL) == KDA_OK);
    /* no-alloc step: a null x is an argument error, found before any device call */
    CHECK(kda_decode_step_noalloc(&cfg, NULL, &w, NULL, NULL, 1, NULL) == KDA_ERR_INVALID_ARG);
    if (fails == 0) printf("abi_check ok\n");
    return fails == 0 ? 0 : 1;
}
