/* A plain C program using the library through include/kda.h alone: the sizes
 * queries, the version string and the host-side argument checks (nothing here
 * touches a device, so it runs without a GPU).  Built as C99 and as C++ by
 * tests/test_c_consumer.py; exits 0 when every check holds. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "kda.h"

static int failures = 0;

#define CHECK(cond)                                                          \
    do {                                                                     \
        if (!(cond)) {                                                       \
            fprintf(stderr, "check failed (line %d): %s\n", __LINE__, #cond); \
            ++failures;                                                      \
        }                                                                    \
    } while (0)

/* distinct, 256-byte aligned stand-in addresses: the calls below are all
 * rejected before any of them is dereferenced */
static void* fake(uintptr_t slot) { return (void*)(uintptr_t)((slot + 1u) << 24); }

int main(void) {
    const char* version = kda_version();
    CHECK(version != NULL && strstr(version, "sm_100a") != NULL);

    /* workspace sizes: the per-chunk records of 4 x 64 chunks x 16 heads, at
     * least; a packed batch of the same tokens needs no less; invalid sizes
     * give 0 */
    {
        const size_t fixed = kda_chunk_fwd_workspace_size(4, 4096, 16, 128, 128, 4, 0, KDA_BF16);
        const size_t packed = kda_chunk_fwd_workspace_size(1, 4 * 4096, 16, 128, 128, 4, 1, KDA_BF16);
        const size_t bwd = kda_chunk_bwd_workspace_size(4, 4096, 16, 128, 128, 4, 0, KDA_BF16);
        CHECK(fixed > (size_t)4 * 64 * 16 * 128 * 128);
        CHECK(packed >= fixed);
        CHECK(bwd > fixed);
        CHECK(kda_chunk_fwd_workspace_size(1, 100, 2, 96, 64, 1, 0, KDA_F32) == 0);
        CHECK(kda_chunk_fwd_workspace_size(2, 100, 2, 64, 64, 2, 1, KDA_F32) == 0);
    }

    /* host-side rejections, each with a message */
    {
        const void* q = fake(0);
        const void* k = fake(1);
        const void* v = fake(2);
        const float* la = (const float*)fake(3);
        const float* beta = (const float*)fake(4);
        void* o = fake(5);
        void* ws = fake(6);
        kda_status s;

        s = kda_chunk_fwd(q, k, v, la, beta, NULL, NULL, 1, 64, 1, 96, 64, 1, KDA_F32, o, NULL, ws,
                          (size_t)1 << 30, NULL);
        CHECK(s == KDA_ERR_UNSUPPORTED);
        CHECK(kda_last_error() != NULL && kda_last_error()[0] != '\0');

        s = kda_chunk_fwd(NULL, k, v, la, beta, NULL, NULL, 1, 64, 1, 64, 64, 1, KDA_F32, o, NULL, ws,
                          (size_t)1 << 30, NULL);
        CHECK(s == KDA_ERR_INVALID_ARG);

        s = kda_chunk_fwd(q, k, v, la, beta, NULL, NULL, 1, 64, 1, 64, 64, 1, KDA_F32, o, NULL, NULL,
                          (size_t)1 << 30, NULL);
        CHECK(s == KDA_ERR_WORKSPACE);

        s = kda_chunk_fwd(q, k, v, la, beta, NULL, NULL, 1, 64, 1, 64, 64, 1, KDA_F32, o, NULL, ws, 16,
                          NULL);
        CHECK(s == KDA_ERR_WORKSPACE);

        s = kda_recurrent_step(q, k, v, la, beta, (float*)fake(7), 2, 2, 80, 64, KDA_BF16, o, NULL);
        CHECK(s == KDA_ERR_UNSUPPORTED);

        /* the output must not alias the state it is read from */
        s = kda_recurrent_step(q, k, v, la, beta, (float*)fake(7), 2, 2, 64, 64, KDA_BF16, fake(7), NULL);
        CHECK(s == KDA_ERR_INVALID_ARG);
    }

    if (failures == 0) printf("host calls ok\n");
    return failures == 0 ? 0 : 1;
}
