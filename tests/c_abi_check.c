/* A plain C99 consumer of include/tri_attn.h: it compiles the header as C, links
 * against libtri_attn.so and exercises every call that must fail on the host
 * before any CUDA work (so it runs without a GPU). Exit status 0 = all checks
 * held; otherwise the number of the first failed check. */
#include <stdio.h>
#include <string.h>

#include "tri_attn.h"

#define CHECK(n, cond)                                         \
    do {                                                       \
        if (!(cond)) {                                         \
            fprintf(stderr, "check %d failed: %s\n", n, #cond); \
            return n;                                          \
        }                                                      \
    } while (0)

int main(void) {
    void *fake = (void *)(uintptr_t)4096;            /* aligned, never dereferenced */
    size_t n = 0;

    CHECK(1, (tri_attn_version() >> 16) >= 1);
    CHECK(2, strcmp(tri_attn_status_string(TRI_ATTN_OK), "ok") == 0);

    tri_attn_problem p;
    memset(&p, 0, sizeof p);
    p.N = 64; p.H = 4; p.c = 32; p.dtype = TRI_ATTN_BF16; p.variant = TRI_ATTN_STARTING;
    CHECK(3, tri_attn_fwd_workspace_size(&p, &n) == TRI_ATTN_OK && n > 0);
    CHECK(4, tri_attn_bwd_workspace_size(&p, &n) == TRI_ATTN_OK && n > 0);
    p.c = 65;                                          /* head dimensions up to 64 */
    CHECK(5, tri_attn_fwd_workspace_size(&p, &n) == TRI_ATTN_ERR_UNSUPPORTED);
    p.c = 32; p.variant = 7;
    CHECK(6, tri_attn_fwd_workspace_size(&p, &n) == TRI_ATTN_ERR_INVALID_ARG);
    p.variant = TRI_ATTN_STARTING;
    CHECK(7, tri_attn_fwd(&p, fake, fake, fake, fake, fake, NULL, fake, (float *)fake, NULL, 0,
                          NULL) == TRI_ATTN_ERR_WORKSPACE);
    {   /* a batch of 3 ending-node problems needs a transposed bias per problem; a
           negative batch or a nonzero reserved field is refused */
        size_t one = 0, three = 0;
        p.variant = TRI_ATTN_ENDING;
        p.batch = 1;
        CHECK(14, tri_attn_fwd_workspace_size(&p, &one) == TRI_ATTN_OK);
        p.batch = 3;
        CHECK(15, tri_attn_fwd_workspace_size(&p, &three) == TRI_ATTN_OK &&
                      three >= one + 2 * (size_t)2 * 4 * 64 * 64);
        p.variant = TRI_ATTN_STARTING;
        p.batch = -1;
        CHECK(16, tri_attn_fwd_workspace_size(&p, &n) == TRI_ATTN_ERR_INVALID_ARG);
        p.batch = 1; p.reserved = 5;
        CHECK(17, tri_attn_fwd_workspace_size(&p, &n) == TRI_ATTN_ERR_INVALID_ARG);
        p.batch = 0; p.reserved = 0;
    }

    tri_mul_problem m = {64, 4, TRI_MUL_OUTGOING};
    CHECK(8, tri_mul_workspace_size(&m, &n) == TRI_ATTN_OK);
    m.N = 60;                                          /* N must be a multiple of 8 */
    CHECK(9, tri_mul_fwd(&m, fake, fake, fake, fake, n, NULL) == TRI_ATTN_ERR_UNSUPPORTED);

    tri_proj_problem q;
    memset(&q, 0, sizeof q);
    q.rows = 64; q.batch = 1; q.cz = 128; q.H = 4; q.c = 32; q.eps = 1e-5f;
    CHECK(10, tri_proj_workspace_size(&q, &n) == TRI_ATTN_OK && n >= (size_t)64 * 128 * 4);
    CHECK(11, tri_proj_out_fwd(&q, fake, fake, (const float *)fake, fake, fake, n - 16, NULL) ==
                  TRI_ATTN_ERR_WORKSPACE);
    q.cz = 96;
    CHECK(12, tri_proj_workspace_size(&q, &n) == TRI_ATTN_ERR_UNSUPPORTED);
    q.cz = 128; q.reserved = 1;
    CHECK(13, tri_proj_workspace_size(&q, &n) == TRI_ATTN_ERR_INVALID_ARG);

    printf("c abi ok\n");
    return 0;
}
