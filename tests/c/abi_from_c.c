/*
 * abi_from_c.c -- the library used from plain C99 through its headers
 * alone (no CUDA or C++ header), on the host-only paths: status strings,
 * the size queries, argument checks that refuse a call before any device
 * work, and the block manager.  Exit code 0 when every check holds, else
 * the number of the first failed check.
 */
#include <stdio.h>
#include <string.h>

#include "pa.h"
#include "pa_block_manager.h"
#include "pa_selftest.h"

#define CHECK(n, cond)                                  \
    do {                                                \
        if (!(cond)) {                                  \
            fprintf(stderr, "check %d failed\n", (n));  \
            return (n);                                 \
        }                                               \
    } while (0)

int main(void)
{
    CHECK(1, strcmp(pa_status_string(PA_OK), "PA_OK") == 0);
    CHECK(2, strcmp(pa_status_string(PA_ERR_UNSUPPORTED), "PA_ERR_UNSUPPORTED") == 0);
    CHECK(3, pa_version() != NULL && pa_version()[0] != '\0');

    /* contexts that fit one partition need no workspace */
    CHECK(4, pa_paged_decode_workspace_size(4, 2, 2, 64, 16, 40, 0) == 0);

    /* refused before any device work: null pointers, an unsupported head_dim */
    CHECK(5, pa_paged_decode(NULL, NULL, NULL, NULL, NULL, NULL, 4, 2, 2, 64, 16, 4, 64, 40,
                             0.125f, 0, NULL, 0, PA_DTYPE_F16, NULL, NULL) == PA_ERR_INVALID_ARG);
    CHECK(6, pa_paged_decode(NULL, NULL, NULL, NULL, NULL, NULL, 4, 2, 2, 96, 16, 4, 64, 40,
                             0.125f, 0, NULL, 0, PA_DTYPE_F16, NULL, NULL) == PA_ERR_UNSUPPORTED);
    CHECK(7, pa_reshape_and_cache_int8(NULL, NULL, NULL, NULL, NULL, 1, 2, 64, 16, 8,
                                       PA_DTYPE_F16, 0.5f, 0.5f, NULL, NULL) == PA_ERR_INVALID_ARG);
    CHECK(8, pa_swap_blocks(NULL, NULL, NULL, NULL, NULL, 1, 2, 64, 16, 8, 8, PA_DTYPE_INT8,
                            NULL, NULL) == PA_ERR_INVALID_ARG);

    /* the test entry points refuse a missing status word or a limit of 0 */
    CHECK(19, pa_selftest_bounded_wait(NULL, NULL, 1000, 1, NULL) == PA_ERR_INVALID_ARG);
    CHECK(20, pa_selftest_decode_abort(NULL, NULL, NULL, NULL, NULL, NULL, 4, 2, 2, 64, 16, 4, 64,
                                       40, 0.125f, 0, NULL, 0, PA_DTYPE_F16, PA_DTYPE_F16, 0, NULL,
                                       NULL) == PA_ERR_INVALID_ARG);

    /* the block manager: allocation, copy-on-write, swap bookkeeping */
    pa_block_manager* bm = pa_bm_create(8, 4, 0);
    CHECK(9, bm != NULL);
    int64_t slots[6];
    int32_t cached = -1;
    CHECK(10, pa_bm_add_sequence(bm, 7, NULL, 6, 0, slots, &cached) == PA_BM_OK && cached == 0);
    CHECK(11, pa_bm_fork(bm, 7, 8) == PA_BM_OK);
    int64_t slot, cow[2];
    int32_t ncow = -1;
    CHECK(12, pa_bm_append_slots(bm, 8, NULL, 1, &slot, cow, 1, &ncow) == PA_BM_OK && ncow == 1);
    CHECK(13, pa_bm_attach_host_pool(bm, 4) == PA_BM_OK);
    int64_t ids[2] = {7, 8}, pairs[8];
    int32_t npairs = -1;
    CHECK(14, pa_bm_swap_out(bm, ids, 2, pairs, 4, &npairs) == PA_BM_OK && npairs == 3);
    CHECK(15, pa_bm_is_swapped(bm, 8) == 1 && pa_bm_num_free_blocks(bm) == 8);
    CHECK(16, pa_bm_swap_in(bm, ids, 2, pairs, 4, &npairs) == PA_BM_OK && npairs == 3);
    pa_bm_stats_t st;
    CHECK(17, pa_bm_stats(bm, &st) == PA_BM_OK && st.used_blocks == 3 && st.stored_tokens == 6 + 3);
    CHECK(18, pa_bm_check(bm) == 0);
    pa_bm_destroy(bm);
    printf("abi from C ok\n");
    return 0;
}
