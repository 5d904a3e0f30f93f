/*
 * The libpa boundary used from plain C (C11, no C++ and no CUDA headers): both headers
 * compile on their own, every declared entry point links, and the calls that need no
 * GPU behave as documented -- the version, the status strings, a block-manager step
 * (allocate, fork, copy-on-write append, tables), and refusals that return before any
 * launch.  Prints "ok" and exits 0, or prints the failed check and exits 1.
 */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "pa.h"
#include "pa_block_manager.h"

#define CHECK(cond)                                                     \
    do {                                                                \
        if (!(cond)) {                                                  \
            printf("FAIL line %d: %s\n", __LINE__, #cond);              \
            return 1;                                                   \
        }                                                               \
    } while (0)

typedef void (*any_fn)(void);

int main(void) {
    /* every entry point of both headers, by address */
    const any_fn fns[] = {
        (any_fn)pa_kv_write, (any_fn)pa_copy_blocks, (any_fn)pa_swap_blocks,
        (any_fn)pa_decode, (any_fn)pa_decode_append, (any_fn)pa_decode_cow,
        (any_fn)pa_decode_planned, (any_fn)pa_decode_planned_units,
        (any_fn)pa_decode_workspace_bytes,
        (any_fn)pa_decode_partition_tokens, (any_fn)pa_decode_static_scratch,
        (any_fn)pa_prefill, (any_fn)pa_get_device_error, (any_fn)pa_status_str,
        (any_fn)pa_version, (any_fn)pa_bm_create, (any_fn)pa_bm_destroy,
        (any_fn)pa_bm_set_sliding_window, (any_fn)pa_bm_blocks_needed,
        (any_fn)pa_bm_num_free_blocks, (any_fn)pa_bm_usage_ratio, (any_fn)pa_bm_can_allocate,
        (any_fn)pa_bm_allocate, (any_fn)pa_bm_fork, (any_fn)pa_bm_free,
        (any_fn)pa_bm_append_slots, (any_fn)pa_bm_append_slots_cow, (any_fn)pa_bm_slot, (any_fn)pa_bm_seq_len,
        (any_fn)pa_bm_block_refcount, (any_fn)pa_bm_set_cpu_pool,
        (any_fn)pa_bm_num_free_cpu_blocks, (any_fn)pa_bm_is_swapped, (any_fn)pa_bm_swap_out,
        (any_fn)pa_bm_swap_in, (any_fn)pa_bm_block_tables};
    for (size_t i = 0; i < sizeof fns / sizeof fns[0]; ++i) CHECK(fns[i] != NULL);

    CHECK(pa_version() == 201);
    CHECK(strcmp(pa_status_str(PA_OK), "ok") == 0);
    CHECK(strcmp(pa_status_str(PA_ERR_HOST_ALLOC), "host memory allocation failed") == 0);

    /* a manager step: a 20-token prompt at block size 8 (3 blocks), forked; the
     * next token of each goes into the shared, partially filled last block */
    pa_block_manager *bm = pa_bm_create(10, 8);
    CHECK(bm != NULL);
    CHECK(pa_bm_blocks_needed(20, 8) == 3);
    CHECK(pa_bm_allocate(bm, 1, 20) == PA_OK);
    CHECK(pa_bm_fork(bm, 1, 2) == PA_OK);
    CHECK(pa_bm_num_free_blocks(bm) == 7);
    const int64_t ids[2] = {1, 2};
    int64_t slots[2], pairs[4];
    int npairs = -1;
    CHECK(pa_bm_append_slots(bm, ids, 2, slots, pairs, 2, &npairs) == PA_OK);
    CHECK(npairs == 1);                     /* the first writer gets a private copy */
    int32_t tables[2 * 4], lens[2];
    CHECK(pa_bm_block_tables(bm, ids, 2, tables, 4, lens) == PA_OK);
    CHECK(lens[0] == 21 && lens[1] == 21);
    CHECK(tables[0] == tables[4] && tables[1] == tables[5]); /* shared full blocks */
    CHECK(tables[2] != tables[6]);                            /* diverged last block */
    CHECK(pairs[1] == tables[2] && pairs[0] == tables[6]);    /* copy of the shared one */
    CHECK(slots[0] == (int64_t)tables[2] * 8 + 4 && slots[1] == (int64_t)tables[6] * 8 + 4);
    CHECK(tables[3] == -1 && tables[7] == -1);
    CHECK(pa_bm_allocate(bm, 3, 1000) == PA_ERR_NO_FREE_BLOCK);
    /* the same step with the copy reported per sequence, for pa_decode_cow */
    CHECK(pa_bm_fork(bm, 1, 4) == PA_OK);
    const int64_t ids2[2] = {4, 1};
    int32_t cow[2 * 3];
    int ncopies = -1;
    CHECK(pa_bm_append_slots_cow(bm, ids2, 2, slots, cow, &ncopies) == PA_OK);
    CHECK(ncopies == 1);                    /* sequence 4 copies the block it shared */
    CHECK(cow[0] == tables[2] && cow[1] == 2 && cow[2] == 5);  /* 21 tokens: 5 rows of block 2 */
    CHECK(cow[3] == -1 && cow[4] == 0 && cow[5] == 0);
    CHECK(slots[1] == (int64_t)tables[2] * 8 + 5);           /* sequence 1 keeps its block */
    pa_bm_destroy(bm);

    /* the plan of a planned launch, host-side: 3 contexts at 256-token partitions in a
     * 4-partition grid (12 rows) need 1 + 3 + 1 = 5 units; full partitions first, then the
     * last ones by decreasing length: (1,0) (1,1) then (1,2: 188 tokens) (0,0: 5) (2,0: 0) */
    const int32_t plan_lens[3] = {5, 700, 0};
    uint32_t plan[16];
    CHECK(pa_decode_planned_units(plan_lens, 3, 8, 2, 128, 16, 64, 1000, 0, 256, plan, 16) == 5);
    CHECK(plan[0] == ((1u << 16) | (0u << 8) | 3u) && plan[1] == ((1u << 16) | (1u << 8) | 3u));
    CHECK(plan[2] == ((1u << 16) | (2u << 8) | 3u) && plan[3] == ((0u << 16) | 1u));
    CHECK(plan[4] == ((2u << 16) | 1u));
    CHECK(pa_decode_planned_units(plan_lens, 3, 8, 2, 128, 16, 64, 1000, 300, 256, plan, 16) == 0);
    CHECK(pa_decode_planned_units(NULL, 3, 8, 2, 128, 16, 64, 1000, 0, 256, plan, 16) == -1);

    /* refusals before any launch (no GPU is touched) */
    char buf[64];
    CHECK(pa_decode(buf, buf, buf, buf, (const int32_t *)buf, (const int32_t *)buf, 1, 8, 2, 96,
                    16, 10, 4, 0.1f, 0, 0, 0, NULL, 0, PA_BF16, NULL) == PA_ERR_UNSUPPORTED);
    CHECK(pa_decode(buf, buf, buf, buf, (const int32_t *)buf, (const int32_t *)buf, 1, 7, 2, 128,
                    16, 10, 4, 0.1f, 0, 0, 0, NULL, 0, PA_BF16, NULL) == PA_ERR_INVALID_ARG);
    CHECK(pa_kv_write(NULL, NULL, NULL, 0, 2, 128, 256, 256, NULL, NULL, 10, 16, PA_BF16, NULL) ==
          PA_OK); /* nothing to write */
    CHECK(pa_prefill(buf, buf, buf, buf, (const int32_t *)buf, (const int32_t *)buf,
                     (const int32_t *)buf, 1, 4, 8, 2, 128, 16, 10, 4, -1.0f, 0, PA_BF16,
                     NULL) == PA_ERR_INVALID_ARG); /* scale must be positive */
    printf("ok\n");
    return 0;
}
