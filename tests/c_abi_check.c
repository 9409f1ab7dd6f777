/* The C-ABI used from plain C99 (no C++, no CUDA headers): the host-only
 * entry points on the tiny bucket (planner, shards, rank buckets, work table,
 * row-wise layout, error path).  Built and run by tests/test_c_abi.py,
 * which checks the printed numbers against the Python binding. */
#include <stdio.h>
#include <stdlib.h>

#include "dbuf.h"

int main(void) {
    /* W[512,256] in 16-row blocks, bias[512] and LayerNorm[256] as one block each. */
    dbuf_tensor_desc t[3] = {{512, 256, 16, 0}, {512, 1, 512, 0}, {256, 1, 256, 0}};
    dbuf_plan_t* plan = NULL;
    if (dbuf_plan(t, 3, 4, 16, 0, &plan) != DBUF_OK) {
        printf("plan failed: %s\n", dbuf_last_error());
        return 1;
    }
    int64_t slice = 0, bucket = 0, padding = 0, n_blocks = 0, offsets[3];
    if (dbuf_plan_info(plan, &slice, &bucket, &padding, &n_blocks, offsets) != DBUF_OK) return 2;
    printf("slice=%lld bucket=%lld padding=%lld n_blocks=%lld offsets=%lld,%lld,%lld\n", (long long)slice,
           (long long)bucket, (long long)padding, (long long)n_blocks, (long long)offsets[0], (long long)offsets[1],
           (long long)offsets[2]);
    int64_t n = 0;
    if (dbuf_work_table(plan, NULL, 0, &n) != DBUF_OK) return 3;
    dbuf_work_item* items = (dbuf_work_item*)malloc(sizeof(dbuf_work_item) * (size_t)n);
    if (!items || dbuf_work_table(plan, items, n, &n) != DBUF_OK) return 4;
    int64_t covered = 0;
    for (int64_t i = 0; i < n; ++i) covered += items[i].n_elems;
    printf("entries=%lld covered=%lld required_bytes=%zu\n", (long long)n, (long long)covered,
           dbuf_required_bytes(plan));
    free(items);
    /* A bad descriptor is refused with a message, not a crash. */
    dbuf_tensor_desc bad = {0, 4, 1, 0};
    dbuf_plan_t* p2 = NULL;
    const dbuf_status st = dbuf_plan(&bad, 1, 2, 16, 0, &p2);
    printf("bad=%d msg_nonempty=%d\n", (int)st, dbuf_last_error()[0] != 0);
    int64_t chunk = 0, q[3], off[3];
    if (dbuf_rowwise_layout(t, 3, 4, &chunk, q, off) != DBUF_OK) return 5;
    printf("rowwise chunk=%lld q=%lld,%lld,%lld\n", (long long)chunk, (long long)q[0], (long long)q[1], (long long)q[2]);
    /* The RaggedShard rows of each tensor per rank, and the last rank's
     * slice as a bucket of its own. */
    dbuf_shard_rows shards[3 * 4];
    if (dbuf_plan_shards(plan, shards) != DBUF_OK) return 6;
    printf("shards_w=%lld,%lld,%lld,%lld\n", (long long)shards[0].row_end, (long long)shards[1].row_end,
           (long long)shards[2].row_end, (long long)shards[3].row_end);
    dbuf_plan_t* last = NULL;
    int64_t first_block = -1, r_padding = 0, r_blocks = 0;
    if (dbuf_plan_rank(plan, 3, &last, &first_block) != DBUF_OK) return 7;
    if (dbuf_plan_info(last, NULL, NULL, &r_padding, &r_blocks, NULL) != DBUF_OK) return 8;
    printf("rank3 first_block=%lld padding=%lld n_blocks=%lld\n", (long long)first_block, (long long)r_padding,
           (long long)r_blocks);
    int32_t dn = -1, dm = -1, rn = -1, rm = -1;
    if (dbuf_plan_dims(plan, &dn, &dm) != DBUF_OK || dbuf_plan_dims(last, &rn, &rm) != DBUF_OK) return 9;
    printf("dims=%d,%d rank3_dims=%d,%d\n", (int)dn, (int)dm, (int)rn, (int)rm);
    dbuf_plan_t* none = NULL;
    printf("rank_bad=%d null_out=%d\n", (int)dbuf_plan_rank(plan, 4, &none, NULL), none == NULL);
    dbuf_plan_free(last);
    dbuf_plan_free(plan);
    dbuf_plan_free(NULL);
    return 0;
}
