/* Plain-C use of the library's C ABI (include/h3rr.h), host-only calls.
 * Built and run by tests/test_c_abi.py: the header must compile as C99 and
 * the exported symbols must link from C.  No call here reaches a GPU: only
 * host functions and argument checks that fail before any launch. */
#include <stdint.h>
#include <stdio.h>
#include <string.h>

#include "h3rr.h"

static int failures = 0;

static void expect(int cond, const char* what)
{
    if (!cond) {
        fprintf(stderr, "FAIL: %s\n", what);
        ++failures;
    }
}

int main(void)
{
    int64_t token_starts[7];
    int32_t head_starts[7];
    int64_t bounds[9] = {0, 3000, 9000, 10000, 17000, 20000, 26000, 30000, 32768};
    int64_t local_bounds[8 + 2 * 6 - 1];
    int32_t local_ids[8 + 6 - 1];
    int32_t offsets[7];
    int64_t chunk_tokens = 0, chunks = 0;
    h3_exec_info info;
    const void* null_ptrs[6] = {0};
    void* null_out[6] = {0};

    expect(h3_abi_version() == H3RR_ABI_VERSION, "abi version");
    expect(strcmp(h3_status_string(H3_OK), "ok") == 0, "status string");

    /* the head table of the partition contract: W=6 -> 10,10,9,9,9,9 */
    expect(h3_partition(32768, 56, 6, bounds, 8, token_starts, head_starts, local_bounds,
                        local_ids, offsets) == H3_OK, "partition");
    expect(head_starts[1] == 10 && head_starts[2] == 20 && head_starts[3] == 29 &&
           head_starts[6] == 56, "head starts");
    expect(token_starts[1] == 5462 && token_starts[6] == 32768, "token starts");
    expect(offsets[6] >= 8 && offsets[6] <= 8 + 6 - 1, "piece count");
    expect(local_bounds[0] == 0 && local_ids[0] == 0, "first piece");
    expect(h3_partition(5, 56, 6, NULL, 0, token_starts, head_starts, NULL, NULL, NULL) ==
           H3_ERR_EMPTY_PARTITION, "empty partition");

    expect(h3_staged_plan(250000, 4, 56, 128, 896000000, &chunk_tokens, &chunks) == H3_OK &&
           chunk_tokens == 62500 && chunks == 16, "staged plan");
    /* the long sequence over 4 ranks: one plane per launch at the pages'
     * window; over 2 ranks each plane moves in two token chunks */
    expect(h3_relayout_chunk_plan(250000, 4, 56, 128, 4, 896000000, &chunk_tokens, &chunks) ==
           H3_OK && chunk_tokens == 62500 && chunks == 4, "chunk plan, 4 ranks");
    expect(h3_relayout_chunk_plan(250000, 4, 56, 128, 2, 896000000, &chunk_tokens, &chunks) ==
           H3_OK && chunk_tokens == 62500 && chunks == 8, "chunk plan, 2 ranks");
    expect(h3_relayout_chunk_plan(250000, 4, 56, 128, 4, 14335, &chunk_tokens, &chunks) ==
           H3_ERR_WINDOW, "window below one token");
    /* token ranges over all planes: the same window holds 15,625 tokens of
     * all four planes of every rank, again 4 launches */
    {
        int32_t per_launch = 0;
        expect(h3_relayout_chunk_plan_ex(250000, 4, 56, 128, 4, 896000000, H3_LAUNCH_CHUNK_TOKENS,
                                         &chunk_tokens, &chunks, &per_launch) == H3_OK &&
                   chunk_tokens == 15625 && chunks == 4 && per_launch == 4,
               "token-range plan, 4 ranks");
        expect(h3_relayout_chunk_plan_ex(250000, 4, 56, 128, 4, 896000000, 0, &chunk_tokens, &chunks,
                                         &per_launch) == H3_OK &&
                   chunk_tokens == 62500 && chunks == 4 && per_launch == 1,
               "one-plane plan through _ex");
        expect(h3_relayout_chunk_plan_ex(250000, 4, 56, 128, 4, 4 * 14336 - 16, H3_LAUNCH_CHUNK_TOKENS,
                                         &chunk_tokens, &chunks, NULL) == H3_ERR_WINDOW,
               "window below one token of every plane");
    }

    /* argument checks fail before anything is launched */
    expect(h3_seq_to_head(NULL, NULL, 1000, 3, 56, 128, 6, 0, NULL, &info) == H3_ERR_INVALID_ARG &&
           info.launches == 0, "null pointer arrays");
    expect(h3_ragged_reduce_scatter(null_ptrs, NULL, null_out, 1000, 7168, 0, NULL, &info) ==
           H3_ERR_INVALID_ARG, "world 0");
    expect(h3_ragged_all_gather(null_ptrs, null_out, 1000, 7164, 6, NULL, &info) ==
           H3_ERR_MISALIGNED, "cols not a multiple of 8");
    expect(h3_seq_to_head_staged_noalloc(null_ptrs, null_out, 1000, 3, 56, 128, 6,
                                         H3RR_STATIC_WINDOW_BYTES + 16, NULL, &info) ==
           H3_ERR_UNSUPPORTED, "noalloc window beyond its array");

    /* one rank per GPU: rank out of range, NULL output, misaligned columns */
    {
        h3_launch_config cfg;
        h3_ipc_handle handle;
        void* mapped = NULL;
        void* fake_out = (void*)(uintptr_t)4096; /* never dereferenced: checks fail first */
        memset(&cfg, 0, sizeof(cfg));
        expect(h3_seq_to_head_rank(NULL, NULL, 1000, 3, 56, 128, 6, 0, 0, NULL, NULL, &info) ==
                   H3_ERR_INVALID_ARG && info.launches == 0, "rank call, null arrays");
        expect(h3_ragged_reduce_scatter_rank(null_ptrs, NULL, fake_out, 1000, 7168, 6, 6, NULL,
                                             NULL, &info) == H3_ERR_INVALID_ARG, "rank out of range");
        expect(h3_ragged_all_gather_rank(null_ptrs, fake_out, 1000, 7164, 6, 0, NULL, NULL, &info) ==
               H3_ERR_MISALIGNED, "rank call, cols not a multiple of 8");
        cfg.flags = H3_LAUNCH_SERIAL | 2;
        expect(h3_ragged_all_gather_rank(null_ptrs, fake_out, 1000, 7168, 6, 0, NULL, &cfg, &info) ==
               H3_ERR_INVALID_ARG, "unknown launch flag");
        expect(sizeof(h3_ipc_handle) == 80, "ipc record size");
        expect(h3_ipc_export(NULL, &handle) == H3_ERR_INVALID_ARG, "ipc export of NULL");
        expect(h3_ipc_open(NULL, &mapped) == H3_ERR_INVALID_ARG && mapped == NULL, "ipc open of NULL");
        expect(h3_ipc_close(NULL, &handle) == H3_ERR_INVALID_ARG, "ipc close of NULL");
    }

    if (failures == 0)
        printf("c abi ok\n");
    return failures == 0 ? 0 : 1;
}
