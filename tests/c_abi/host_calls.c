/* A plain C99 consumer of the C ABI (include/pagedkv.h): host-only calls
 * (allocator, workspace queries, status strings, an empty decode batch), so
 * it runs without a GPU.  Exits 0 and prints "ok" when every check holds.
 *
 * The allocator part replays the aiknowledge.cn "2.2 PagedAttention 与 KV
 * Cache 分页管理" worked example (section 2.2.3): a 35-token sequence in
 * 16-token blocks mapped to physical blocks 7, 3, 9.
 */
#include <stdio.h>
#include <string.h>

#include "pagedkv.h"

static int failures = 0;
#define CHECK(cond)                                                   \
    do {                                                              \
        if (!(cond)) {                                                \
            fprintf(stderr, "check failed at line %d: %s\n", __LINE__, #cond); \
            failures++;                                               \
        }                                                             \
    } while (0)

int main(void) {
    int32_t order[16] = {7, 3, 9, 12, 0, 1, 2, 4, 5, 6, 8, 10, 11, 13, 14, 15};
    pkv_alloc* a = pkv_alloc_create(16, 16, order);
    CHECK(a != NULL);
    if (!a) return 1;

    /* 35 tokens: blocks 7, 3, 9; slots block * 16 + offset */
    int64_t slots[64];
    int32_t cow[2];
    int ncow = -1;
    CHECK(pkv_seq_add(a, 0) == PKV_OK);
    CHECK(pkv_seq_append_slots(a, 0, 35, slots, cow, 1, &ncow) == PKV_OK && ncow == 0);
    CHECK(slots[0] == 112 && slots[15] == 127 && slots[16] == 48 && slots[31] == 63 && slots[34] == 146);
    int32_t bt[8];
    int n = 0;
    int64_t len = 0;
    CHECK(pkv_seq_block_table(a, 0, bt, 8, &n, &len) == PKV_OK);
    CHECK(n == 3 && len == 35 && bt[0] == 7 && bt[1] == 3 && bt[2] == 9);

    /* filling block 9 takes nothing; token 48 takes the queue's front, 12 */
    CHECK(pkv_seq_append_slots(a, 0, 13, slots, cow, 1, &ncow) == PKV_OK && ncow == 0);
    CHECK(pkv_seq_append_slots(a, 0, 1, slots, cow, 1, &ncow) == PKV_OK && slots[0] == 12 * 16);

    /* a fork shares every block; the child's first write copies the partial last one */
    CHECK(pkv_seq_fork(a, 0, 1) == PKV_OK);
    CHECK(pkv_block_refcount(a, 12) == 2);
    CHECK(pkv_seq_append_slots(a, 1, 1, slots, cow, 1, &ncow) == PKV_OK && ncow == 1 && cow[0] == 12);
    CHECK(pkv_block_refcount(a, 12) == 1 && pkv_block_refcount(a, cow[1]) == 1);

    int free_blocks = 0, used_blocks = 0;
    int64_t fails = -1, copies = -1;
    CHECK(pkv_alloc_stats(a, &free_blocks, &used_blocks, &fails, &copies) == PKV_OK);
    CHECK(free_blocks + used_blocks == 16 && used_blocks == 5 && fails == 0 && copies == 1);

    /* exhaustion is all-or-nothing */
    CHECK(pkv_seq_append_slots(a, 0, 16 * 16, slots, cow, 1, &ncow) == PKV_ERR_NO_FREE_BLOCK);
    CHECK(strlen(pkv_last_error()) > 0);
    CHECK(pkv_seq_block_table(a, 0, bt, 8, &n, &len) == PKV_OK && n == 4 && len == 49);
    CHECK(pkv_seq_free(a, 1) == PKV_OK && pkv_seq_free(a, 0) == PKV_OK);
    CHECK(pkv_alloc_stats(a, &free_blocks, &used_blocks, &fails, &copies) == PKV_OK);
    CHECK(free_blocks == 16 && used_blocks == 0 && fails == 1);
    pkv_alloc_destroy(a);

    /* host queries and an empty batch (no launch) */
    CHECK(pkv_attention_workspace_bytes(4, 4, 64, 512, 0) == 0);
    /* partials (rows x partitions x (D + 2) floats), rounded up to 256 bytes, then 8 bytes per row */
    CHECK(pkv_attention_workspace_bytes(8, 64, 128, 100160, 512) ==
          ((size_t)8 * 64 * 196 * 130 * 4 + 255) / 256 * 256 + (size_t)8 * 64 * 8);
    CHECK(pkv_attention_partition_size(64, 32, 32, 128, 2048, 0) == 512);
    CHECK(strcmp(pkv_status_str(PKV_OK), "ok") == 0);
    CHECK(pkv_paged_attention_decode(NULL, NULL, NULL, NULL, NULL, 4, NULL, 0, 4, 4, 64, 16, 8, 0.0f, 0, NULL, 0,
                                     PKV_BF16, NULL) == PKV_OK);

    if (failures) return 1;
    printf("ok\n");
    return 0;
}
