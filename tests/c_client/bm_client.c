/*
 * A plain C client of the library's C ABI (no Python): drives the host-side
 * block manager through the glossary "PagedAttention" worked example (section
 * "How paging works": 40 tokens, blocks of 16, free list 41, 7, 19, 2, 33 ->
 * block table 41, 7, 19) and the copy-on-write rule of its section "Sharing
 * blocks across sequences", checks the copy pairs with the host pair check,
 * caches a prompt's full blocks and shares them with a second request, swaps
 * both sequences to a second manager, packs shared-prefix units from host
 * tables, checks workspace sizes and status strings.  Prints "ok"
 * and exits 0 when every check holds.
 */
#include <stdio.h>
#include <stdlib.h>

#include "pagedkv.h"

#define CHECK(c)                                                 \
    do {                                                         \
        if (!(c)) {                                              \
            fprintf(stderr, "check failed: %s (line %d)\n", #c, __LINE__); \
            return 1;                                            \
        }                                                        \
    } while (0)

int main(void) {
    CHECK(pkv_version() >= 100);
    CHECK(pkv_status_string(PKV_OK) != NULL);

    /* the worked example: a 64-block pool whose free list starts 41, 7, 19, 2, 33 */
    int32_t order[64];
    int n = 0;
    const int32_t head[5] = {41, 7, 19, 2, 33};
    for (int i = 0; i < 5; ++i) order[n++] = head[i];
    for (int b = 0; b < 64; ++b) {
        int used = 0;
        for (int i = 0; i < 5; ++i) used |= head[i] == b;
        if (!used) order[n++] = b;
    }
    pkv_block_manager* m = pkv_bm_create(64, 16, order);
    CHECK(m != NULL);
    CHECK(pkv_bm_add_sequence(m, 0) == PKV_OK);
    int64_t id = 0, slot = 0, pairs[2];
    int np = 0;
    for (int t = 0; t < 40; ++t) {
        CHECK(pkv_bm_append_slots(m, &id, 1, &slot, pairs, 1, &np) == PKV_OK);
        CHECK(np == 0);
    }
    int32_t table[4], len = 0;
    CHECK(pkv_bm_block_tables(m, &id, 1, table, 4, -1, &len) == PKV_OK);
    CHECK(table[0] == 41 && table[1] == 7 && table[2] == 19 && table[3] == -1 && len == 40);
    CHECK(3 * 16 - len == 8);                        /* unused slots under paging */
    CHECK(slot == 19 * 16 + 39 % 16);                /* the 40th token's slot */

    /* fork, then the child's first token: the shared partial block is copied for the writer */
    CHECK(pkv_bm_fork(m, 0, 1) == PKV_OK);
    CHECK(pkv_bm_ref_count(m, 19) == 2);
    int64_t child = 1;
    CHECK(pkv_bm_append_slots(m, &child, 1, &slot, pairs, 1, &np) == PKV_OK);
    CHECK(np == 1 && pairs[0] == 19 && pairs[1] == 2);  /* the next free block in FIFO order */
    CHECK(pkv_check_block_pairs(pairs, np, 64, 64, 1) == PKV_OK);
    {
        const int64_t onto_source[4] = {19, 2, 2, 5};      /* block 2 written, then read */
        const int64_t repeated[4] = {19, 2, 7, 2};
        const int64_t outside[2] = {19, 64};
        CHECK(pkv_check_block_pairs(onto_source, 2, 64, 64, 1) == PKV_ERR_INVALID_ARG);
        CHECK(pkv_check_block_pairs(onto_source, 2, 64, 64, 0) == PKV_OK);
        CHECK(pkv_check_block_pairs(repeated, 2, 64, 64, 0) == PKV_ERR_INVALID_ARG);
        CHECK(pkv_check_block_pairs(outside, 1, 64, 64, 0) == PKV_ERR_INVALID_ARG);
    }
    CHECK(pkv_bm_ref_count(m, 19) == 1 && pkv_bm_ref_count(m, 41) == 2);
    /* the parent is now the only holder of block 19: it writes in place */
    CHECK(pkv_bm_append_slots(m, &id, 1, &slot, pairs, 1, &np) == PKV_OK);
    CHECK(np == 0 && slot == 19 * 16 + 40 % 16);

    CHECK(pkv_bm_free_sequence(m, 0) == PKV_OK);
    CHECK(pkv_bm_free_sequence(m, 1) == PKV_OK);
    CHECK(pkv_bm_num_free(m) == 64);
    CHECK(pkv_bm_add_sequence(m, 1) == PKV_OK);
    CHECK(pkv_bm_add_sequence(m, 1) == PKV_ERR_INVALID_ARG);
    CHECK(pkv_bm_free_sequence(m, 1) == PKV_OK);

    /* prefix caching: a 40-token prompt cached, then a second request with the same first 35
     * tokens shares the two full blocks they cover (32 tokens) */
    int32_t prompt[40];
    for (int t = 0; t < 40; ++t) prompt[t] = 1000 + 3 * t;
    int64_t a = 10, b = 11;
    CHECK(pkv_bm_add_sequence(m, a) == PKV_OK);
    for (int t = 0; t < 40; ++t) CHECK(pkv_bm_append_slots(m, &a, 1, &slot, pairs, 1, &np) == PKV_OK);
    CHECK(pkv_bm_cache_sequence(m, a, prompt, 40) == PKV_OK);
    CHECK(pkv_bm_num_cached(m) == 2);                /* two full blocks; the partial one is not */
    int hit = -1;
    CHECK(pkv_bm_add_sequence_cached(m, b, prompt, 35, &hit) == PKV_OK);
    CHECK(hit == 32 && pkv_bm_sequence_length(m, b) == 32);
    int32_t ta[3], tb[3];
    CHECK(pkv_bm_block_tables(m, &a, 1, ta, 3, -1, NULL) == PKV_OK);
    CHECK(pkv_bm_block_tables(m, &b, 1, tb, 3, -1, NULL) == PKV_OK);
    CHECK(ta[0] == tb[0] && ta[1] == tb[1] && tb[2] == -1 && pkv_bm_ref_count(m, ta[0]) == 2);

    /* swap both sequences to a second manager: one destination block per distinct source block */
    pkv_block_manager* h = pkv_bm_create(16, 16, NULL);
    CHECK(h != NULL);
    const int64_t both[2] = {10, 11};
    int64_t sp[2 * 6];
    int nsp = 0;
    CHECK(pkv_bm_swap(m, h, both, 2, sp, 6, &nsp) == PKV_OK);
    CHECK(nsp == 3);                                 /* a's three blocks; b's two are among them */
    CHECK(pkv_check_block_pairs(sp, nsp, 64, 16, 0) == PKV_OK);
    CHECK(pkv_bm_sequence_length(m, a) == -1 && pkv_bm_sequence_length(h, a) == 40);
    CHECK(pkv_bm_sequence_length(h, b) == 32 && pkv_bm_num_free(h) == 13);
    CHECK(pkv_bm_block_tables(h, &b, 1, tb, 3, -1, NULL) == PKV_OK);
    CHECK(pkv_bm_ref_count(h, tb[0]) == 2 && pkv_bm_ref_count(h, tb[1]) == 2);
    pkv_bm_destroy(h);
    pkv_bm_destroy(m);

    /* shared-prefix units from host tables: three sequences share their first two full blocks,
     * a fourth shares nothing; units of at most two members */
    {
        const int32_t tables[4 * 3] = {5, 6, 7, 5, 6, 9, 5, 6, 10, 1, 2, -1};
        const int32_t lens[4] = {40, 40, 35, 20};
        int32_t spl[4], us[4 * 2], ul[4];
        int nu = -1, mp = -1;
        CHECK(pkv_find_shared_prefixes(tables, lens, 4, 3, 16, 2, spl, us, ul, 4, &nu, &mp) == PKV_OK);
        CHECK(nu == 2 && mp == 32 && ul[0] == 32 && ul[1] == 32);
        CHECK(spl[0] == 32 && spl[1] == 32 && spl[2] == 32 && spl[3] == 0);
        CHECK(us[0] == 0 && us[1] == 1 && us[2] == 2 && us[3] == -1);
        CHECK(pkv_find_shared_prefixes(tables, lens, 4, 3, 16, 2, spl, us, ul, 1, &nu, &mp) ==
              PKV_ERR_INVALID_ARG);                     /* two units needed, room for one */
    }

    /* workspace sizes: none when every sequence fits one partition (an explicit 128-token
     * partition, or the automatic rule, which splits a small batch down to 4 blocks but not
     * below); the FP8 prefill's widened pools (2 x 6 blocks x 2 heads x 16 x 64 x 2 bytes) plus
     * a 256-byte-aligned table */
    CHECK(pkv_decode_workspace_bytes(1, 8, 8, 128, PKV_F16, 16, 100, 128) == 0);
    CHECK(pkv_decode_workspace_bytes(1, 8, 8, 128, PKV_F16, 16, 60, 0) == 0);
    CHECK(pkv_decode_workspace_bytes(1, 8, 8, 128, PKV_F16, 16, 100, 0) > 0);
    CHECK(pkv_decode_workspace_bytes(1, 8, 8, 128, PKV_F16, 16, 100, 16) > 0);
    CHECK(pkv_prefill_fp8_workspace_bytes(2, 3, 2, 64, 16) == 2 * 24576 + 256);
    CHECK(pkv_prefill_fp8_workspace_bytes(0, 3, 2, 64, 16) == 0);
    printf("ok\n");
    return 0;
}
