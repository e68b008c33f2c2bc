/* abi_from_c.c -- the boundary used from plain C99 (no CUDA headers, no C++):
 * include/pa.h compiles as C, the structs have the documented sizes, and the
 * host-only entry points behave as declared.  No GPU call is made: every
 * device entry point used here returns before anything is enqueued.
 * Prints the FNV-1a chained digests of tokens 0..47 (three blocks) as hex,
 * one per line, for the calling test to compare with its own restatement. */
#include <stdio.h>
#include <string.h>

#include "pa.h"

#define CHECK(c)                                                     \
    do {                                                             \
        if (!(c)) {                                                  \
            fprintf(stderr, "check failed, line %d: %s\n", __LINE__, #c); \
            return 1;                                                \
        }                                                            \
    } while (0)

int main(void)
{
    pa_cache_desc_t d;
    pa_cache_desc_t bad;
    pa_block_hash_t h[3];
    pa_prefix_cache_t *c;
    int32_t toks[48];
    int32_t ids[3] = {7, 8, 9};
    int32_t hit[3] = {-1, -1, -1};
    int64_t nb = -1;
    int i, j;

    CHECK(sizeof(pa_cache_desc_t) == 24);
    CHECK(sizeof(pa_attn_options_t) == 32 + 3 * sizeof(void *));
    CHECK(sizeof(pa_block_hash_t) == 32);
    CHECK(pa_abi_version() == 4);
    CHECK(strcmp(pa_status_string(PA_ERR_WORKSPACE_TOO_SMALL), "PA_ERR_WORKSPACE_TOO_SMALL") == 0);

    memset(&d, 0, sizeof d);
    d.num_blocks = 1024;
    d.num_kv_heads = 8;
    d.head_dim = 128;
    d.block_size = 16;
    d.layout = PA_LAYOUT_HND;
    CHECK(pa_workspace_size(4, 4, 32, &d, 1000) > 0);
    bad = d;
    bad.head_dim = 96;
    CHECK(pa_workspace_size(4, 4, 32, &bad, 1000) == 0);
    /* nothing to write: returns before any CUDA call */
    CHECK(pa_kv_write(NULL, NULL, 1024, NULL, 0, NULL, NULL, &d, NULL) == PA_OK);
    CHECK(pa_kv_write(NULL, NULL, 1024, NULL, 4, NULL, NULL, &d, NULL) == PA_ERR_INVALID_ARG);

    for (i = 0; i < 48; ++i)
        toks[i] = i;
    CHECK(pa_prefix_block_hashes(toks, 47, NULL, PA_HASH_FNV1A64, h, &nb) == PA_OK && nb == 2);
    CHECK(pa_prefix_block_hashes(toks, 48, NULL, PA_HASH_FNV1A64, h, &nb) == PA_OK && nb == 3);
    c = pa_prefix_cache_create();
    CHECK(c != NULL);
    CHECK(pa_prefix_cache_insert(c, h, ids, 2) == PA_OK);
    CHECK(pa_prefix_cache_size(c) == 2);
    CHECK(pa_prefix_cache_longest_hit(c, h, 3, hit) == 2 && hit[0] == 7 && hit[1] == 8);
    CHECK(pa_prefix_cache_remove_block(c, 7) == PA_OK);
    CHECK(pa_prefix_cache_longest_hit(c, h, 3, hit) == 0);
    pa_prefix_cache_destroy(c);

    for (i = 0; i < 3; ++i) {
        for (j = 0; j < 32; ++j)
            printf("%02x", h[i].bytes[j]);
        printf("\n");
    }
    return 0;
}
