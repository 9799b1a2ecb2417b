/* The C ABI used from C, with only include/msa.h: prints the layout of the
 * two descriptor structs (compared by the test with the Python binding's
 * mirrors) and checks calls that the host rejects before any device work.
 * No device memory is touched: FAKE is an aligned address never read. */
#include <stddef.h>
#include <stdint.h>
#include <stdio.h>

#include "msa.h"

#define CHECK(c)                                                           \
    do {                                                                   \
        if (!(c)) {                                                        \
            fprintf(stderr, "FAIL line %d: %s\n", __LINE__, #c);           \
            return 1;                                                      \
        }                                                                  \
    } while (0)

int main(void)
{
    void* const FAKE = (void*)(uintptr_t)(1u << 20);
    msa_seqs s = {NULL, (const int32_t*)FAKE, 2, 1, 8};
    msa_cache c = {(const uint8_t*)FAKE, (const uint8_t*)FAKE, (const uint8_t*)FAKE,
                   (const uint8_t*)FAKE, (const uint8_t*)FAKE, (const uint8_t*)FAKE,
                   1.0f, 1.0f, 1.0f, 16, MSA_IDX_NVFP4};
    uint16_t* out = (uint16_t*)FAKE;
    const uint8_t* q = (const uint8_t*)FAKE;
    size_t big = (size_t)1 << 40;

    printf("msa_cache %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu %zu\n", sizeof(msa_cache),
           offsetof(msa_cache, idx_data), offsetof(msa_cache, idx_scale),
           offsetof(msa_cache, k_data), offsetof(msa_cache, k_scale),
           offsetof(msa_cache, v_data), offsetof(msa_cache, v_scale),
           offsetof(msa_cache, s_idx), offsetof(msa_cache, s_k), offsetof(msa_cache, s_v),
           offsetof(msa_cache, num_pages), offsetof(msa_cache, idx_dtype));
    printf("msa_seqs %zu %zu %zu %zu %zu %zu\n", sizeof(msa_seqs),
           offsetof(msa_seqs, page_table), offsetof(msa_seqs, seq_lens),
           offsetof(msa_seqs, batch), offsetof(msa_seqs, q_tokens),
           offsetof(msa_seqs, max_pages));
    printf("msa_prefix_groups %zu %zu %zu %zu\n", sizeof(msa_prefix_groups),
           offsetof(msa_prefix_groups, seq_start), offsetof(msa_prefix_groups, prefix_blocks),
           offsetof(msa_prefix_groups, num_groups));

    CHECK(msa_workspace_size(&s) > 0);
    s.batch = 0;
    CHECK(msa_workspace_size(&s) == 0);
    s.batch = 2;

    CHECK(msa_decode(NULL, &s, q, 1.0f, q, 1.0f, 0.1f, out, NULL, FAKE, big, NULL) ==
          MSA_ERR_INVALID_ARG);
    CHECK(msa_decode(&c, &s, q, 1.0f, q, 1.0f, 0.1f, out, NULL, NULL, big, NULL) ==
          MSA_ERR_WORKSPACE);
    c.idx_dtype = 7;
    CHECK(msa_decode(&c, &s, q, 1.0f, q, 1.0f, 0.1f, out, NULL, FAKE, big, NULL) ==
          MSA_ERR_INVALID_ARG);
    c.idx_dtype = MSA_IDX_NVFP4_EXACT;
    c.idx_scale = NULL;                       /* required for NVFP4 index keys */
    CHECK(msa_decode(&c, &s, q, 1.0f, q, 1.0f, 0.1f, out, NULL, FAKE, big, NULL) ==
          MSA_ERR_INVALID_ARG);
    c.idx_dtype = MSA_IDX_NVFP4;
    c.idx_scale = (const uint8_t*)FAKE;
    CHECK(msa_indexer_score_part(&c, &s, q, 1.0f, NULL, (float*)FAKE, 0, 0, FAKE, big, NULL) ==
          MSA_ERR_INVALID_ARG);
    CHECK(msa_indexer_score_part(&c, &s, q, 1.0f, NULL, (float*)FAKE, 3, 3, FAKE, big, NULL) ==
          MSA_ERR_INVALID_ARG);
    CHECK(msa_indexer_score_part(&c, &s, q, 1.0f, NULL, (float*)FAKE, 0, MSA_MAX_PARTS + 1, FAKE,
                                 big, NULL) == MSA_ERR_INVALID_ARG);
    CHECK(msa_kv_insert(&c, &s, NULL, (const uint16_t*)FAKE, (const uint16_t*)FAKE, FAKE, big,
                        NULL) == MSA_ERR_INVALID_ARG);
    {   /* prefix groups: present, 1..batch groups, and a page table */
        msa_prefix_groups g = {(const int32_t*)FAKE, (const int32_t*)FAKE, 1};
        CHECK(msa_indexer_score_grouped(&c, &s, NULL, q, 1.0f, NULL, (float*)FAKE, FAKE, big, NULL) ==
              MSA_ERR_INVALID_ARG);
        CHECK(msa_indexer_score_grouped(&c, &s, &g, q, 1.0f, NULL, (float*)FAKE, FAKE, big, NULL) ==
              MSA_ERR_INVALID_ARG);   /* s.page_table is NULL */
        s.page_table = (const int32_t*)FAKE;
        g.num_groups = 3;             /* more groups than sequences */
        CHECK(msa_decode_grouped(&c, &s, &g, q, 1.0f, q, 1.0f, 0.1f, out, NULL, FAKE, big, NULL) ==
              MSA_ERR_INVALID_ARG);
        g.num_groups = 0;
        CHECK(msa_decode_grouped(&c, &s, &g, q, 1.0f, q, 1.0f, 0.1f, out, NULL, FAKE, big, NULL) ==
              MSA_ERR_INVALID_ARG);
        s.page_table = NULL;
    }
    CHECK(msa_status_string(MSA_OK) != NULL && msa_status_string(MSA_ERR_TIMEOUT) != NULL);
    puts("ok");
    return 0;
}
