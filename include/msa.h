/*
 * msa.h -- C ABI of libmsa: the long-context decode path of MiniMax Sparse
 * Attention (MSA) over an NVFP4 paged KV cache, on one NVIDIA B200 (sm_100a).
 *
 * Method source: the vLLM blog post "vLLM 為 MiniMax-M3.1-Flash 提供 Day-0
 * 支援" (hot.atechcom.net), cited as [post, "<section>"]:
 *   "MSA primer" -- the cache is split into 128-token blocks; an indexer
 *     scores every cached key with one index query per GQA group against one
 *     shared index-key head, max-pools the scores to one score per block;
 *     attention then runs exactly over the top 16 blocks, the most recent
 *     block always kept, so a query sees at most 2,048 keys.
 *   "What is new in the MiniMax-M3.1 architecture" -- NVFP4 cache for both
 *     the indexer and the attention path.
 *   "NVIDIA Blackwell optimized MSA kernels" -- FP8 queries; the NVFP4 cache
 *     is dequantised to FP8 (E4M3) inside the kernel and fed to FP8 MMA.
 *   "Quick start" (serving flags) -- block size 128, NVFP4 KV and NVFP4
 *     indexer cache dtypes.
 *
 * Shapes fixed by the model the post describes (compile-time constants):
 *   MSA_BLOCK_TOKENS = 128 tokens per block/page, MSA_TOPK = 16 blocks,
 *   MSA_KV_HEADS = 4 KV heads = 4 GQA groups = 4 index queries per token,
 *   MSA_Q_HEADS = 64 query heads (query head h reads KV head h / 16),
 *   MSA_HEAD_DIM = 128 for queries, keys, values and index keys.
 *
 * Conventions for every entry point:
 *   - All tensor pointers are DEVICE pointers to caller-owned memory; the
 *     library never allocates, frees or keeps a pointer after returning.
 *   - Every call is asynchronous on `stream` (NULL = legacy default stream).
 *   - Host-side argument checks run before any launch; a failed check returns
 *     an error code and launches nothing.  Besides NULL pointers, alignment,
 *     sizes and scales, they check that the first and the last byte of every
 *     buffer (sized from the arguments) is device memory of the current
 *     device, or managed memory: a pageable or pinned host buffer, another
 *     device's memory or an address CUDA does not know returns
 *     MSA_ERR_INVALID_ARG (MSA_ERR_WORKSPACE for the workspace) instead of
 *     faulting the GPU.  A buffer that ends inside another allocation is not
 *     detected.
 *   - Device-side checks (page ids, selected block ids, sequence lengths) never
 *     trap: a bad item is skipped and the first error code is recorded in the
 *     workspace; msa_get_last_error() reads it.
 *   - Every pointer must be 16-byte aligned.  Per-tensor scales must be
 *     finite and > 0.
 *
 * Cache layout (one layer; P = num_pages physical pages of 128 tokens):
 *   NVFP4 tensor = 4-bit E2M1 codes + one E4M3 scale byte per 16 contiguous
 *   elements + one fp32 scale per tensor.  Element d of a 128-vector lives
 *   in byte d/2 (even d: low nibble, odd d: high nibble); scale byte s
 *   covers elements 16s..16s+15.  Decoded value of an element:
 *       E4M3_rne_satfinite( e2m1(code) * e4m3(scale) ) * s_tensor
 *   idx_data  [P][128][64]     NVFP4 index-key codes        (idx_dtype NVFP4)
 *   idx_scale [P][128][8]      NVFP4 index-key block scales
 *   idx_data  [P][128][128]    E4M3 index keys, idx_scale NULL (idx_dtype FP8)
 *   (idx_dtype NVFP4_EXACT: the NVFP4 layout above, but the indexer scores
 *   the keys at their exact value e2m1(code) * e4m3(scale) * s_idx, without
 *   the E4M3 re-rounding -- the FP16 scoring of [post, "NVIDIA Rubin
 *   optimized MSA"]; K and V are always decoded as above.)
 *   k_data, v_data   [P][4][128][64]  NVFP4 codes  (page, kv head, token)
 *   k_scale, v_scale [P][4][128][8]   E4M3 block scales
 * Sequences: sequence b holds seq_lens[b] tokens, which INCLUDE its q_tokens
 *   new tokens; query token t sits at position pos = seq_lens[b]-q_tokens+t
 *   and sees every key j <= pos.  Logical block i of sequence b is physical
 *   page page_table[b*max_pages+i] (page b*max_pages+i if page_table NULL).
 * Queries: qi [B][T][4][128] E4M3 index queries (scale s_qi);
 *          q  [B][T][64][128] E4M3 attention queries (scale s_q).
 * Selection: sel [B][T][4][16] int32 logical block ids, ascending, -1 pad.
 * Output: out [B][T][64][128] bf16 (raw uint16 bits).
 */
#ifndef MSA_H
#define MSA_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

#if defined(__GNUC__)
#define MSA_API __attribute__((visibility("default")))
#else
#define MSA_API
#endif

#define MSA_BLOCK_TOKENS 128
#define MSA_TOPK 16
#define MSA_HEAD_DIM 128
#define MSA_KV_HEADS 4
#define MSA_Q_HEADS 64
#define MSA_MAX_BATCH 4096
#define MSA_MAX_PARTS 64        /* context parts of msa_indexer_score_part */

/* A cudaStream_t, declared without the CUDA headers. */
typedef struct CUstream_st* msa_stream_t;

typedef enum {
    MSA_OK = 0,
    MSA_ERR_INVALID_ARG = 1,    /* a host-side argument check failed            */
    MSA_ERR_UNSUPPORTED = 2,    /* valid request this build does not handle      */
    MSA_ERR_CUDA = 3,           /* a CUDA runtime call failed (launch, memset)   */
    MSA_ERR_DEVICE_BOUNDS = 4,  /* device check: page id / block id / length bad */
    MSA_ERR_TIMEOUT = 5,        /* device check: a bounded wait ran out          */
    MSA_ERR_WORKSPACE = 6       /* workspace NULL or smaller than required       */
} msa_status;

/* Index-key format and scoring arithmetic (msa_cache.idx_dtype):
 *   MSA_IDX_NVFP4        NVFP4 keys, re-rounded to E4M3, FP8 tensor-core MMA;
 *   MSA_IDX_FP8          E4M3 keys, FP8 MMA;
 *   MSA_IDX_NVFP4_EXACT  NVFP4 keys decoded exactly to FP16 and scored with
 *                        FP16 MMA against the index queries widened to FP16
 *                        (exact products, fp32 accumulation). */
enum { MSA_IDX_NVFP4 = 0, MSA_IDX_FP8 = 1, MSA_IDX_NVFP4_EXACT = 2 };

/* One layer's cache (device pointers, caller-owned). */
typedef struct {
    const uint8_t* idx_data;
    const uint8_t* idx_scale;   /* NULL for MSA_IDX_FP8, required otherwise */
    const uint8_t* k_data;
    const uint8_t* k_scale;
    const uint8_t* v_data;
    const uint8_t* v_scale;
    float s_idx, s_k, s_v;      /* per-tensor fp32 scales (> 0) */
    int32_t num_pages;          /* pages in each pool */
    int32_t idx_dtype;          /* MSA_IDX_NVFP4, MSA_IDX_FP8 or MSA_IDX_NVFP4_EXACT */
} msa_cache;

/* The batch of sequences of one decode step. */
typedef struct {
    const int32_t* page_table;  /* device [batch][max_pages], or NULL (contiguous) */
    const int32_t* seq_lens;    /* device [batch]; q_tokens <= len <= max_pages*128 */
    int32_t batch;              /* 1 .. MSA_MAX_BATCH */
    int32_t q_tokens;           /* query tokens per sequence, >= 1 */
    int32_t max_pages;          /* row length of page_table; upper bound on blocks */
} msa_seqs;

/* Sequences of the batch that share a cached prefix: [post, "AMD GPU
 * support", "NVFP4 MSA kernel"] dequantises a shared-prefix page once for
 * the requests that share it.  Group g is the sequences [seq_start[g],
 * seq_start[g+1]) (consecutive in the batch); the first prefix_blocks[g]
 * logical blocks of each of them are the same physical pages (equal page
 * table entries), and every key of those blocks is visible to every query of
 * the group (prefix_blocks[g]*128 <= seq_lens[b] - q_tokens).  Groups cover
 * the batch: seq_start[0] = 0, non-decreasing, seq_start[num_groups] = batch;
 * a sequence without a shared prefix is a group of one with prefix 0.
 * Arrays that break these rules are reported on the device
 * (MSA_ERR_DEVICE_BOUNDS) and give unspecified scores; they are clamped to
 * the batch and the page table, so no access leaves the buffers. */
typedef struct {
    const int32_t* seq_start;      /* device [num_groups + 1] */
    const int32_t* prefix_blocks;  /* device [num_groups] */
    int32_t num_groups;            /* 1 .. batch */
} msa_prefix_groups;

/* Bytes of device workspace the calls below need for `seqs` (error flags,
 * block scores, selection, attention partials).  The size depends on `seqs`
 * alone (not on the device), so it can be computed without a GPU.  The
 * workspace must be zeroed once (msa_workspace_init) before its first use and
 * may be reused by later calls on the same stream.  Returns 0 if seqs is
 * invalid (its pointers are not dereferenced).
 * When every (sequence, group) selects its blocks several times over
 * (q_tokens * 16 >= 4 * max_pages, as in prefill) and the rows fit in 1 GiB,
 * the size also holds the decode-once rows: every visible block's K and V
 * decoded to E4M3 once per step (32 KB per sequence, block and KV head), which
 * the attention then reads instead of decoding per (token, group) ([post,
 * "AMD GPU support", "NVFP4 MSA kernel"]: a page dequantised once for the
 * requests that read it).  A workspace smaller than this size but large
 * enough for the rest runs the same step without those rows; the results are
 * bit-identical. */
MSA_API size_t msa_workspace_size(const msa_seqs* seqs);

/* Zero the workspace's error flags (asynchronous on stream). */
MSA_API msa_status msa_workspace_init(void* ws, size_t ws_bytes, msa_stream_t stream);

/* Step (1)+(2) of [post, "MSA primer"]: indexer scores and the max-pool.
 *   token score s[b,t,g,j] = s_qi*s_idx * sum_d qi[b,t,g,d] * k_idx[b,j,d],
 *   block score S[b,t,g,i] = max over the keys j <= pos of block i.
 * token_scores: optional [B][T][4][max_pages*128] fp32 (NULL = skip); for
 *   every block i < ceil(len/128): the score for keys j <= pos, -inf for keys
 *   j > pos; entries of blocks i >= ceil(len/128) untouched.
 * block_scores: [B][T][4][max_pages] fp32; written for i < ceil(len/128);
 *   -inf where block i has no key visible to the query.
 * Index keys are NVFP4 or FP8, scored as cache->idx_dtype says. */
MSA_API msa_status msa_indexer_score(const msa_cache* cache, const msa_seqs* seqs,
                             const uint8_t* qi, float s_qi,
                             float* token_scores, float* block_scores,
                             void* ws, size_t ws_bytes, msa_stream_t stream);

/* msa_indexer_score restricted to one part of every sequence's context: the
 * context split of [post, "NVFP4 indexer DCP"], where each GPU scores all
 * four index heads over its share of the pages and the shares' results are
 * combined into one exact selection.  Part `part` of `nparts` of a sequence
 * with nblk = ceil(len/128) blocks is the logical blocks
 *     [floor(nblk*part/nparts), floor(nblk*(part+1)/nparts))
 * (the parts tile 0..nblk-1; a part may be empty).  Only those blocks are
 * read (so the page table entries and pages of other parts are never
 * touched) and only their entries of token_scores / block_scores are
 * written, with exactly the values msa_indexer_score writes for them; the
 * element-wise max of all parts' block_scores, each pre-filled with -inf,
 * is msa_indexer_score's block_scores.  Causal masking uses each block's
 * absolute position.  1 <= nparts <= MSA_MAX_PARTS, 0 <= part < nparts,
 * else MSA_ERR_INVALID_ARG; other arguments as msa_indexer_score. */
MSA_API msa_status msa_indexer_score_part(const msa_cache* cache, const msa_seqs* seqs,
                             const uint8_t* qi, float s_qi,
                             float* token_scores, float* block_scores,
                             int32_t part, int32_t nparts,
                             void* ws, size_t ws_bytes, msa_stream_t stream);

/* Step (3) of [post, "MSA primer"]: per (b, t, g) select the top 16 blocks
 * among the blocks visible to the query (0 .. pos/128), the latest block
 * always kept: the latest plus the 15 best other blocks ranked by (score
 * descending, block id ascending); all blocks when at most 16 are visible.
 * scores: block scores [B][T][4][max_pages] (is_token_level = 0) or token
 *   scores [B][T][4][max_pages*128] (is_token_level = 1, max-pooled first).
 * sel: [B][T][4][16] int32, ascending ids, -1 padding. */
MSA_API msa_status msa_block_maxpool_topk(const float* scores, int32_t is_token_level,
                                  const msa_seqs* seqs, int32_t* sel,
                                  void* ws, size_t ws_bytes, msa_stream_t stream);

/* Step (4) of [post, "MSA primer"] with the dequantisation of [post, "NVIDIA
 * Blackwell optimized MSA kernels"]: for every query head h of group g=h/16,
 * softmax over the keys j <= pos of the selected blocks of
 *   softmax_scale * s_q * s_k * (q_h . k_j),
 * output s_v * sum_j p_j v_j rounded to bf16.  K and V are NVFP4, decoded to
 * E4M3 in the kernel and contracted with FP8 MMA; the probabilities P enter
 * the P.V product as the sum of two E4M3 terms (P to about 2^-8 relative).
 * sel entries -1 are skipped; ids outside 0..pos/128 are a device error. */
MSA_API msa_status msa_sparse_attn_decode(const msa_cache* cache, const msa_seqs* seqs,
                                  const uint8_t* q, float s_q, const int32_t* sel,
                                  float softmax_scale, uint16_t* out,
                                  void* ws, size_t ws_bytes, msa_stream_t stream);

/* msa_indexer_score for a batch whose sequences share prefixes (`groups`,
 * which requires a page table): the same scores, but each shared-prefix
 * page is read and decoded for a tile of up to 128 index queries drawn from
 * all the sequences of its group (the tiles of one page run side by side,
 * so the page comes from HBM once and from L2 after that), instead of once
 * per sequence; the remaining blocks of each sequence are scored as by
 * msa_indexer_score.  [post, "AMD GPU support", "NVFP4 MSA kernel"]. */
MSA_API msa_status msa_indexer_score_grouped(const msa_cache* cache, const msa_seqs* seqs,
                             const msa_prefix_groups* groups,
                             const uint8_t* qi, float s_qi,
                             float* token_scores, float* block_scores,
                             void* ws, size_t ws_bytes, msa_stream_t stream);

/* The whole decode step: indexer -> max-pool -> top-16 -> sparse attention,
 * back to back on `stream` with intermediates in the workspace.
 * sel_out: optional [B][T][4][16] copy of the selection (NULL = skip). */
MSA_API msa_status msa_decode(const msa_cache* cache, const msa_seqs* seqs,
                      const uint8_t* qi, float s_qi, const uint8_t* q, float s_q,
                      float softmax_scale, uint16_t* out, int32_t* sel_out,
                      void* ws, size_t ws_bytes, msa_stream_t stream);

/* msa_decode with the indexer of msa_indexer_score_grouped (shared-prefix
 * pages decoded once per tile of the group's index queries); the selection
 * and the output are those of msa_decode. */
MSA_API msa_status msa_decode_grouped(const msa_cache* cache, const msa_seqs* seqs,
                      const msa_prefix_groups* groups,
                      const uint8_t* qi, float s_qi, const uint8_t* q, float s_q,
                      float softmax_scale, uint16_t* out, int32_t* sel_out,
                      void* ws, size_t ws_bytes, msa_stream_t stream);

/* Write the new tokens into the cache: for every sequence b, the q_tokens
 * tokens at positions seq_lens[b]-q_tokens .. seq_lens[b]-1 (the same
 * tokens msa_decode treats as the queries' own) are quantised and stored at
 * their page (page_table, or b*max_pages + block when it is NULL) and slot
 * ([post, "What is new in the MiniMax-M3.1 architecture"]: NVFP4 KV cache
 * for the indexer and the attention; [post, "QKV GEMM + norm + RoPE + KV
 * insert fusion"] names the insertion).
 *   k_new, v_new: device bf16 [B][T][4][128] (per KV head); idx_new: device
 *   bf16 [B][T][128] (the shared index-key head); all 16-byte aligned.
 *   NVFP4 rows: per 16 elements the scale byte is E4M3 (nearest-even,
 *   saturating) of amax/(6*s_t), each code the nearest E2M1 value of
 *   x/(scale*s_t) (ties to the even code, saturating at 6), s_t = the
 *   cache's s_k, s_v or s_idx; FP8 index keys are E4M3 of x/s_idx.
 * The cache buffers are written through the descriptor's pointers (they
 * must be writable device memory); nothing else in the cache changes.
 * Pages outside the pool or invalid lengths are reported in the workspace
 * (MSA_ERR_DEVICE_BOUNDS via msa_get_last_error) and those rows skipped. */
MSA_API msa_status msa_kv_insert(const msa_cache* cache, const msa_seqs* seqs,
                                 const uint16_t* k_new, const uint16_t* v_new,
                                 const uint16_t* idx_new, void* ws, size_t ws_bytes,
                                 msa_stream_t stream);

/* Synchronise `stream`, return the first device-side error recorded in the
 * workspace since the last call (MSA_OK if none) and clear it.
 * detail (optional) receives the offending value (page id, block id, ...). */
MSA_API msa_status msa_get_last_error(void* ws, msa_stream_t stream, int32_t* detail);

/* Debug/parity hook: decode every (scale byte, code) pair with the kernels'
 * own NVFP4 -> E4M3 path.  out: device [256][16] uint8, out[s*16+c] =
 * E4M3 byte of rne_satfinite(e2m1(c) * e4m3(s)). */
MSA_API msa_status msa_debug_nvfp4_table(uint8_t* out, msa_stream_t stream);

/* Size of the library-owned scratch used by msa_decode_static (16 MiB); every
 * GPU that loads the library holds it until the process exits. */
#define MSA_STATIC_WORKSPACE_BYTES (16u << 20)

/* msa_decode without a caller-provided workspace: the pages have no
 * counterpart for this entry point.  It is for callers that cannot allocate
 * device memory where they call it -- code that runs under another
 * framework's caching allocator it does not control, plugin or custom-op
 * interfaces whose execution path forbids device allocations, or hot serving
 * loops where a cudaMalloc would synchronise the device.  Inputs and outputs
 * are caller-owned as for msa_decode; the scratch is a fixed device array of
 * MSA_STATIC_WORKSPACE_BYTES inside the library, and nothing is allocated or
 * freed by this call.
 *   - Returns MSA_ERR_WORKSPACE when the step's workspace without the
 *     decode-once rows (see msa_workspace_size) is larger than
 *     MSA_STATIC_WORKSPACE_BYTES (the batch needs a caller workspace and
 *     msa_decode), MSA_ERR_INVALID_ARG / MSA_ERR_CUDA as msa_decode; the
 *     decode-once rows are used when they fit as well.
 *   - The first call on a device looks up the array's device address for
 *     that device (cudaGetSymbolAddress, with the device current); make that
 *     first call before any stream capture on the device.  The address is
 *     kept with the identity of the device's CUDA context; after a
 *     cudaDeviceReset the next call finds a new context and looks the
 *     address up again (that call, too, should come before any capture).
 *   - All calls on a device share the one array and it keeps the previous
 *     call's contents; each call clears what must start at zero.  Calls that
 *     overlap on the GPU (different streams, or different host threads
 *     without ordering) race on the array: serialise them.
 *   - Device-side bounds errors are recorded in the shared array, which the
 *     next call clears; this entry point does not report them. */
MSA_API msa_status msa_decode_static(const msa_cache* cache, const msa_seqs* seqs,
                                     const uint8_t* qi, float s_qi, const uint8_t* q, float s_q,
                                     float softmax_scale, uint16_t* out, int32_t* sel_out,
                                     msa_stream_t stream);

/* Static description of an error code. */
MSA_API const char* msa_status_string(msa_status status);

#ifdef __cplusplus
}
#endif

#endif /* MSA_H */
