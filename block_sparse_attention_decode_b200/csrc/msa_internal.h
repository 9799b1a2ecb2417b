// msa_internal.h -- kernel argument blocks and launchers shared between the
// C-ABI layer (msa_api.cu) and the kernel files.  Not part of the ABI.
#pragma once

#include "msa.h"
#include <cstddef>
#include <cstdint>
#include <utility>
#include <cuda.h>
#include <cuda_runtime.h>

#include "msa_device.cuh"

namespace msa {

// Launch `kernel` with programmatic stream serialisation: it may start while
// the previous kernel on the stream is finishing (its launch and prologue
// overlap that kernel's last CTAs).  The kernel calls grid_dependency_wait()
// before it touches global memory the previous work writes or reads.
template <typename... KArgs, typename... Args>
cudaError_t launch_dependent(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                             cudaStream_t st, Args&&... args) {
  cudaLaunchConfig_t cfg{};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  return cudaLaunchKernelEx(&cfg, kernel, std::forward<Args>(args)...);
}

constexpr int kIdxThreads = 14 * 32;    // 8 decoders, 4 epilogue warps, producer, MMA warp
// Indexer arithmetic: NVFP4 keys re-rounded to E4M3 (FP8 MMA), E4M3 keys, or
// NVFP4 keys decoded exactly to FP16 (FP16 MMA).
enum : int { kIdxNvfp4 = 0, kIdxFp8 = 1, kIdxF16 = 2 };

struct IdxArgs {
  CUtensorMap tmap_idx;        // rows of idx_data: 64-byte rows (64B swizzle) or 128 (128B swizzle)
  CUtensorMap tmap_qi;         // rows of qi (128 bytes, 128B swizzle), boxes of one query tile
  const uint8_t* idx_data;     // NVFP4 codes [P][128][64] or FP8 keys [P][128][128]
  const uint8_t* idx_scale;    // [P][128][8] (NVFP4 keys only)
  const int32_t* page_table;   // [B][max_pages] or null
  const int32_t* seq_lens;     // [B]
  const uint8_t* qi;           // [B][T][4][128] E4M3
  float* token_scores;         // [B][T][4][max_pages*128] or null
  float* block_scores;         // [B][T][4][max_pages]
  Flags* flags;
  int* work;                   // [2] in the workspace header: next item, CTAs done (0 on entry)
  float score_scale;           // s_qi * s_idx
  int B, T, max_pages, num_pages;
  int part, nparts;            // score blocks [nblk*part/nparts, nblk*(part+1)/nparts) of each sequence
  // Sequences sharing a cached prefix (null grp_start: none): group g is the
  // sequences [grp_start[g], grp_start[g+1]), whose first grp_prefix[g]
  // logical blocks are the same physical pages.  shared = 1 scores only those
  // prefix blocks, once per group, against the index queries of all the
  // group's sequences; shared = 0 scores every sequence's blocks from its
  // group's prefix on.
  const int32_t* grp_start;
  const int32_t* grp_prefix;
  int ngroups;
  int shared;
  // 64-row tiles of at most 32 query rows (E4M3 query modes): tile row r sits
  // at MMA row 16 (r / 8) + r % 8, so that each TMEM lane quarter holds eight
  // rows and all four epilogue warps share the work; tmap_qi has 8-row boxes
  int spread;
};

size_t indexer_smem_bytes(int mode, int batch, int T);
int idx_tile_queries(int T);   // index queries per tile (the MMA's M side): 64 or 128
bool idx_spread_rows(int T, int mode, int shared);   // the `spread` placement above
cudaError_t launch_indexer(const IdxArgs& a, int mode, cudaStream_t st);

// Grid of a persistent kernel on the current device: the device's SMs times
// the CTAs of `kernel` resident per SM for `threads` threads, `smem` bytes of
// dynamic shared memory and `tmem_cols` of the 512 TMEM columns per CTA
// (0 = none).  Raises the kernel's dynamic shared-memory limit to `smem` on
// the current device first (once per device, kernel and size; thread-safe).
// Any CUDA error is returned, never replaced by a default.
cudaError_t persistent_grid(const void* kernel, int threads, size_t smem, int tmem_cols, int* grid);

// Workspace bytes of a step without the decode-once rows (0 for invalid
// sequences): what a fixed-size workspace must hold at least.
size_t workspace_base_size(const msa_seqs* s);

// Encode a tensor map over `rows` rows of `row_bytes` (64 or 128) bytes with
// 128-row boxes and the matching shared-memory swizzle.  False on failure.
bool encode_row_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes,
                     uint32_t box_rows = kBlock);

// Top-k over block scores of every (b, t, g) row.
cudaError_t launch_topk(const float* block_scores, const int32_t* seq_lens, int B, int T,
                        int max_pages, int32_t* sel, Flags* flags, cudaStream_t st);
// Max-pool token scores [B][T][4][max_pages*128] into block scores.
cudaError_t launch_maxpool(const float* token_scores, const int32_t* seq_lens, int B, int T,
                           int max_pages, float* block_scores, Flags* flags, cudaStream_t st);

constexpr int kAttThreads = 14 * 32;    // 4 decoders, 8 softmax warps, producer, MMA warp
constexpr int kAttStages = 2;            // raw K/V blocks in flight per CTA
constexpr int kAttWorkOffset = 72;       // int[2] in the workspace header (see kWorkOffset)
constexpr int kPartialFloats = kHpg * kDim + 2 * kHpg;   // O[16][128], m[16], l[16]

struct AttnArgs {
  CUtensorMap tmap_k, tmap_v;  // K / V code rows [P*4*128][64 B], 64-byte swizzle, 128-row boxes
  // Decode-once mode (dkv = 1): every visible block of every sequence is
  // decoded to E4M3 once, into kd / vd = [B][max_pages][4][128 keys][128 B]
  // in the workspace, and the attention loads those rows (128-byte swizzle)
  // instead of decoding per item
  CUtensorMap tmap_kd, tmap_vd;
  uint8_t *kd, *vd;
  int dkv;
  CUtensorMap tmap_q;          // query rows [B*T*64][128 B], 128-byte swizzle, 16-row boxes
  const uint8_t *k_data, *k_scale, *v_data, *v_scale;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const uint8_t* q;            // [B][T][64][128] E4M3
  const int32_t* sel;          // [B][T][4][16]
  uint16_t* out;               // [B][T][64][128] bf16
  float* partials;             // [units][splits][kPartialFloats]
  int* counters;               // [units]
  Flags* flags;
  int* work;                   // [2] in the workspace header: next item, CTAs done (0 on entry)
  float logit_scale_log2;      // softmax_scale * s_q * s_k * log2(e)
  float out_scale;             // s_v
  int B, T, max_pages, num_pages, splits;
};

size_t attn_smem_bytes();
int attn_splits(long long rows, int num_sms);
cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st);

// Quantise the new tokens into the cache (msa_kv_insert).
struct InsArgs {
  uint8_t *idx_data, *idx_scale, *k_data, *k_scale, *v_data, *v_scale;
  const int32_t* page_table;
  const int32_t* seq_lens;
  const uint16_t *k_new, *v_new;   // bf16 [B][T][4][128]
  const uint16_t* idx_new;         // bf16 [B][T][128]
  Flags* flags;
  float s_idx, s_k, s_v;
  int B, T, max_pages, num_pages, idx_fp8;
};
cudaError_t launch_insert(const InsArgs& a, cudaStream_t st);

// The kernels' NVFP4 -> E4M3 table for all (scale, code) pairs.
cudaError_t launch_nvfp4_table(uint8_t* out, cudaStream_t st);

}  // namespace msa
