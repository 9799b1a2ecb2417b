// msa_api.cu -- the C ABI declared in include/msa.h: argument checks, the
// workspace layout, the work planner and the kernel launches.
#include <algorithm>
#include <cmath>
#include <cstring>
#include <mutex>

#include "msa.h"
#include "msa_internal.h"

using namespace msa;

namespace {

constexpr size_t kAlign = 256;
constexpr size_t align_up(size_t x) { return (x + kAlign - 1) / kAlign * kAlign; }

// SM count the attention's split heuristic is planned for (B200: 148 SMs).
// The workspace layout depends on it, so it is a constant of the library
// rather than a property queried from whatever device is current: the size
// msa_workspace_size reports is then the same on every machine.  The
// persistent grids themselves use the device's real SM count.
constexpr int kPlanSms = 148;

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool good_scale(float s) { return std::isfinite(s) && s > 0.f; }

// Workspace layout (byte offsets).
struct Layout {
  size_t flags, bscores, sel, counters, partials, dkv, total_base, total;
  int splits;
  bool dkv_ok;     // the batch qualifies for the decode-once attention
  bool use_dkv;    // ... and the caller's workspace holds its rows
  size_t used() const { return use_dkv ? total : total_base; }   // bytes the call touches
};

// Decode-once attention: when every (sequence, group) selects each of its
// blocks several times over (T x 16 >= 4 x max_pages, as in prefill), all
// visible blocks are decoded to E4M3 once into the workspace (32 KB per
// (sequence, block, KV head)) and the attention reads them instead of
// decoding per (token, group); the scratch is capped at 1 GiB.
constexpr unsigned long long kDkvMaxBytes = 1ull << 30;

bool seqs_ok(const msa_seqs* s) {
  if (!s || !s->seq_lens) return false;
  if (!aligned16(s->seq_lens) || (s->page_table && !aligned16(s->page_table))) return false;
  if (s->batch < 1 || s->batch > MSA_MAX_BATCH || s->q_tokens < 1 || s->max_pages < 1) return false;
  if ((long long)s->max_pages * MSA_BLOCK_TOKENS < s->q_tokens) return false;
  if ((long long)s->max_pages * MSA_BLOCK_TOKENS > 0x7FFFFFFFLL) return false;
  const long long rows = (long long)s->batch * s->q_tokens * MSA_KV_HEADS;
  return rows <= 0x7FFFFFFFLL / MSA_TOPK;
}

Layout layout_for(const msa_seqs* s) {
  Layout L{};
  const long long rows = (long long)s->batch * s->q_tokens * kG;
  L.splits = attn_splits(rows, kPlanSms);
  size_t off = 0;
  L.flags = off;    off += align_up(sizeof(Flags));
  L.bscores = off;  off += align_up((size_t)rows * s->max_pages * sizeof(float));
  L.sel = off;      off += align_up((size_t)rows * kTopk * sizeof(int32_t));
  L.counters = off; off += align_up((size_t)rows * sizeof(int));
  L.partials = off;
  if (L.splits > 1) off += align_up((size_t)rows * L.splits * kPartialFloats * sizeof(float));
  L.total_base = off;
  const unsigned long long dkv_bytes = 2ull * s->batch * s->max_pages * kG * kBlock * kDim;
  L.dkv_ok = (long long)s->q_tokens * kTopk >= 4LL * s->max_pages && dkv_bytes <= kDkvMaxBytes;
  L.dkv = off;
  if (L.dkv_ok) off += align_up((size_t)dkv_bytes);
  L.total = off;
  L.use_dkv = false;
  return L;
}

msa_status check_cache(const msa_cache* c, bool need_index, bool need_kv) {
  if (!c) return MSA_ERR_INVALID_ARG;
  if (c->num_pages < 1) return MSA_ERR_INVALID_ARG;
  if (need_index) {
    if (c->idx_dtype != MSA_IDX_NVFP4 && c->idx_dtype != MSA_IDX_FP8 &&
        c->idx_dtype != MSA_IDX_NVFP4_EXACT)
      return MSA_ERR_INVALID_ARG;
    if (!c->idx_data || !aligned16(c->idx_data)) return MSA_ERR_INVALID_ARG;
    if (c->idx_dtype != MSA_IDX_FP8 && (!c->idx_scale || !aligned16(c->idx_scale)))
      return MSA_ERR_INVALID_ARG;
    if (!good_scale(c->s_idx)) return MSA_ERR_INVALID_ARG;
  }
  if (need_kv) {
    const uint8_t* p[4] = {c->k_data, c->k_scale, c->v_data, c->v_scale};
    for (const uint8_t* x : p)
      if (!x || !aligned16(x)) return MSA_ERR_INVALID_ARG;
    if (!good_scale(c->s_k) || !good_scale(c->s_v)) return MSA_ERR_INVALID_ARG;
  }
  return MSA_OK;
}

// The decode-once rows are used when the workspace holds them (the size
// msa_workspace_size reports); a workspace of the base size runs the same
// step with the attention decoding per item.
msa_status check_ws(const msa_seqs* s, void* ws, size_t ws_bytes, Layout* L) {
  *L = layout_for(s);
  if (!ws || !aligned16(ws) || ws_bytes < L->total_base) return MSA_ERR_WORKSPACE;
  L->use_dkv = L->dkv_ok && ws_bytes >= L->total;
  return MSA_OK;
}

// Memory check before any launch: the first and the last byte of
// [p, p + bytes) must be device memory of the current device (or managed
// memory).  Pageable or pinned host memory, another device's memory and
// addresses CUDA does not know are rejected with `bad`, so that a wrong
// pointer from a C caller returns an error instead of faulting the GPU.
// A buffer that ends inside another allocation is not detected.  NULL
// pointers pass (whether a pointer may be NULL is checked before).
msa_status check_buf(const void* p, size_t bytes, msa_status bad = MSA_ERR_INVALID_ARG) {
  if (p == nullptr || bytes == 0) return MSA_OK;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) { cudaGetLastError(); return MSA_ERR_CUDA; }
  const uint8_t* ends[2] = {static_cast<const uint8_t*>(p), static_cast<const uint8_t*>(p) + bytes - 1};
  for (const uint8_t* x : ends) {
    cudaPointerAttributes at{};
    const cudaError_t e = cudaPointerGetAttributes(&at, x);
    if (e == cudaErrorInvalidValue) { cudaGetLastError(); return bad; }
    if (e != cudaSuccess) { cudaGetLastError(); return MSA_ERR_CUDA; }
    if (at.type == cudaMemoryTypeManaged) continue;
    if (at.type != cudaMemoryTypeDevice || at.device != dev) return bad;
  }
  return MSA_OK;
}

// The cache pools and the sequence descriptors, sized by num_pages / batch.
msa_status check_cache_mem(const msa_cache* c, bool need_index, bool need_kv) {
  const size_t P = (size_t)c->num_pages;
  msa_status st;
  if (need_index) {
    const size_t row = c->idx_dtype == MSA_IDX_FP8 ? MSA_HEAD_DIM : MSA_HEAD_DIM / 2;
    if ((st = check_buf(c->idx_data, P * MSA_BLOCK_TOKENS * row)) != MSA_OK) return st;
    if (c->idx_dtype != MSA_IDX_FP8 &&
        (st = check_buf(c->idx_scale, P * MSA_BLOCK_TOKENS * 8)) != MSA_OK)
      return st;
  }
  if (need_kv) {
    const size_t codes = P * MSA_KV_HEADS * MSA_BLOCK_TOKENS * (MSA_HEAD_DIM / 2);
    const size_t scales = P * MSA_KV_HEADS * MSA_BLOCK_TOKENS * 8;
    if ((st = check_buf(c->k_data, codes)) != MSA_OK || (st = check_buf(c->v_data, codes)) != MSA_OK ||
        (st = check_buf(c->k_scale, scales)) != MSA_OK || (st = check_buf(c->v_scale, scales)) != MSA_OK)
      return st;
  }
  return MSA_OK;
}

msa_status check_seqs_mem(const msa_seqs* s) {
  msa_status st = check_buf(s->seq_lens, (size_t)s->batch * 4);
  if (st != MSA_OK) return st;
  return check_buf(s->page_table, (size_t)s->batch * s->max_pages * 4);
}

// Prefix groups: present, 1 .. batch groups, and a page table to share pages.
msa_status check_groups(const msa_prefix_groups* g, const msa_seqs* s) {
  if (!g || !g->seq_start || !g->prefix_blocks) return MSA_ERR_INVALID_ARG;
  if (!aligned16(g->seq_start) || !aligned16(g->prefix_blocks)) return MSA_ERR_INVALID_ARG;
  if (g->num_groups < 1 || g->num_groups > s->batch) return MSA_ERR_INVALID_ARG;
  if (!s->page_table) return MSA_ERR_INVALID_ARG;
  return MSA_OK;
}

msa_status check_groups_mem(const msa_prefix_groups* g) {
  msa_status st = check_buf(g->seq_start, ((size_t)g->num_groups + 1) * 4);
  if (st != MSA_OK) return st;
  return check_buf(g->prefix_blocks, (size_t)g->num_groups * 4);
}

// Rows (sequence, token) of the step and the per-row byte counts of the
// query, output and selection buffers.
size_t n_tok(const msa_seqs* s) { return (size_t)s->batch * s->q_tokens; }
constexpr size_t kQiBytes = MSA_KV_HEADS * MSA_HEAD_DIM;            // per token
constexpr size_t kQBytes = MSA_Q_HEADS * MSA_HEAD_DIM;              // per token
constexpr size_t kOutBytes = MSA_Q_HEADS * MSA_HEAD_DIM * 2;        // per token
constexpr size_t kSelBytes = MSA_KV_HEADS * MSA_TOPK * 4;           // per token

template <typename T>
T* at(void* ws, size_t off) { return reinterpret_cast<T*>(static_cast<uint8_t*>(ws) + off); }

msa_status cuda_status(cudaError_t e) { return e == cudaSuccess ? MSA_OK : MSA_ERR_CUDA; }

msa_status run_indexer(const msa_cache* c, const msa_seqs* s, const uint8_t* qi, float s_qi,
                       float* token_scores, float* block_scores, void* ws, const Layout& L,
                       cudaStream_t st, int part = 0, int nparts = 1,
                       const msa_prefix_groups* groups = nullptr, int shared = 0) {
  IdxArgs a{};
  if (groups != nullptr) {
    a.grp_start = groups->seq_start;
    a.grp_prefix = groups->prefix_blocks;
    a.ngroups = groups->num_groups;
    a.shared = shared;
  }
  const bool fp8 = c->idx_dtype == MSA_IDX_FP8;
  if (!encode_row_tmap(&a.tmap_idx, c->idx_data, (uint64_t)c->num_pages * MSA_BLOCK_TOKENS,
                       fp8 ? MSA_HEAD_DIM : MSA_HEAD_DIM / 2))
    return MSA_ERR_CUDA;
  const int mode = fp8 ? kIdxFp8 : (c->idx_dtype == MSA_IDX_NVFP4_EXACT ? kIdxF16 : kIdxNvfp4);
  // the query tiles: 64 rows when a sequence has at most 64 index queries,
  // else (and for shared prefixes, whose tiles span sequences) 128; loaded
  // in boxes of 8 rows when they are spread over the four lane quarters
  a.spread = idx_spread_rows(s->q_tokens, mode, shared) ? 1 : 0;
  const int tile = a.spread ? 8 : (shared || idx_tile_queries(s->q_tokens) == 128) ? 128 : 64;
  if (!encode_row_tmap(&a.tmap_qi, qi, (uint64_t)s->batch * s->q_tokens * MSA_KV_HEADS, MSA_HEAD_DIM,
                       tile))
    return MSA_ERR_CUDA;
  a.idx_data = c->idx_data;
  a.idx_scale = c->idx_scale;
  a.page_table = s->page_table;
  a.seq_lens = s->seq_lens;
  a.qi = qi;
  a.token_scores = token_scores;
  a.block_scores = block_scores;
  a.flags = at<Flags>(ws, L.flags);
  a.work = at<int>(ws, L.flags + kWorkOffset);
  a.score_scale = s_qi * c->s_idx;
  a.B = s->batch;
  a.T = s->q_tokens;
  a.max_pages = s->max_pages;
  a.num_pages = c->num_pages;
  a.part = part;
  a.nparts = nparts;
  return cuda_status(launch_indexer(a, mode, st));
}

msa_status run_attn(const msa_cache* c, const msa_seqs* s, const uint8_t* q, float s_q,
                    const int32_t* sel, float softmax_scale, uint16_t* out, void* ws,
                    const Layout& L, cudaStream_t st) {
  const long long rows = (long long)s->batch * s->q_tokens * kG;
  if (L.splits > 1) {
    cudaError_t e = cudaMemsetAsync(at<int>(ws, L.counters), 0, (size_t)rows * sizeof(int), st);
    if (e != cudaSuccess) return MSA_ERR_CUDA;
  }
  // TMA row coordinates are 32-bit: (page * 4 + group) * 128 must fit
  if ((long long)c->num_pages * MSA_KV_HEADS * MSA_BLOCK_TOKENS > 0x7FFFFFFFLL) return MSA_ERR_UNSUPPORTED;
  AttnArgs a{};
  const uint64_t kv_rows = (uint64_t)c->num_pages * MSA_KV_HEADS * MSA_BLOCK_TOKENS;
  if (!encode_row_tmap(&a.tmap_k, c->k_data, kv_rows, MSA_HEAD_DIM / 2) ||
      !encode_row_tmap(&a.tmap_v, c->v_data, kv_rows, MSA_HEAD_DIM / 2) ||
      !encode_row_tmap(&a.tmap_q, q, (uint64_t)rows * (MSA_Q_HEADS / MSA_KV_HEADS), MSA_HEAD_DIM,
                       MSA_Q_HEADS / MSA_KV_HEADS))
    return MSA_ERR_CUDA;
  if (L.use_dkv) {
    const uint64_t drows = (uint64_t)s->batch * s->max_pages * MSA_KV_HEADS * MSA_BLOCK_TOKENS;
    a.kd = at<uint8_t>(ws, L.dkv);
    a.vd = a.kd + drows * MSA_HEAD_DIM;
    if (!encode_row_tmap(&a.tmap_kd, a.kd, drows, MSA_HEAD_DIM) ||
        !encode_row_tmap(&a.tmap_vd, a.vd, drows, MSA_HEAD_DIM))
      return MSA_ERR_CUDA;
    a.dkv = 1;
  }
  a.k_data = c->k_data;
  a.k_scale = c->k_scale;
  a.v_data = c->v_data;
  a.v_scale = c->v_scale;
  a.page_table = s->page_table;
  a.seq_lens = s->seq_lens;
  a.q = q;
  a.sel = sel;
  a.out = out;
  a.partials = at<float>(ws, L.partials);
  a.counters = at<int>(ws, L.counters);
  a.flags = at<Flags>(ws, L.flags);
  a.work = at<int>(ws, L.flags + kAttWorkOffset);
  a.logit_scale_log2 = (float)((double)softmax_scale * s_q * c->s_k * 1.4426950408889634);
  a.out_scale = c->s_v;
  a.B = s->batch;
  a.T = s->q_tokens;
  a.max_pages = s->max_pages;
  a.num_pages = c->num_pages;
  a.splits = L.splits;
  return cuda_status(launch_attn(a, st));
}

}  // namespace

namespace msa {

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

bool encode_row_tmap(CUtensorMap* map, const void* base, uint64_t rows, uint32_t row_bytes,
                     uint32_t box_rows) {
  static EncodeTiledFn fn = nullptr;
  if (fn == nullptr) {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) != cudaSuccess ||
        q != cudaDriverEntryPointSuccess || p == nullptr) {
      cudaGetLastError();
      return false;
    }
    fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  if ((row_bytes != 64 && row_bytes != 128) || box_rows < 1 || box_rows > 256) return false;
  const cuuint64_t dims[2] = {row_bytes, rows};
  const cuuint64_t strides[1] = {row_bytes};
  const cuuint32_t box[2] = {row_bytes, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  const CUtensorMapSwizzle sw = row_bytes == 64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B;
  return fn(map, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, sw, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

namespace {

// CTAs of a kernel resident per SM (registers, shared memory, threads, TMEM).
cudaError_t ctas_per_sm(const void* kernel, int dev, int threads, size_t smem, int tmem_cols,
                        int* n_out) {
  int smem_sm = 0, regs_sm = 0, max_threads = 0;
  cudaFuncAttributes fa{};
  cudaError_t e;
  if ((e = cudaFuncGetAttributes(&fa, kernel)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&smem_sm, cudaDevAttrMaxSharedMemoryPerMultiprocessor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&regs_sm, cudaDevAttrMaxRegistersPerMultiprocessor, dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&max_threads, cudaDevAttrMaxThreadsPerMultiProcessor, dev)) != cudaSuccess)
    return e;
  const int warps = (threads + 31) / 32;
  const int regs_warp = ((fa.numRegs * 32 + 255) / 256) * 256;      // allocation granularity
  int n = regs_warp > 0 ? regs_sm / (regs_warp * warps) : max_threads / (warps * 32);
  const size_t per_cta_smem = smem + fa.sharedSizeBytes + 1024;      // 1 KB reserved per CTA
  n = (int)std::min<long long>(n, (long long)(smem_sm / per_cta_smem));
  n = std::min(n, max_threads / (warps * 32));
  if (tmem_cols > 0) n = std::min(n, 512 / tmem_cols);
  if (n < 1) return cudaErrorInvalidConfiguration;
  *n_out = n;
  return cudaSuccess;
}

// Per (kernel, device): the dynamic shared-memory limit set so far (only
// ever raised: a smaller launch after a larger one keeps the larger limit)
// and the grid computed for the last size seen.
struct GridEntry {
  const void* kernel;
  int dev;
  size_t smem_limit;
  size_t smem;
  int grid;
};
std::mutex g_grid_mu;
GridEntry g_grid[64];
int g_grid_n = 0;

}  // namespace

size_t workspace_base_size(const msa_seqs* s) { return seqs_ok(s) ? layout_for(s).total_base : 0; }

cudaError_t persistent_grid(const void* kernel, int threads, size_t smem, int tmem_cols, int* grid) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  std::lock_guard<std::mutex> lock(g_grid_mu);
  GridEntry* ent = nullptr;
  for (int i = 0; i < g_grid_n; ++i)
    if (g_grid[i].kernel == kernel && g_grid[i].dev == dev) ent = &g_grid[i];
  if (ent != nullptr && ent->smem == smem && ent->smem_limit >= smem) {
    *grid = ent->grid;
    return cudaSuccess;
  }
  if (ent == nullptr || ent->smem_limit < smem) {
    // with the table full (more kernels x devices than it holds), the limit
    // goes straight to the device maximum so that no later call lowers it
    int limit = (int)smem;
    if (ent == nullptr && g_grid_n == (int)(sizeof(g_grid) / sizeof(g_grid[0])) &&
        (e = cudaDeviceGetAttribute(&limit, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
      return e;
    if ((e = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, limit)) !=
        cudaSuccess)
      return e;
  }
  int sms = 0, per_sm = 0;
  if ((e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev)) != cudaSuccess) return e;
  if ((e = ctas_per_sm(kernel, dev, threads, smem, tmem_cols, &per_sm)) != cudaSuccess) return e;
  *grid = sms * per_sm;
  if (ent == nullptr && g_grid_n < (int)(sizeof(g_grid) / sizeof(g_grid[0]))) {
    ent = &g_grid[g_grid_n++];
    ent->kernel = kernel;
    ent->dev = dev;
    ent->smem_limit = 0;
  }
  if (ent != nullptr) {
    ent->smem_limit = std::max(ent->smem_limit, smem);
    ent->smem = smem;
    ent->grid = *grid;
  }
  return cudaSuccess;
}

}  // namespace msa

extern "C" {

size_t msa_workspace_size(const msa_seqs* seqs) {
  if (!seqs_ok(seqs)) return 0;
  return layout_for(seqs).total;
}

msa_status msa_workspace_init(void* ws, size_t ws_bytes, msa_stream_t stream) {
  if (!ws || ws_bytes < sizeof(Flags)) return MSA_ERR_WORKSPACE;
  const msa_status st = check_buf(ws, sizeof(Flags), MSA_ERR_WORKSPACE);
  if (st != MSA_OK) return st;
  return cuda_status(cudaMemsetAsync(ws, 0, align_up(sizeof(Flags)) <= ws_bytes ? align_up(sizeof(Flags)) : ws_bytes,
                                     (cudaStream_t)stream));
}

msa_status msa_indexer_score(const msa_cache* cache, const msa_seqs* seqs, const uint8_t* qi,
                             float s_qi, float* token_scores, float* block_scores, void* ws,
                             size_t ws_bytes, msa_stream_t stream) {
  return msa_indexer_score_part(cache, seqs, qi, s_qi, token_scores, block_scores, 0, 1, ws,
                                ws_bytes, stream);
}

msa_status msa_indexer_score_part(const msa_cache* cache, const msa_seqs* seqs, const uint8_t* qi,
                                  float s_qi, float* token_scores, float* block_scores,
                                  int32_t part, int32_t nparts, void* ws, size_t ws_bytes,
                                  msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  if (nparts < 1 || nparts > MSA_MAX_PARTS || part < 0 || part >= nparts) return MSA_ERR_INVALID_ARG;
  msa_status st = check_cache(cache, true, false);
  if (st != MSA_OK) return st;
  if (!qi || !aligned16(qi) || !block_scores || !aligned16(block_scores) || !good_scale(s_qi))
    return MSA_ERR_INVALID_ARG;
  if (token_scores && !aligned16(token_scores)) return MSA_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(seqs, ws, ws_bytes, &L)) != MSA_OK) return st;
  const size_t nt = n_tok(seqs), bs_bytes = nt * MSA_KV_HEADS * seqs->max_pages * 4;
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK ||
      (st = check_cache_mem(cache, true, false)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_buf(qi, nt * kQiBytes)) != MSA_OK || (st = check_buf(block_scores, bs_bytes)) != MSA_OK ||
      (st = check_buf(token_scores, bs_bytes * MSA_BLOCK_TOKENS)) != MSA_OK)
    return st;
  return run_indexer(cache, seqs, qi, s_qi, token_scores, block_scores, ws, L,
                     (cudaStream_t)stream, part, nparts);
}

msa_status msa_block_maxpool_topk(const float* scores, int32_t is_token_level, const msa_seqs* seqs,
                                  int32_t* sel, void* ws, size_t ws_bytes, msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  if (!scores || !aligned16(scores) || !sel || !aligned16(sel)) return MSA_ERR_INVALID_ARG;
  if (is_token_level != 0 && is_token_level != 1) return MSA_ERR_INVALID_ARG;
  Layout L;
  msa_status st = check_ws(seqs, ws, ws_bytes, &L);
  if (st != MSA_OK) return st;
  const size_t nt = n_tok(seqs), bs_bytes = nt * MSA_KV_HEADS * seqs->max_pages * 4;
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_buf(scores, is_token_level ? bs_bytes * MSA_BLOCK_TOKENS : bs_bytes)) != MSA_OK ||
      (st = check_buf(sel, nt * kSelBytes)) != MSA_OK)
    return st;
  const cudaStream_t s = (cudaStream_t)stream;
  const float* bs = scores;
  if (is_token_level) {
    float* dst = at<float>(ws, L.bscores);
    st = cuda_status(launch_maxpool(scores, seqs->seq_lens, seqs->batch, seqs->q_tokens,
                                    seqs->max_pages, dst, at<Flags>(ws, L.flags), s));
    if (st != MSA_OK) return st;
    bs = dst;
  }
  return cuda_status(launch_topk(bs, seqs->seq_lens, seqs->batch, seqs->q_tokens, seqs->max_pages,
                                 sel, at<Flags>(ws, L.flags), s));
}

msa_status msa_sparse_attn_decode(const msa_cache* cache, const msa_seqs* seqs, const uint8_t* q,
                                  float s_q, const int32_t* sel, float softmax_scale,
                                  uint16_t* out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  msa_status st = check_cache(cache, false, true);
  if (st != MSA_OK) return st;
  if (!q || !aligned16(q) || !sel || !aligned16(sel) || !out || !aligned16(out))
    return MSA_ERR_INVALID_ARG;
  if (!good_scale(s_q) || !good_scale(softmax_scale)) return MSA_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(seqs, ws, ws_bytes, &L)) != MSA_OK) return st;
  const size_t nt = n_tok(seqs);
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK ||
      (st = check_cache_mem(cache, false, true)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_buf(q, nt * kQBytes)) != MSA_OK || (st = check_buf(sel, nt * kSelBytes)) != MSA_OK ||
      (st = check_buf(out, nt * kOutBytes)) != MSA_OK)
    return st;
  return run_attn(cache, seqs, q, s_q, sel, softmax_scale, out, ws, L, (cudaStream_t)stream);
}

msa_status msa_decode(const msa_cache* cache, const msa_seqs* seqs, const uint8_t* qi, float s_qi,
                      const uint8_t* q, float s_q, float softmax_scale, uint16_t* out,
                      int32_t* sel_out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  msa_status st = check_cache(cache, true, true);
  if (st != MSA_OK) return st;
  if (!qi || !aligned16(qi) || !q || !aligned16(q) || !out || !aligned16(out))
    return MSA_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return MSA_ERR_INVALID_ARG;
  if (!good_scale(s_qi) || !good_scale(s_q) || !good_scale(softmax_scale))
    return MSA_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(seqs, ws, ws_bytes, &L)) != MSA_OK) return st;
  const size_t nt = n_tok(seqs);
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK ||
      (st = check_cache_mem(cache, true, true)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_buf(qi, nt * kQiBytes)) != MSA_OK || (st = check_buf(q, nt * kQBytes)) != MSA_OK ||
      (st = check_buf(out, nt * kOutBytes)) != MSA_OK || (st = check_buf(sel_out, nt * kSelBytes)) != MSA_OK)
    return st;
  const cudaStream_t s = (cudaStream_t)stream;
  float* bs = at<float>(ws, L.bscores);
  int32_t* sel = sel_out ? sel_out : at<int32_t>(ws, L.sel);
  if ((st = run_indexer(cache, seqs, qi, s_qi, nullptr, bs, ws, L, s)) != MSA_OK) return st;
  st = cuda_status(launch_topk(bs, seqs->seq_lens, seqs->batch, seqs->q_tokens, seqs->max_pages,
                               sel, at<Flags>(ws, L.flags), s));
  if (st != MSA_OK) return st;
  return run_attn(cache, seqs, q, s_q, sel, softmax_scale, out, ws, L, s);
}

msa_status msa_indexer_score_grouped(const msa_cache* cache, const msa_seqs* seqs,
                                     const msa_prefix_groups* groups, const uint8_t* qi, float s_qi,
                                     float* token_scores, float* block_scores, void* ws,
                                     size_t ws_bytes, msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  msa_status st = check_cache(cache, true, false);
  if (st != MSA_OK) return st;
  if ((st = check_groups(groups, seqs)) != MSA_OK) return st;
  if (!qi || !aligned16(qi) || !block_scores || !aligned16(block_scores) || !good_scale(s_qi))
    return MSA_ERR_INVALID_ARG;
  if (token_scores && !aligned16(token_scores)) return MSA_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(seqs, ws, ws_bytes, &L)) != MSA_OK) return st;
  const size_t nt = n_tok(seqs), bs_bytes = nt * MSA_KV_HEADS * seqs->max_pages * 4;
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK ||
      (st = check_cache_mem(cache, true, false)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_groups_mem(groups)) != MSA_OK ||
      (st = check_buf(qi, nt * kQiBytes)) != MSA_OK || (st = check_buf(block_scores, bs_bytes)) != MSA_OK ||
      (st = check_buf(token_scores, bs_bytes * MSA_BLOCK_TOKENS)) != MSA_OK)
    return st;
  const cudaStream_t s = (cudaStream_t)stream;
  if ((st = run_indexer(cache, seqs, qi, s_qi, token_scores, block_scores, ws, L, s, 0, 1, groups, 1)) != MSA_OK)
    return st;
  return run_indexer(cache, seqs, qi, s_qi, token_scores, block_scores, ws, L, s, 0, 1, groups, 0);
}

msa_status msa_decode_grouped(const msa_cache* cache, const msa_seqs* seqs,
                              const msa_prefix_groups* groups, const uint8_t* qi, float s_qi,
                              const uint8_t* q, float s_q, float softmax_scale, uint16_t* out,
                              int32_t* sel_out, void* ws, size_t ws_bytes, msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  msa_status st = check_cache(cache, true, true);
  if (st != MSA_OK) return st;
  if ((st = check_groups(groups, seqs)) != MSA_OK) return st;
  if (!qi || !aligned16(qi) || !q || !aligned16(q) || !out || !aligned16(out))
    return MSA_ERR_INVALID_ARG;
  if (sel_out && !aligned16(sel_out)) return MSA_ERR_INVALID_ARG;
  if (!good_scale(s_qi) || !good_scale(s_q) || !good_scale(softmax_scale))
    return MSA_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(seqs, ws, ws_bytes, &L)) != MSA_OK) return st;
  const size_t nt = n_tok(seqs);
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK ||
      (st = check_cache_mem(cache, true, true)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_groups_mem(groups)) != MSA_OK ||
      (st = check_buf(qi, nt * kQiBytes)) != MSA_OK || (st = check_buf(q, nt * kQBytes)) != MSA_OK ||
      (st = check_buf(out, nt * kOutBytes)) != MSA_OK || (st = check_buf(sel_out, nt * kSelBytes)) != MSA_OK)
    return st;
  const cudaStream_t s = (cudaStream_t)stream;
  float* bs = at<float>(ws, L.bscores);
  int32_t* sel = sel_out ? sel_out : at<int32_t>(ws, L.sel);
  if ((st = run_indexer(cache, seqs, qi, s_qi, nullptr, bs, ws, L, s, 0, 1, groups, 1)) != MSA_OK) return st;
  if ((st = run_indexer(cache, seqs, qi, s_qi, nullptr, bs, ws, L, s, 0, 1, groups, 0)) != MSA_OK) return st;
  st = cuda_status(launch_topk(bs, seqs->seq_lens, seqs->batch, seqs->q_tokens, seqs->max_pages,
                               sel, at<Flags>(ws, L.flags), s));
  if (st != MSA_OK) return st;
  return run_attn(cache, seqs, q, s_q, sel, softmax_scale, out, ws, L, s);
}

msa_status msa_kv_insert(const msa_cache* cache, const msa_seqs* seqs, const uint16_t* k_new,
                         const uint16_t* v_new, const uint16_t* idx_new, void* ws, size_t ws_bytes,
                         msa_stream_t stream) {
  if (!seqs_ok(seqs)) return MSA_ERR_INVALID_ARG;
  msa_status st = check_cache(cache, true, true);
  if (st != MSA_OK) return st;
  if (!k_new || !aligned16(k_new) || !v_new || !aligned16(v_new) || !idx_new || !aligned16(idx_new))
    return MSA_ERR_INVALID_ARG;
  Layout L;
  if ((st = check_ws(seqs, ws, ws_bytes, &L)) != MSA_OK) return st;
  const size_t nt = n_tok(seqs);
  if ((st = check_buf(ws, L.used(), MSA_ERR_WORKSPACE)) != MSA_OK ||
      (st = check_cache_mem(cache, true, true)) != MSA_OK || (st = check_seqs_mem(seqs)) != MSA_OK ||
      (st = check_buf(k_new, nt * MSA_KV_HEADS * MSA_HEAD_DIM * 2)) != MSA_OK ||
      (st = check_buf(v_new, nt * MSA_KV_HEADS * MSA_HEAD_DIM * 2)) != MSA_OK ||
      (st = check_buf(idx_new, nt * MSA_HEAD_DIM * 2)) != MSA_OK)
    return st;
  InsArgs a{};
  a.idx_data = const_cast<uint8_t*>(cache->idx_data);
  a.idx_scale = const_cast<uint8_t*>(cache->idx_scale);
  a.k_data = const_cast<uint8_t*>(cache->k_data);
  a.k_scale = const_cast<uint8_t*>(cache->k_scale);
  a.v_data = const_cast<uint8_t*>(cache->v_data);
  a.v_scale = const_cast<uint8_t*>(cache->v_scale);
  a.page_table = seqs->page_table;
  a.seq_lens = seqs->seq_lens;
  a.k_new = k_new;
  a.v_new = v_new;
  a.idx_new = idx_new;
  a.flags = at<Flags>(ws, L.flags);
  a.s_idx = cache->s_idx;
  a.s_k = cache->s_k;
  a.s_v = cache->s_v;
  a.B = seqs->batch;
  a.T = seqs->q_tokens;
  a.max_pages = seqs->max_pages;
  a.num_pages = cache->num_pages;
  a.idx_fp8 = cache->idx_dtype == MSA_IDX_FP8;
  return cuda_status(launch_insert(a, (cudaStream_t)stream));
}

msa_status msa_get_last_error(void* ws, msa_stream_t stream, int32_t* detail) {
  if (!ws) return MSA_ERR_WORKSPACE;
  const msa_status st = check_buf(ws, sizeof(Flags), MSA_ERR_WORKSPACE);
  if (st != MSA_OK) return st;
  const cudaStream_t s = (cudaStream_t)stream;
  Flags h{};
  if (cudaMemcpyAsync(&h, ws, sizeof(Flags), cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MSA_ERR_CUDA;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MSA_ERR_CUDA;
  if (detail) *detail = h.detail;
  if (h.code != 0) {
    const Flags zero{};
    if (cudaMemcpyAsync(ws, &zero, sizeof(Flags), cudaMemcpyHostToDevice, s) != cudaSuccess ||
        cudaStreamSynchronize(s) != cudaSuccess)
      return MSA_ERR_CUDA;
  }
  return (msa_status)h.code;
}

msa_status msa_debug_nvfp4_table(uint8_t* out, msa_stream_t stream) {
  if (!out || !aligned16(out)) return MSA_ERR_INVALID_ARG;
  const msa_status st = check_buf(out, 256 * 16);
  if (st != MSA_OK) return st;
  return cuda_status(launch_nvfp4_table(out, (cudaStream_t)stream));
}

const char* msa_status_string(msa_status status) {
  switch (status) {
    case MSA_OK: return "ok";
    case MSA_ERR_INVALID_ARG: return "invalid argument";
    case MSA_ERR_UNSUPPORTED: return "unsupported request";
    case MSA_ERR_CUDA: return "CUDA runtime error";
    case MSA_ERR_DEVICE_BOUNDS: return "device bounds check failed (page id, block id or length)";
    case MSA_ERR_TIMEOUT: return "device wait timed out";
    case MSA_ERR_WORKSPACE: return "workspace missing or too small";
  }
  return "unknown status";
}

}  // extern "C"
