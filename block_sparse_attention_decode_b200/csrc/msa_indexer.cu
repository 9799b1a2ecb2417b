// msa_indexer.cu -- indexer scores + block max-pool on the 5th-generation
// tensor core ([post, "MSA primer"]: one index query per GQA group scores
// every cached key against one shared index-key head; the scores are
// max-pooled to one score per 128-token block).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Per page (= one 128-token block) the scores are one dense contraction
//   D[M queries x 128 keys] = Qi[M x 128] * K_page[128 keys x 128]^T
// with a tile of index queries as the M side (T tokens x 4 groups; M = 64
// when the tile holds at most 64 index queries, else tiles of 128) and the
// page's keys as the N side.  Each query's row of D then sits in one TMEM
// lane, so the block max is a reduction along the lane's columns: inside the
// thread, plus two shuffles when a 16x256b load spreads a row over four
// threads.  With M = 64 the accumulator occupies lanes 0-15 of each 32-lane
// quarter (rows 16q..16q+15 in quarter q).
//
// Work split: the pages of all sequences form one flat list, cut into chunks
// of kChunkPages; a work item is (query tile, chunk).  A launch may score
// only part `part` of `nparts` of every sequence's blocks (the context split
// of [post, "NVFP4 indexer DCP"]); the flat list then holds only those
// blocks.  Persistent CTAs take items from a counter in the workspace header
// as they go (ragged batches and CTAs sharing an SM still finish together);
// the last CTA to finish resets the counter.  Warp roles, a few pages apart:
//   warp 8 (producer): per page one tiled TMA load of the codes (64-byte
//     swizzle, so that row-per-thread reads are bank-conflict free) and one
//     bulk copy of the scales into a ring of shared-memory stages (FP8 index
//     keys: one TMA load with the 128-byte swizzle, which is already the
//     MMA's B operand);
//   warps 0-3 (decoders): thread = key row.  NVFP4 rows are decoded to signed
//     E4M3 (dq8: a table row per scale byte, byte permutes for magnitudes
//     and signs) and stored as 128-byte rows with the 128-byte swizzle -- the
//     K-major B operand -- into one of two buffers, so page k+1 is decoded
//     while page k's MMAs run.  When the query tile changes they also stage
//     the tile's index queries (the A operand) into one of two buffers;
//   warp 9 (MMA): one thread issues per page 4 tcgen05.mma of K = 32 (E4M3;
//     8 of K = 16 for FP16) into one of two TMEM accumulators;
//   warps 4-7 (epilogue): warp 4+q reads the accumulator lanes of quarter q,
//     masks keys after each query's position, takes each query's maximum
//     over the page's keys and writes the block score.
// Every wait is a bounded mbarrier wait; on a timeout a thread records
// MSA_ERR_TIMEOUT and leaves its loop, and TMEM is freed before exit.
//
// Modes (the template parameter MODE):
//   kIdxNvfp4  NVFP4 keys re-rounded to E4M3, FP8 MMA (the decode above);
//   kIdxFp8    E4M3 keys, scored from the TMA buffer as they are;
//   kIdxF16    NVFP4 keys decoded exactly to FP16 (e2m1 x scale needs no
//              rounding in FP16) and scored with FP16 MMA against the index
//              queries widened to FP16 -- the exact scores of [post, "NVIDIA
//              Rubin optimized MSA"].  Query and key rows are 256 bytes, held
//              as two 128-byte K-halves; 8 MMAs of K = 16 per page.
#include "msa_internal.h"

namespace msa {

constexpr int kIdxDecWarps = 4;             // warps 0-3: one key row per thread
constexpr int kIdxEpiWarp0 = 4;             // warps 4-7: one per TMEM lane quarter
constexpr int kIdxProducerWarp = 8;
constexpr int kIdxMmaWarp = 9;
static_assert(kIdxThreads == 10 * 32, "warp roles");

enum : int { kPageLoad = 0, kPageMasked = 1, kPageBad = 2, kPageEnd = 3 };
constexpr int kChunkPages = 8;              // pages per work item
constexpr int kInfoRing = 8;                // per-page info slots (decoders -> MMA, epilogue)
constexpr int kIdxTmemCols = 256;           // two accumulators of 128 columns

template <int MODE>
struct IdxCfg {
  static constexpr bool kFp8 = MODE == kIdxFp8;
  static constexpr bool kF16 = MODE == kIdxF16;
  static constexpr int kRow = kF16 ? 256 : 128;            // bytes per query / key row
  static constexpr int kRaw = kFp8 ? kBlock * kDim : kPageCodes + kPageScales;
  static constexpr int kRawStride = (kRaw + 1023) / 1024 * 1024;
  static constexpr int kStages = kFp8 ? 5 : (kF16 ? 3 : 4);   // raw pages in flight
  static constexpr int kNB = kFp8 ? 0 : 2;                 // decoded key pages (B operand), page k in k % 2
  static constexpr int kBBytes = kBlock * kRow;
};

struct IdxLayout {
  int qbuf, raw, bbuf, lut, bars, meta, pinfo, tslot, prefix, scratch, total;
};

template <int MODE, int M>
__host__ __device__ inline IdxLayout idx_layout(int batch) {
  using C = IdxCfg<MODE>;
  IdxLayout L;
  int off = 0;
  L.qbuf = off;    off += 2 * M * C::kRow;                 // two query tiles (multiples of 1024)
  L.raw = off;     off += C::kStages * C::kRawStride;
  L.bbuf = off;    off += C::kNB * C::kBBytes;
  L.lut = off;     off += MODE == kIdxNvfp4 ? 256 * 8 : 0;
  L.bars = off;    off += (2 * C::kStages + 8) * 8;
  L.meta = off;    off += C::kStages * 8 * 4;              // per stage: b, i, kind, tile, L
  L.pinfo = off;   off += kInfoRing * 8 * 4;               // per page: b, i, kind, tile, L, qsel
  L.tslot = off;   off += 16;
  L.prefix = off;  off += (batch + 1) * 4;
  L.scratch = off; off += kIdxThreads * 4;
  L.total = off + 1024;                                   // alignment slack
  return L;
}

// Index queries per tile: a tile is the M side of the MMA.
int idx_tile_queries(int T) { return kG * T <= 64 ? 64 : 128; }

size_t indexer_smem_bytes(int mode, int batch, int T) {
  const bool m64 = idx_tile_queries(T) == 64;
  if (mode == kIdxFp8) return (size_t)(m64 ? idx_layout<kIdxFp8, 64>(batch) : idx_layout<kIdxFp8, 128>(batch)).total;
  if (mode == kIdxF16) return (size_t)(m64 ? idx_layout<kIdxF16, 64>(batch) : idx_layout<kIdxF16, 128>(batch)).total;
  return (size_t)(m64 ? idx_layout<kIdxNvfp4, 64>(batch) : idx_layout<kIdxNvfp4, 128>(batch)).total;
}

// The part of a sequence of length L this launch scores: logical blocks
// [first, first + count) with first = floor(nblk * part / nparts) -- the
// context split of [post, "NVFP4 indexer DCP"] (parts 0 of 1: every block).
// Invalid lengths give 0 blocks.
__device__ __forceinline__ int part_blocks(const IdxArgs& a, int L, int* first) {
  *first = 0;
  if (L < a.T || L > a.max_pages * kBlock) return 0;
  const int nblk = (L + kBlock - 1) / kBlock;
  if (a.nparts == 1) return nblk;
  // nblk * nparts fits in 32 bits: nblk < 2^24 (L <= max_pages * 128 < 2^31), nparts <= 64
  const int lo = nblk * a.part / a.nparts;
  const int hi = nblk * (a.part + 1) / a.nparts;
  *first = lo;
  return hi - lo;
}

// Exclusive prefix over the number of blocks this launch scores in each
// sequence, in shared memory (prefix[B] = total pages).  Invalid lengths
// count as 0 blocks and are reported once (by CTA 0).
__device__ void page_prefix(const IdxArgs& a, int* prefix, int* scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (a.B + nt - 1) / nt;
  const int lo = tid * per, hi = min(a.B, lo + per);
  int sum = 0;
  for (int b = lo; b < hi; ++b) {
    const int L = a.seq_lens[b];
    int first;
    const int nb = part_blocks(a, L, &first);
    if ((L < a.T || L > a.max_pages * kBlock) && blockIdx.x == 0)
      report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
    sum += nb;
  }
  scratch[tid] = sum;
  __syncthreads();
  if (tid == 0) {
    int run = 0;
    for (int k = 0; k < nt; ++k) { const int v = scratch[k]; scratch[k] = run; run += v; }
    prefix[a.B] = run;
  }
  __syncthreads();
  int run = scratch[tid];
  for (int b = lo; b < hi; ++b) {
    prefix[b] = run;
    int first;
    run += part_blocks(a, a.seq_lens[b], &first);
  }
  __syncthreads();
}

__device__ __forceinline__ void sts128(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// Instruction descriptor of the page MMA: M x 128, fp32 accumulate, both
// operands K-major; E4M3 (kind::f8f6f4) or FP16 (kind::f16), whose format
// fields both read 0.
template <int M>
__host__ __device__ constexpr uint32_t idx_idesc() { return idesc_e4m3_f32(M, kBlock); }

template <int MODE, int M>
__global__ void __launch_bounds__(kIdxThreads, 2) indexer_kernel(const __grid_constant__ IdxArgs a) {
  using C = IdxCfg<MODE>;
  constexpr bool FP8 = C::kFp8, F16 = C::kF16;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
  const IdxLayout Ly = idx_layout<MODE, M>(a.B);
  uint8_t* qbuf = smem + Ly.qbuf;
  uint8_t* raw = smem + Ly.raw;
  uint8_t* bbuf = smem + Ly.bbuf;
  uint2* lut = reinterpret_cast<uint2*>(smem + Ly.lut);
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* raw_empty = raw_full + S;
  uint64_t* b_full = raw_empty + S;      // [2] decoders -> MMA: page k ready (k % 2)
  uint64_t* b_empty = b_full + 2;        // [2] MMA -> decoders: page k consumed
  uint64_t* d_full = b_empty + 2;        // [2] MMA -> epilogue
  uint64_t* d_empty = d_full + 2;        // [2] epilogue -> MMA
  int* meta = reinterpret_cast<int*>(smem + Ly.meta);
  int* pinfo = reinterpret_cast<int*>(smem + Ly.pinfo);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly.tslot);
  int* prefix = reinterpret_cast<int*>(smem + Ly.prefix);
  int* scratch = reinterpret_cast<int*>(smem + Ly.scratch);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (MODE == kIdxNvfp4) build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], FP8 ? 1 : kIdxDecWarps);   // FP8: released by the MMA
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&b_full[x], kIdxDecWarps);
      mbar_init(&b_empty[x], 1);
      mbar_init(&d_full[x], 1);
      mbar_init(&d_empty[x], 4);
    }
    mbar_fence_init();
  }
  if (warp == kIdxMmaWarp) {
    tmem_alloc(tslot, kIdxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  page_prefix(a, prefix, scratch);   // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem = *tslot;

  const int total = prefix[a.B];
  const int nq_all = kG * a.T;                                // index queries per sequence
  const int gy = (nq_all + M - 1) / M;                        // query tiles
  const int nchunks = (total + kChunkPages - 1) / kChunkPages;
  const int items = nchunks * gy;
  const long long ctx = (long long)a.max_pages * kBlock;

  if (warp == kIdxProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0;                                  // page slot (stage k % S)
      bool ok = true;
      auto slot = [&](int kk) -> bool {           // wait until stage kk % S is free
        return kk < S || mbar_wait(&raw_empty[kk % S], ((kk / S) - 1) & 1);
      };
      int first_b = -1, first = 0;                // part_blocks of sequence first_b
      int item = atomicAdd(&a.work[0], 1);
      while (item < items && ok) {
        const int nxt = atomicAdd(&a.work[0], 1);  // claimed early: its latency overlaps this item
        const int y = item / nchunks, p0 = (item % nchunks) * kChunkPages;
        const int p1 = min(total, p0 + kChunkPages);
        const int t_last = (min(nq_all, (y + 1) * M) - 1) >> 2;
        int b;
        {  // prefix[b] <= p0 < prefix[b+1]
          int l = 0, r = a.B;
          while (r - l > 1) { const int m = (l + r) >> 1; if (prefix[m] <= p0) l = m; else r = m; }
          b = l;
        }
        int li = p0 - prefix[b];                    // index among this part's blocks of b
        for (int pg = p0; pg < p1; ++pg, ++k, ++li) {
          if (!slot(k)) { report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1); ok = false; break; }
          const int s = k % S;
          while (li >= prefix[b + 1] - prefix[b]) { li -= prefix[b + 1] - prefix[b]; ++b; }
          const int L = a.seq_lens[b];
          if (b != first_b) {                       // first block of b's part
            first_b = b;
            part_blocks(a, L, &first);
          }
          const int i = first + li;                 // logical block
          int kind = kPageLoad;
          const long long p = a.page_table ? (long long)a.page_table[(long long)b * a.max_pages + i]
                                           : (long long)b * a.max_pages + i;
          if (i * kBlock > L - a.T + t_last) {
            kind = kPageMasked;                     // no key of the block is visible to the tile
          } else if (p < 0 || p >= a.num_pages) {
            report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)p);
            kind = kPageBad;
          }
          int* m = meta + 8 * s;
          m[0] = b; m[1] = i; m[2] = kind; m[3] = y; m[4] = L;
          uint8_t* dst = raw + s * C::kRawStride;
          if (kind == kPageLoad) {
            mbar_expect_tx(&raw_full[s], C::kRaw);
            tma_load_2d(dst, &a.tmap_idx, 0, (int)(p * kBlock), &raw_full[s]);
            if (!FP8) bulk_g2s(dst + kPageCodes, a.idx_scale + p * kPageScales, kPageScales, &raw_full[s]);
          } else {
            mbar_arrive(&raw_full[s]);
          }
        }
        item = nxt;
      }
      if (ok) {   // end marker
        if (!slot(k)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1);
        } else {
          meta[8 * (k % S) + 2] = kPageEnd;
          mbar_arrive(&raw_full[k % S]);
        }
      }
      // every CTA has made its last claim once all have arrived here
      __threadfence();
      if (atomicAdd(&a.work[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&a.work[0], 0);
        atomicExch(&a.work[1], 0);
      }
    }
  } else if (warp == kIdxMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idx_idesc<M>();
      for (int k = 0;; ++k) {
        const int x = k & 1;                       // accumulator and page-ready barrier
        if (!mbar_wait(&b_full[x], (k >> 1) & 1)) { report(a.flags, 5, 2); break; }
        if (k >= 2 && !mbar_wait(&d_empty[x], ((k >> 1) - 1) & 1)) { report(a.flags, 5, 3); break; }
        tc_fence_after();
        const int* pf = pinfo + 8 * (k % kInfoRing);
        const int kind = pf[2], qsel = pf[5];
        if (kind == kPageLoad) {
          const uint32_t d = tmem + (uint32_t)(x * kBlock);
          const uint32_t qa = smem_u32(qbuf + qsel * M * C::kRow);
          const uint32_t kb = FP8 ? smem_u32(raw + (k % S) * C::kRawStride)
                                  : smem_u32(bbuf + x * C::kBBytes);
          if constexpr (F16) {
            // K-half h of the queries starts M rows further, of the keys 128 rows further
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc_mma_ss_f16(d, desc_kmajor_sw128(qa + (kk >> 2) * M * 128) + 2 * (kk & 3),
                            desc_kmajor_sw128(kb + (kk >> 2) * kBlock * 128) + 2 * (kk & 3), idesc, kk > 0);
          } else {
            const uint64_t ad = desc_kmajor_sw128(qa), bd = desc_kmajor_sw128(kb);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc_mma_ss(d, ad + 2 * kk, bd + 2 * kk, idesc, kk > 0);
          }
        }
        tc_commit(&d_full[x]);
        if (kind == kPageEnd) break;
        if (FP8) tc_commit(&raw_empty[k % S]);   // the stage was the B operand
        tc_commit(&b_empty[x]);                   // page k consumed (and its B buffer free)
      }
    }
  } else if (warp >= kIdxEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp - kIdxEpiWarp0;             // TMEM lane quarter
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    // rows of the tile this warp reads: M = 64: 16q..16q+15; M = 128: 32q..32q+31
    constexpr int kRows = M == 64 ? 16 : 32;
    for (int k = 0;; ++k) {
      const int x = k & 1;
      if (!mbar_wait(&d_full[x], (k >> 1) & 1)) { report(a.flags, 5, 6); break; }
      tc_fence_after();
      const int* pf = pinfo + 8 * (k % kInfoRing);
      const int pb = pf[0], pi = pf[1], pkind = pf[2], py = pf[3], pL = pf[4];
      if (pkind == kPageEnd) break;
      const int qbase = py * M + kRows * q;          // first index query of this warp's rows
      const bool active = qbase < nq_all;            // warp-uniform
      const int pos0 = pL - a.T;
      if (active && pkind == kPageLoad) {
        const uint32_t dcol = (uint32_t)(x * kBlock);
        if constexpr (M == 64) {
          // 16x256b: thread (g, t) holds rows g and g+8 of the quarter, columns 8c+2t, 8c+2t+1
          const int g = lane >> 2, t = lane & 3;
          float m0 = -INFINITY, m1 = -INFINITY;
          const int qa0 = qbase + g, qa1 = qa0 + 8;
          const int lim0 = pos0 + (qa0 >> 2), lim1 = pos0 + (qa1 >> 2);   // last visible key
          const bool need_mask = pi * kBlock + kBlock - 1 > pos0 + (qbase >> 2);
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {                // columns 64h .. 64h+63
            float v[32];
            tmem_ld_16x256b_x8(lane_base + dcol + 64 * h, v);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int key = pi * kBlock + 64 * h + 8 * (i >> 2) + 2 * t + (i & 1);
                if (key > ((i & 2) ? lim1 : lim0)) v[i] = -INFINITY;
              }
            }
            if (a.token_scores != nullptr) {
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                const int qa = (i & 2) ? qa1 : qa0, tt = qa >> 2;
                if (tt < a.T) {
                  float* rowp = a.token_scores + (((long long)pb * a.T + tt) * kG + (qa & 3)) * ctx;
                  const int col = pi * kBlock + 64 * h + 8 * (i >> 2) + 2 * t;
                  rowp[col] = v[i] * a.score_scale;
                  rowp[col + 1] = v[i + 1] * a.score_scale;
                }
              }
            }
            float r0[16], r1[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              r0[2 * c] = v[4 * c]; r0[2 * c + 1] = v[4 * c + 1];
              r1[2 * c] = v[4 * c + 2]; r1[2 * c + 1] = v[4 * c + 3];
            }
            m0 = fmaxf(m0, max_of<16>(r0));
            m1 = fmaxf(m1, max_of<16>(r1));
          }
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
          m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
          if (t < 2) {
            const int qa = t == 0 ? qa0 : qa1, tt = qa >> 2;
            if (tt < a.T)
              a.block_scores[(((long long)pb * a.T + tt) * kG + (qa & 3)) * a.max_pages + pi] =
                  (t == 0 ? m0 : m1) * a.score_scale;
          }
        } else {
          // 32x32b: thread = row (index query qbase + lane), all 128 columns
          const int qa = qbase + lane, tt = qa >> 2;
          const int lim = pos0 + tt;
          const bool need_mask = pi * kBlock + kBlock - 1 > pos0 + (qbase >> 2);
          float m = -INFINITY;
#pragma unroll 1
          for (int h = 0; h < 4; ++h) {
            float v[32];
            tmem_ld_32x32b_x32(lane_base + dcol + 32 * h, v);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (pi * kBlock + 32 * h + i > lim) v[i] = -INFINITY;
            }
            if (a.token_scores != nullptr && tt < a.T) {
              float* rowp = a.token_scores + (((long long)pb * a.T + tt) * kG + (qa & 3)) * ctx +
                            pi * kBlock + 32 * h;
#pragma unroll
              for (int i = 0; i < 32; ++i) rowp[i] = v[i] * a.score_scale;
            }
            m = fmaxf(m, max_of<32>(v));
          }
          if (tt < a.T)
            a.block_scores[(((long long)pb * a.T + tt) * kG + (qa & 3)) * a.max_pages + pi] =
                m * a.score_scale;
        }
      } else if (active && pkind == kPageMasked) {
        // no key of the block is visible to any query of the tile
        for (int r = lane; r < kRows; r += 32) {
          const int qa = qbase + r, tt = qa >> 2;
          if (tt >= a.T) continue;
          const long long row = ((long long)pb * a.T + tt) * kG + (qa & 3);
          a.block_scores[row * a.max_pages + pi] = -INFINITY;
          if (a.token_scores != nullptr)
            for (int j = 0; j < kBlock; ++j) a.token_scores[row * ctx + pi * kBlock + j] = -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[x]);
    }
  } else {
    // ------------------------------------------------------------ decoders
    const int row = 32 * warp + lane;                                     // key row of this thread
    int cur_b = -1, cur_y = -1, qsel = 1;
    for (int k = 0;; ++k) {
      const int s = k % S;
      if (!mbar_wait(&raw_full[s], (k / S) & 1)) { report(a.flags, 5, 5); break; }
      // page k-2 consumed by the MMA: its B buffer (k % 2) and the page-ready
      // barrier k % 2 are free, and every MMA of pages <= k-2 has completed
      if (k >= 2 && !mbar_wait(&b_empty[k & 1], ((k >> 1) - 1) & 1)) {
        report(a.flags, 5, 4);
        break;
      }
      const int* m = meta + 8 * s;
      const int nb = m[0], ni = m[1], nkind = m[2], ny = m[3], nL = m[4];
      if (nkind != kPageEnd && (nb != cur_b || ny != cur_y)) {
        cur_b = nb;
        cur_y = ny;
        qsel ^= 1;
        // A operand: the index queries of tile ny of sequence nb, K-major
        // with the 128-byte swizzle, zero rows past the sequence's queries.
        // Its previous user (a tile that ended two or more pages ago) has
        // completed: the MMA of page k-2 has (the wait above).
        uint8_t* qb = qbuf + qsel * M * C::kRow;
        const int qbase = ny * M;
        for (int idx = row; idx < M * 8; idx += kIdxDecWarps * 32) {
          const int nrow = idx >> 3, c = idx & 7;
          const int qg = qbase + nrow;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (qg < nq_all)
            v = *reinterpret_cast<const uint4*>(a.qi + ((long long)nb * nq_all + qg) * kDim + 16 * c);
          if constexpr (F16) {
            // dims 16c..16c+15 -> FP16 chunks 2c, 2c+1 of 8 dims: K-half c / 4,
            // chunk positions (2c % 8, 2c % 8 + 1) ^ (row % 8) in its 128-byte row
            const uint4 lo = make_uint4(e4m3x2_to_f16x2(v.x), e4m3x2_to_f16x2(v.x >> 16),
                                        e4m3x2_to_f16x2(v.y), e4m3x2_to_f16x2(v.y >> 16));
            const uint4 hi = make_uint4(e4m3x2_to_f16x2(v.z), e4m3x2_to_f16x2(v.z >> 16),
                                        e4m3x2_to_f16x2(v.w), e4m3x2_to_f16x2(v.w >> 16));
            uint8_t* rowp = qb + (c >> 2) * M * 128 + nrow * 128;
            const int j = (2 * c) & 7;
            sts128(rowp + ((j ^ (nrow & 7)) << 4), lo);
            sts128(rowp + (((j + 1) ^ (nrow & 7)) << 4), hi);
          } else {
            sts128(qb + nrow * 128 + ((c ^ (nrow & 7)) << 4), v);
          }
        }
      }
      if (!FP8 && nkind == kPageLoad) {
        const uint8_t* rs = raw + s * C::kRawStride;
        uint8_t* bb = bbuf + (k & 1) * C::kBBytes;
        // 64-byte code rows loaded with the 64-byte swizzle: chunk c of row r
        // sits at chunk position c ^ ((r / 2) % 4); chunk c = elements
        // 32c..32c+31 under scale bytes 2c and 2c+1
        const uint2 sc = *reinterpret_cast<const uint2*>(rs + kPageCodes + row * kRowScales);
        const int sw = (row >> 1) & 3;
        if constexpr (F16) {
          // FP16 key row: 256 bytes as two 128-byte K-halves (rows 128 apart),
          // each with the 128-byte swizzle; chunk c -> 16-byte chunks 4c..4c+3
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w4 = lds128(rs + row * kRowCodes + ((c ^ sw) << 4));
            const uint32_t s2 = e4m3x2_to_f16x2((c < 2 ? sc.x : sc.y) >> (16 * (c & 1)));
            const uint32_t s_lo = prmt(s2, 0u, 0x1010u), s_hi = prmt(s2, 0u, 0x3232u);
            uint32_t o[16];
            e2m1x8_to_f16x2(w4.x, o + 0);
            e2m1x8_to_f16x2(w4.y, o + 4);
            e2m1x8_to_f16x2(w4.z, o + 8);
            e2m1x8_to_f16x2(w4.w, o + 12);
#pragma unroll
            for (int mm = 0; mm < 16; ++mm) o[mm] = hmul2(o[mm], mm < 8 ? s_lo : s_hi);
            uint8_t* rowp = bb + (c >> 1) * kBlock * 128 + row * 128;
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int ch = 4 * (c & 1) + j;
              sts128(rowp + ((ch ^ (row & 7)) << 4),
                     make_uint4(o[4 * j], o[4 * j + 1], o[4 * j + 2], o[4 * j + 3]));
            }
          }
        } else {
          // E4M3 key row: 128 bytes with the 128-byte swizzle; code chunk c ->
          // row chunks 2c, 2c+1
          uint8_t* rowp = bb + row * 128;
#pragma unroll
          for (int c = 0; c < 4; ++c) {
            const uint4 w4 = lds128(rs + row * kRowCodes + ((c ^ sw) << 4));
            const uint32_t sb = (c < 2 ? sc.x : sc.y) >> (16 * (c & 1));   // scales 2c, 2c+1
            const uint2 r0 = lut[sb & 0xFFu], r1 = lut[(sb >> 8) & 0xFFu];
            uint32_t o[8];
            dq8(w4.x, r0, o[0], o[1]);
            dq8(w4.y, r0, o[2], o[3]);
            dq8(w4.z, r1, o[4], o[5]);
            dq8(w4.w, r1, o[6], o[7]);
            sts128(rowp + (((2 * c) ^ (row & 7)) << 4), make_uint4(o[0], o[1], o[2], o[3]));
            sts128(rowp + (((2 * c + 1) ^ (row & 7)) << 4), make_uint4(o[4], o[5], o[6], o[7]));
          }
        }
      }
      fence_async_smem();   // generic-proxy writes (queries, keys) -> the MMA
      __syncwarp();
      if (lane == 0) {
        if (warp == 0) {
          int* pf = pinfo + 8 * (k % kInfoRing);
          pf[0] = nb; pf[1] = ni; pf[2] = nkind; pf[3] = ny; pf[4] = nL; pf[5] = qsel;
        }
        if (!FP8) mbar_arrive(&raw_empty[s]);
        mbar_arrive(&b_full[k & 1]);
      }
      if (nkind == kPageEnd) break;
    }
  }

  // ---- teardown: every role leaves its loop (normally or on a timeout)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kIdxMmaWarp) tmem_dealloc(tmem, kIdxTmemCols);
}

template <int MODE, int M>
static cudaError_t launch_mode(const IdxArgs& a, cudaStream_t st) {
  auto kern = indexer_kernel<MODE, M>;
  const size_t smem = (size_t)idx_layout<MODE, M>(a.B).total;
  int grid = 0;                                 // persistent: items are claimed in the kernel
  cudaError_t e = persistent_grid(reinterpret_cast<const void*>(kern), kIdxThreads, smem,
                                  kIdxTmemCols, &grid);
  if (e != cudaSuccess) return e;
  kern<<<grid, kIdxThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(const IdxArgs& a, int mode, cudaStream_t st) {
  const bool m64 = idx_tile_queries(a.T) == 64;
  if (mode == kIdxFp8) return m64 ? launch_mode<kIdxFp8, 64>(a, st) : launch_mode<kIdxFp8, 128>(a, st);
  if (mode == kIdxF16) return m64 ? launch_mode<kIdxF16, 64>(a, st) : launch_mode<kIdxF16, 128>(a, st);
  return m64 ? launch_mode<kIdxNvfp4, 64>(a, st) : launch_mode<kIdxNvfp4, 128>(a, st);
}

}  // namespace msa
