// msa_indexer.cu -- indexer scores + block max-pool on the 5th-generation
// tensor core ([post, "MSA primer"]: one index query per GQA group scores
// every cached key against one shared index-key head; the scores are
// max-pooled to one score per 128-token block).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Per page (= one 128-token block) the scores are one dense FP8 contraction
//   D[128 keys x NQ queries] = K_page[128 x 128] * Qi[NQ x 128]^T
// with the keys as the M side (the block max is a reduction over TMEM
// lanes) and a chunk of NQ index queries (T tokens x 4 groups, padded to
// 16, 32, 64, 128 or 256) as the N side.
//
// Work split: the pages of all sequences form one flat list, cut into chunks
// of kChunkPages; a work item is (query tile of NQ index queries, chunk).
// A launch may score only part `part` of `nparts` of every sequence's blocks
// (the context split of [post, "NVFP4 indexer DCP"]); the flat list then
// holds only those blocks.
// Persistent CTAs (two per SM) take items from a counter in the workspace
// header as they go, so that CTAs sharing an SM -- which the warp schedulers
// do not serve equally -- and ragged batches still finish together; the last
// CTA to finish resets the counter.  Warp roles inside a CTA, all running a
// few pages apart:
//   warp 12 (producer): per page one tiled TMA load of the codes (64-byte
//     swizzle, so that row-per-thread reads are bank-conflict free) and one
//     bulk copy of the scales into a ring of shared-memory stages;
//   warps 0-3 (decoders): thread = key row (= TMEM lane).  NVFP4 rows are
//     decoded by sign: K+ holds E4M3(|v|) of the positive elements, K- of the
//     negative ones (one prmt per 4 codes each, see dq8_split), and both go
//     straight to tensor memory with tcgen05.st into one of two A buffers --
//     the A operand never touches shared memory, and page k+1 is decoded
//     while page k's MMAs run;
//   warp 13 (MMA): one thread issues per page 4 tcgen05.mma with A = K+ and 4
//     with A = K- and the negate-A bit (K = 32 each, A from TMEM, B = the
//     queries in shared memory) into a double-buffered TMEM accumulator;
//   warps 4-11 (epilogue, two groups of four taking the even and the odd
//     pages, so that two pages are reduced at once): warp 4+4j+q reads the
//     accumulator lanes of quarter q, masks keys after each query's position,
//     and reduces over keys: in-thread over the four keys a 16x256b load
//     gives each thread, then xor shuffles across lane groups; after a
//     rendezvous on an mbarrier each warp combines the four quarters' partial
//     maxima of a quarter of the columns and writes those block scores.
// Every wait is a bounded mbarrier wait; on a timeout a thread records
// MSA_ERR_TIMEOUT and leaves its loop, and TMEM is freed before exit.
//
// Modes (the template parameter MODE):
//   kIdxNvfp4  NVFP4 keys re-rounded to E4M3, FP8 MMA (the sign split above);
//   kIdxFp8    E4M3 keys, copied to TMEM as they are;
//   kIdxF16    NVFP4 keys decoded exactly to FP16 (e2m1 x scale needs no
//              rounding in FP16) and scored with FP16 MMA against the index
//              queries widened to FP16 -- the exact scores of [post, "NVIDIA
//              Rubin optimized MSA"].  One A buffer holds the 128 FP16 values
//              of each row in 64 columns; the queries take two 128-byte
//              swizzled K-halves in shared memory; 8 MMAs of K = 16 per page.
#include "msa_internal.h"

namespace msa {

constexpr int kIdxDecoders = 4;             // one per TMEM lane quarter, full rows
constexpr int kIdxEpilogue = 4;             // per group: one per TMEM lane quarter
constexpr int kIdxEpiWarp0 = 4;             // two groups: even and odd pages
constexpr int kIdxProducerWarp = 12;
constexpr int kIdxMmaWarp = 13;
constexpr int kABufCols = 64;               // TMEM columns of one A buffer (K+ | K-, or FP16)
constexpr int kACols = 2 * kABufCols;       // two A buffers

enum : int { kPageLoad = 0, kPageMasked = 1, kPageBad = 2, kPageEnd = 3 };
constexpr int kChunkPages = 8;              // pages per work item

struct IdxLayout {
  int qbuf, raw, raw_stride, lut, red, bars, meta, tinfo, pinfo, tslot, prefix, scratch, total;
};

// Bytes of one raw page in shared memory (codes [+ scales]), 1024-aligned.
__host__ __device__ inline int raw_stage_stride(bool fp8idx) {
  return fp8idx ? kBlock * kDim : ((kPageCodes + kPageScales + 1023) / 1024) * 1024;
}

// Bytes of one query row in shared memory: E4M3, or two 128-byte K-halves of FP16.
__host__ __device__ constexpr int q_row_bytes(int mode) { return mode == kIdxF16 ? 256 : 128; }

__host__ __device__ inline IdxLayout idx_layout(int nq, int mode, int batch) {
  IdxLayout L;
  int off = 0;
  L.qbuf = off;    off += 2 * nq * q_row_bytes(mode);     // nq % 8 == 0 -> 1024-aligned
  L.raw_stride = raw_stage_stride(mode == kIdxFp8);
  L.raw = off;     off += kIdxRawStages * L.raw_stride;
  L.lut = off;     off += 256 * 8;
  L.red = off;     off += 2 * kIdxEpilogue * nq * 4;          // [group][quarter][nq]
  L.bars = off;    off += (2 * kIdxRawStages + 10) * 8;
  L.meta = off;    off += 4 * kIdxRawStages * 4;           // per stage: b, i, kind, tile
  L.tinfo = off;   off += 2 * 2 * 4;                       // per A buffer: what, qsel
  L.pinfo = off;   off += 4 * 8 * 4;                       // ring of 4: b, i, kind, L, tile
  L.tslot = off;   off += 16;
  L.prefix = off;  off += (batch + 1) * 4;
  L.scratch = off; off += kIdxThreads * 4;
  L.total = off + 1024;                                   // alignment slack
  return L;
}

// N of the MMA: with A in tensor memory and M = 128, N is a multiple of 16
// from 16 to 256 (the tcgen05.mma shape table), so one query token's 4 index
// queries are padded to 16.
int idx_nq(int T) {
  const int nq = kG * T;
  if (nq <= 16) return 16;
  if (nq <= 32) return 32;
  if (nq <= 64) return 64;
  if (nq <= 128) return 128;
  return 256;
}

size_t indexer_smem_bytes(int mode, int batch, int T) {
  return (size_t)idx_layout(idx_nq(T), mode, batch).total;
}

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
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
// count as 0 blocks and are reported once (by CTA (0,0)).
__device__ void page_prefix(const IdxArgs& a, int* prefix, int* scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (a.B + nt - 1) / nt;
  const int lo = tid * per, hi = min(a.B, lo + per);
  int sum = 0;
  for (int b = lo; b < hi; ++b) {
    const int L = a.seq_lens[b];
    int first;
    const int nb = part_blocks(a, L, &first);
    if ((L < a.T || L > a.max_pages * kBlock) && blockIdx.x == 0 && blockIdx.y == 0)
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

template <int NQ, int MODE>
__global__ void __launch_bounds__(kIdxThreads, 2) indexer_kernel(const __grid_constant__ IdxArgs a) {
  constexpr bool FP8IDX = MODE == kIdxFp8;
  constexpr bool F16 = MODE == kIdxF16;
  constexpr int kQRow = q_row_bytes(MODE);
  constexpr int kND = NQ <= 64 ? 2 : 1;                      // accumulator buffers
  constexpr int kCols = pow2_at_least(kACols + kND * NQ);    // TMEM columns
  constexpr int kChunk = NQ < 32 ? NQ : (NQ >= 128 ? 16 : 32);   // columns per TMEM load
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
  const IdxLayout Ly = idx_layout(NQ, MODE, a.B);
  uint8_t* qbuf = smem + Ly.qbuf;
  uint8_t* raw = smem + Ly.raw;
  uint2* lut = reinterpret_cast<uint2*>(smem + Ly.lut);
  float* red = reinterpret_cast<float*>(smem + Ly.red);            // [group][quarter][NQ]
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* raw_empty = raw_full + kIdxRawStages;
  uint64_t* a_full = raw_empty + kIdxRawStages;                    // decoders -> MMA [2]
  uint64_t* a_empty = a_full + 2;                                  // MMA -> decoders [2]
  uint64_t* acc_full = a_empty + 2;                                // MMA -> epilogue [2]
  uint64_t* acc_empty = acc_full + 2;                              // epilogue -> MMA [2]
  uint64_t* red_full = acc_empty + 2;                              // group rendezvous [2]
  int* meta = reinterpret_cast<int*>(smem + Ly.meta);              // [stage][b, i, kind, tile]
  int* tinfo = reinterpret_cast<int*>(smem + Ly.tinfo);            // [A buffer][what, qsel]
  int* pinfo = reinterpret_cast<int*>(smem + Ly.pinfo);            // [k % 4][b, i, kind, L, tile]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly.tslot);
  int* prefix = reinterpret_cast<int*>(smem + Ly.prefix);
  int* scratch = reinterpret_cast<int*>(smem + Ly.scratch);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (MODE == kIdxNvfp4) build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < kIdxRawStages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kIdxDecoders);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&a_full[x], kIdxDecoders);
      mbar_init(&a_empty[x], 1);
      mbar_init(&acc_full[x], 1);
      mbar_init(&acc_empty[x], kIdxEpilogue);
      mbar_init(&red_full[x], kIdxEpilogue);
    }
    mbar_fence_init();
  }
  if (warp == kIdxMmaWarp) {
    tmem_alloc(tslot, kCols);
    tmem_relinquish();
  }
  tc_fence_before();
  page_prefix(a, prefix, scratch);   // ends with __syncthreads
  tc_fence_after();
  const uint32_t tmem = *tslot;

  const int total = prefix[a.B];
  const int gy = (kG * a.T + NQ - 1) / NQ;                  // query tiles
  const int nchunks = (total + kChunkPages - 1) / kChunkPages;
  const int items = nchunks * gy;
  const long long ctx = (long long)a.max_pages * kBlock;

  if (warp == kIdxProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      int k = 0;                                  // page slot (stage k % kIdxRawStages)
      bool ok = true;
      auto slot = [&](int kk) -> bool {           // wait until stage kk % S is free
        return kk < kIdxRawStages ||
               mbar_wait(&raw_empty[kk % kIdxRawStages], ((kk / kIdxRawStages) - 1) & 1);
      };
      int first_b = -1, first = 0;                // part_blocks of sequence first_b
      int item = atomicAdd(&a.work[0], 1);
      while (item < items && ok) {
        const int nxt = atomicAdd(&a.work[0], 1);  // claimed early: its latency overlaps this item
        const int y = item / nchunks, p0 = (item % nchunks) * kChunkPages;
        const int p1 = min(total, p0 + kChunkPages);
        const int t_last = min(a.T - 1, (y * NQ + NQ - 1) >> 2);
        int b;
        {  // prefix[b] <= p0 < prefix[b+1]
          int l = 0, r = a.B;
          while (r - l > 1) { const int m = (l + r) >> 1; if (prefix[m] <= p0) l = m; else r = m; }
          b = l;
        }
        int li = p0 - prefix[b];                    // index among this part's blocks of b
        for (int pg = p0; pg < p1; ++pg, ++k, ++li) {
          if (!slot(k)) { report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1); ok = false; break; }
          const int s = k % kIdxRawStages;
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
            kind = kPageMasked;
          } else if (p < 0 || p >= a.num_pages) {
            report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)p);
            kind = kPageBad;
          }
          meta[4 * s + 0] = b;
          meta[4 * s + 1] = i;
          meta[4 * s + 2] = kind;
          meta[4 * s + 3] = y;
          uint8_t* dst = raw + s * Ly.raw_stride;
          if (kind == kPageLoad) {
            if (FP8IDX) {
              mbar_expect_tx(&raw_full[s], kBlock * kDim);
              tma_load_2d(dst, &a.tmap_idx, 0, (int)(p * kBlock), &raw_full[s]);
            } else {
              mbar_expect_tx(&raw_full[s], kPageCodes + kPageScales);
              tma_load_2d(dst, &a.tmap_idx, 0, (int)(p * kBlock), &raw_full[s]);
              bulk_g2s(dst + kPageCodes, a.idx_scale + p * kPageScales, kPageScales, &raw_full[s]);
            }
          } else {
            mbar_arrive(&raw_full[s]);
          }
        }
        item = nxt;
      }
      // two end markers: one for each epilogue group
      for (int e = 0; e < 2 && ok; ++e, ++k) {
        if (!slot(k)) { report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1); break; }
        meta[4 * (k % kIdxRawStages) + 2] = kPageEnd;
        mbar_arrive(&raw_full[k % kIdxRawStages]);
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
      constexpr uint32_t idesc = F16 ? idesc_f16_f32(128, NQ) : idesc_e4m3_f32(128, NQ);
      constexpr uint32_t idesc_neg = idesc | (1u << 13);     // negate A
      // B descriptors of the two query buffers; a K slice (32 E4M3 or 16
      // FP16 values) starts 32 bytes further (2 in the descriptor's 16-byte
      // address units); FP16 queries continue in a second 128-byte-wide tile
      // NQ rows further for K >= 64.
      const uint64_t bdesc0 = desc_kmajor_sw128(smem_u32(qbuf));
      const uint64_t bdesc1 = desc_kmajor_sw128(smem_u32(qbuf + NQ * kQRow));
      constexpr uint64_t kHalf = (uint64_t)(NQ * 128 / 16);    // second K-half, descriptor units
      // Page k uses A buffer k % 2 and accumulator k % kND; with two
      // accumulators one commit (to acc_full[k % 2]) releases both.
      auto issue = [&](int k, int ab, int x, int& ends) -> bool {
        if (!mbar_wait(&a_full[ab], (k >> 1) & 1)) { report(a.flags, 5, 2); return false; }
        if (k >= kND && !mbar_wait(&acc_empty[x], ((k / kND) - 1) & 1)) { report(a.flags, 5, 3); return false; }
        tc_fence_after();
        const int what = tinfo[2 * ab];            // 0 = MMA, 1 = nothing to score, 2 = end
        ends += (what == 2);
        if (what == 0) {
          const uint32_t d = tmem + kACols + x * NQ;
          const uint32_t ta = tmem + ab * kABufCols;
          const uint64_t bd = tinfo[2 * ab + 1] ? bdesc1 : bdesc0;
          if constexpr (F16) {
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc_mma_f16_ts(d, ta + 8 * kk, bd + (kk >> 2) * kHalf + 2 * (kk & 3), idesc, kk > 0);
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc_mma_e4m3_ts(d, ta + 8 * kk, bd + 2 * kk, idesc, kk > 0);
          }
          if (MODE == kIdxNvfp4) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc_mma_e4m3_ts(d, ta + 32 + 8 * kk, bd + 2 * kk, idesc_neg, 1);
          }
        }
        if constexpr (kND == 2) {
          tc_commit(&acc_full[ab]);
        } else {
          tc_commit(&a_empty[ab]);
          tc_commit(&acc_full[x]);
        }
        return true;
      };
      int ends = 0;
      for (int k = 0; ends < 2; k += 2) {
        if (!issue(k, 0, 0, ends)) break;
        if (ends < 2 && !issue(k + 1, 1, kND == 2 ? 1 : 0, ends)) break;
      }
    }
  } else if (warp >= kIdxEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int quarter = warp & 3, group = (warp - kIdxEpiWarp0) >> 2;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);   // this warp's TMEM lanes
    const int g = lane >> 2, tq = lane & 3;
    // With two accumulators the groups alternate pages; with one (NQ >= 128)
    // group 0 takes every page, since a waiter two phases ahead of an
    // mbarrier would read its parity wrong.
    constexpr int kStep = kND == 2 ? 2 : 1;
    const bool active = kND == 2 || group == 0;
    for (int kk = group; active; kk += kStep) {
      const int xd = kk % kND, xe = group, jr = kk / kStep;   // jr: this group's page count
      if (!mbar_wait(&acc_full[xd], (kk / kND) & 1)) { report(a.flags, 5, 6); break; }
      tc_fence_after();
      const int* pf = pinfo + 8 * (kk & 3);
      const int pb = pf[0], pi = pf[1], pkind = pf[2], pL = pf[3];
      if (pkind == kPageEnd) {
        if (lane == 0) mbar_arrive(&acc_empty[xd]);
        break;
      }
      const int qbase = pf[4] * NQ;                // first index query of this page's tile
      const int t_first = qbase >> 2;
      if (pkind == kPageLoad) {
        const int pos0 = pL - a.T;
        const bool need_mask = pi * kBlock + kBlock - 1 > pos0 + t_first;
        // 16x256b loads: thread (g, t) holds keys g, g+8 (first load) and
        // g+16, g+24 (second) of this quarter's 32, columns 8c+2t and 8c+2t+1.
        constexpr int kR = kChunk / 8;                       // column groups per load
#pragma unroll 1
        for (int c0 = 0; c0 < NQ; c0 += kChunk) {
          float va[4 * kR], vb[4 * kR];
          tmem_ld_16x256b<kR>(lane_base + kACols + xd * NQ + c0, va);
          tmem_ld_16x256b<kR>(lane_base + (16u << 16) + kACols + xd * NQ + c0, vb);
          tmem_wait_ld();
          const int kb = pi * kBlock + 32 * quarter + g;     // key of va[.][0..1]
          if (need_mask) {   // keys after a query's position do not count
#pragma unroll
            for (int i = 0; i < 4 * kR; ++i) {
              const int col = c0 + 8 * (i >> 2) + 2 * tq + (i & 1);
              const int lim = pos0 + ((qbase + col) >> 2);
              const int dk = (i & 2) ? 8 : 0;
              if (kb + dk > lim) va[i] = -INFINITY;
              if (kb + 16 + dk > lim) vb[i] = -INFINITY;
            }
          }
          if (a.token_scores != nullptr) {
#pragma unroll
            for (int i = 0; i < 4 * kR; ++i) {
              const int col = c0 + 8 * (i >> 2) + 2 * tq + (i & 1);
              const int qg = qbase + col, t = qg >> 2;
              const int dk = (i & 2) ? 8 : 0;
              if (t < a.T) {
                float* rowp = a.token_scores + (((long long)pb * a.T + t) * kG + (qg & 3)) * ctx;
                rowp[kb + dk] = va[i] * a.score_scale;
                rowp[kb + 16 + dk] = vb[i] * a.score_scale;
              }
            }
          }
          // max over this thread's 4 keys, then over the 8 lane groups g
          float m[2 * kR];
#pragma unroll
          for (int c = 0; c < kR; ++c) {
#pragma unroll
            for (int e = 0; e < 2; ++e)
              m[2 * c + e] = fmaxf(fmax3(va[4 * c + e], va[4 * c + 2 + e], vb[4 * c + e]),
                                   vb[4 * c + 2 + e]);
          }
#pragma unroll
          for (int off = 4; off < 32; off <<= 1) {
#pragma unroll
            for (int i = 0; i < 2 * kR; ++i) m[i] = fmaxf(m[i], __shfl_xor_sync(0xffffffffu, m[i], off));
          }
          if (g == 0) {
            float* dst = red + (xe * kIdxEpilogue + quarter) * NQ + c0 + 2 * tq;
#pragma unroll
            for (int c = 0; c < kR; ++c) { dst[8 * c] = m[2 * c]; dst[8 * c + 1] = m[2 * c + 1]; }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      // rendezvous of the four quarters (bounded mbarrier wait), then each
      // warp combines a quarter of the columns
      if (lane == 0) mbar_arrive(&red_full[xe]);
      if (!mbar_wait(&red_full[xe], jr & 1)) { report(a.flags, 5, 7); break; }
      if (pkind != kPageBad) {
        constexpr int kPer = NQ / kIdxEpilogue;
        for (int j = lane; j < kPer; j += 32) {
          const int col = quarter * kPer + j;
          const int qg = qbase + col, t = qg >> 2;
          if (t >= a.T) continue;
          float m = -INFINITY;
          if (pkind == kPageLoad) {
#pragma unroll
            for (int w = 0; w < kIdxEpilogue; ++w) m = fmaxf(m, red[(xe * kIdxEpilogue + w) * NQ + col]);
          }
          a.block_scores[(((long long)pb * a.T + t) * kG + (qg & 3)) * a.max_pages + pi] =
              m * a.score_scale;
          if (pkind == kPageMasked && a.token_scores != nullptr) {
            float* rowp = a.token_scores + (((long long)pb * a.T + t) * kG + (qg & 3)) * ctx;
            for (int r = 0; r < kBlock; ++r) rowp[pi * kBlock + r] = -INFINITY;
          }
        }
      }
      __syncwarp();
      // The accumulator (and, through the MMA order, this page's partial
      // maxima and info slot) is released only after the combine: the MMA
      // that refills it waits for all four arrivals, so red[xe] is not
      // rewritten (page kk+2) before every warp has read it.
      if (lane == 0) mbar_arrive(&acc_empty[xd]);
    }
  } else {
    // ------------------------------------------------------------ decoders
    const int quarter = warp;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * quarter) << 16);   // this warp's TMEM lanes
    const int row = 32 * quarter + lane;                                  // key row of this thread
    int cur_b = -1, cur_y = -1, qsel = 1, L = 0, ends = 0;
    for (int k = 0; ends < 2; ++k) {
      const int s = k % kIdxRawStages, ab = k & 1;
      if (!mbar_wait(&raw_full[s], (k / kIdxRawStages) & 1)) { report(a.flags, 5, 5); break; }
      if (k >= 2 && !mbar_wait(kND == 2 ? &acc_full[ab] : &a_empty[ab], ((k >> 1) - 1) & 1)) {
        report(a.flags, 5, 4);
        break;
      }
      tc_fence_after();
      const int nb = meta[4 * s + 0], ni = meta[4 * s + 1], nkind = meta[4 * s + 2];
      const int ny = meta[4 * s + 3];
      ends += (nkind == kPageEnd);
      if (nkind != kPageEnd && (nb != cur_b || ny != cur_y)) {
        cur_b = nb;
        cur_y = ny;
        L = a.seq_lens[nb];
        qsel ^= 1;
        // B operand: the index queries of tile ny of sequence nb, swizzled
        // (its previous user, an MMA of page k-2 or earlier, has completed:
        // the wait above).
        uint8_t* qb = qbuf + qsel * NQ * kQRow;
        const int qbase = ny * NQ;
        for (int idx = warp * 32 + lane; idx < NQ * 8; idx += kIdxDecoders * 32) {
          const int nrow = idx / 8, c = idx % 8;
          const int qg = qbase + nrow, t = qg >> 2;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (t < a.T)
            v = *reinterpret_cast<const uint4*>(
                a.qi + (((long long)nb * a.T + t) * kG + (qg & 3)) * kDim + 16 * c);
          if constexpr (F16) {
            // dims 16c..16c+15 -> FP16 chunks 2c, 2c+1 of 8 dims: K-half c / 4,
            // chunk positions (2c % 8, 2c % 8 + 1) ^ (row % 8) in its 128-byte row
            const uint4 lo = make_uint4(e4m3x2_to_f16x2(v.x), e4m3x2_to_f16x2(v.x >> 16),
                                        e4m3x2_to_f16x2(v.y), e4m3x2_to_f16x2(v.y >> 16));
            const uint4 hi = make_uint4(e4m3x2_to_f16x2(v.z), e4m3x2_to_f16x2(v.z >> 16),
                                        e4m3x2_to_f16x2(v.w), e4m3x2_to_f16x2(v.w >> 16));
            uint8_t* rowp = qb + (c >> 2) * NQ * 128 + nrow * 128;
            const int j = (2 * c) & 7;
            sts128(rowp + ((j ^ (nrow & 7)) << 4), lo);
            sts128(rowp + (((j + 1) ^ (nrow & 7)) << 4), hi);
          } else {
            sts128(qb + nrow * 128 + ((c ^ (nrow & 7)) << 4), v);
          }
        }
        fence_async_smem();
      }
      if (nkind == kPageLoad) {
        const uint8_t* rs = raw + s * Ly.raw_stride;
        const uint32_t abase = lane_base + ab * kABufCols;
        if constexpr (FP8IDX) {
          // 128-byte rows loaded with the 128-byte swizzle: chunk c of row r
          // sits at chunk position c ^ (r % 8).
#pragma unroll
          for (int c2 = 0; c2 < 4; ++c2) {
            const uint4 x0 = lds128(rs + row * 128 + (((2 * c2) ^ (row & 7)) << 4));
            const uint4 x1 = lds128(rs + row * 128 + (((2 * c2 + 1) ^ (row & 7)) << 4));
            const uint32_t w8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
            tmem_st8(abase + 8 * c2, w8);
          }
        } else if constexpr (F16) {
          // 64-byte code rows (64-byte swizzle, as below); chunk c = elements
          // 32c..32c+31 under scale bytes 2c and 2c+1 -> FP16 columns 16c..16c+15
          const uint2 sc = *reinterpret_cast<const uint2*>(rs + kPageCodes + row * kRowScales);
          const int sw = (row >> 1) & 3;
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
            for (int m = 0; m < 16; ++m) o[m] = hmul2(o[m], m < 8 ? s_lo : s_hi);
            tmem_st16(abase + 16 * c, o);
          }
        } else {
          // 64-byte code rows loaded with the 64-byte swizzle: chunk c of
          // row r sits at chunk position c ^ ((r / 2) % 4).
          const uint2 sc = *reinterpret_cast<const uint2*>(rs + kPageCodes + row * kRowScales);
          const int sw = (row >> 1) & 3;
          // warp-uniform branch: tcgen05.st is a .sync.aligned warp instruction
          if (__all_sync(0xffffffffu, ((sc.x | sc.y) & 0x80808080u) == 0u)) {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 w4 = lds128(rs + row * kRowCodes + ((c ^ sw) << 4));
              const uint32_t sb = (c < 2 ? sc.x : sc.y) >> (16 * (c & 1));   // scales 2c, 2c+1
              const uint2 r0 = lut[sb & 0xFFu], r1 = lut[(sb >> 8) & 0xFFu];
              uint32_t pw[8], nw[8];
              dq8_split_pos(w4.x, r0, pw[0], pw[1], nw[0], nw[1]);
              dq8_split_pos(w4.y, r0, pw[2], pw[3], nw[2], nw[3]);
              dq8_split_pos(w4.z, r1, pw[4], pw[5], nw[4], nw[5]);
              dq8_split_pos(w4.w, r1, pw[6], pw[7], nw[6], nw[7]);
              tmem_st8(abase + 8 * c, pw);
              tmem_st8(abase + 32 + 8 * c, nw);
            }
          } else {
#pragma unroll
            for (int c = 0; c < 4; ++c) {
              const uint4 w4 = lds128(rs + row * kRowCodes + ((c ^ sw) << 4));
              const uint32_t sb = (c < 2 ? sc.x : sc.y) >> (16 * (c & 1));
              const uint32_t s0 = sb & 0xFFu, s1 = (sb >> 8) & 0xFFu;
              const uint2 r0 = lut[s0 & 0x7Fu], r1 = lut[s1 & 0x7Fu];
              const uint32_t f0 = (s0 & 0x80u) ? 0x88888888u : 0u;
              const uint32_t f1 = (s1 & 0x80u) ? 0x88888888u : 0u;
              uint32_t pw[8], nw[8];
              dq8_split(w4.x, r0, f0, pw[0], pw[1], nw[0], nw[1]);
              dq8_split(w4.y, r0, f0, pw[2], pw[3], nw[2], nw[3]);
              dq8_split(w4.z, r1, f1, pw[4], pw[5], nw[4], nw[5]);
              dq8_split(w4.w, r1, f1, pw[6], pw[7], nw[6], nw[7]);
              tmem_st8(abase + 8 * c, pw);
              tmem_st8(abase + 32 + 8 * c, nw);
            }
          }
        }
        tmem_wait_st();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(&raw_empty[s]);
        if (warp == 0) {
          tinfo[2 * ab] = nkind == kPageEnd ? 2 : (nkind != kPageLoad);
          tinfo[2 * ab + 1] = qsel;
          int* pf = pinfo + 8 * (k & 3);
          pf[0] = nb; pf[1] = ni; pf[2] = nkind; pf[3] = L; pf[4] = ny;
        }
        mbar_arrive(&a_full[ab]);
      }
    }
  }

  // ---- teardown: every role leaves its loop (normally or on a timeout)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kIdxMmaWarp) tmem_dealloc(tmem, kCols);
}

template <int NQ, int MODE>
static cudaError_t launch_nq(const IdxArgs& a, int num_sms, cudaStream_t st) {
  auto kern = indexer_kernel<NQ, MODE>;
  const size_t smem = (size_t)idx_layout(NQ, MODE, a.B).total;
  static size_t configured = 0;
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), kIdxThreads, smem,
                                 pow2_at_least(kACols + (NQ <= 64 ? 2 : 1) * NQ));
  const int gx = num_sms * per_sm;              // persistent: items are claimed in the kernel
  kern<<<gx, kIdxThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(const IdxArgs& a, int mode, int num_sms, cudaStream_t st) {
  const int nq = idx_nq(a.T);
#define MSA_IDX_CASE(NQV)                                                     \
  if (nq == NQV) {                                                            \
    if (mode == kIdxFp8) return launch_nq<NQV, kIdxFp8>(a, num_sms, st);      \
    if (mode == kIdxF16) return launch_nq<NQV, kIdxF16>(a, num_sms, st);      \
    return launch_nq<NQV, kIdxNvfp4>(a, num_sms, st);                         \
  }
  MSA_IDX_CASE(16)
  MSA_IDX_CASE(32)
  MSA_IDX_CASE(64)
  MSA_IDX_CASE(128)
  MSA_IDX_CASE(256)
#undef MSA_IDX_CASE
  return cudaErrorInvalidValue;
}

}  // namespace msa
