// msa_indexer.cu -- indexer scores + block max-pool on the 5th-generation
// tensor core ([post, "MSA primer"]: one index query per GQA group scores
// every cached key against one shared index-key head; the scores are
// max-pooled to one score per 128-token block).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Per page (= one 128-token block) the scores are one dense FP8 contraction
//   D[128 keys x NQ queries] = K_page[128 x 128] * Qi[NQ x 128]^T
// with the keys as the M side (the block max is a reduction over TMEM
// lanes) and a chunk of NQ index queries (T tokens x 4 groups, padded to a
// multiple of 8) as the N side.
//
// Work split: the pages of all sequences form one flat list; CTA x takes one
// contiguous slice of it (even load for ragged lengths); grid y tiles the
// index queries in chunks of NQ.  Warp roles inside a CTA:
//   warp 4 (producer): per page one tiled TMA load of the codes (64-byte
//     swizzle, so that row-per-thread reads are bank-conflict free) and one
//     bulk copy of the scales into a ring of shared-memory stages;
//   warps 0-3 (workers): thread = key row (= TMEM lane).  NVFP4 rows are
//     decoded by sign: K+ holds E4M3(|v|) of the positive elements, K- of the
//     negative ones (one prmt per 4 codes each, see dq8_split), and both go
//     straight to tensor memory with tcgen05.st -- the A operand never
//     touches shared memory.  One page behind, the workers read the
//     accumulator from TMEM, mask keys after each query's position and
//     reduce the 128 keys with redux.sync.max.f32 (combining the four warps'
//     partial maxima in shared memory);
//   warp 5 (MMA): one thread issues per page 4 tcgen05.mma with A = K+ and 4
//     with A = K- and the negate-A bit (K = 32 each, A from TMEM, B = the
//     queries in shared memory) into a double-buffered TMEM accumulator.
// Every wait is a bounded mbarrier wait; on a timeout a thread records
// MSA_ERR_TIMEOUT and leaves its loop, and TMEM is freed before exit.
#include "msa_internal.h"

namespace msa {

constexpr int kIdxWorkers = 4;
constexpr int kIdxProducerWarp = 4;
constexpr int kIdxMmaWarp = 5;
constexpr int kACols = 64;                  // TMEM columns of the A operand (K+ | K-)

enum : int { kPageLoad = 0, kPageMasked = 1, kPageBad = 2 };

struct IdxLayout {
  int qbuf, raw, raw_stride, lut, red, bars, meta, tinfo, cnt, tslot, prefix, scratch, total;
};

// Bytes of one raw page in shared memory (codes [+ scales]), 1024-aligned.
__host__ __device__ inline int raw_stage_stride(bool fp8idx) {
  return fp8idx ? kBlock * kDim : ((kPageCodes + kPageScales + 1023) / 1024) * 1024;
}

__host__ __device__ inline IdxLayout idx_layout(int nq, bool fp8idx, int batch) {
  IdxLayout L;
  int off = 0;
  L.qbuf = off;    off += 2 * nq * 128;                   // nq % 8 == 0 -> 1024-aligned
  L.raw_stride = raw_stage_stride(fp8idx);
  L.raw = off;     off += kIdxRawStages * L.raw_stride;
  L.lut = off;     off += 256 * 8;
  L.red = off;     off += 2 * kIdxWorkers * nq * 4;
  L.bars = off;    off += (2 * kIdxRawStages + 6) * 8;
  L.meta = off;    off += 3 * kIdxRawStages * 4;
  L.tinfo = off;   off += 4 * 4;
  L.cnt = off;     off += 2 * 4;
  L.tslot = off;   off += 16;
  L.prefix = off;  off += (batch + 1) * 4;
  L.scratch = off; off += kIdxThreads * 4;
  L.total = off + 1024;                                   // alignment slack
  return L;
}

int idx_nq(int T) {
  const int nq = kG * T;
  if (nq <= 8) return 8;
  if (nq <= 16) return 16;
  if (nq <= 32) return 32;
  if (nq <= 64) return 64;
  if (nq <= 128) return 128;
  return 256;
}

size_t indexer_smem_bytes(bool fp8idx, int batch, int T) {
  return (size_t)idx_layout(idx_nq(T), fp8idx, batch).total;
}

__host__ __device__ constexpr int pow2_at_least(int x) {
  int p = 32;
  while (p < x) p *= 2;
  return p;
}

// Exclusive prefix over the number of blocks of each sequence, in shared
// memory (prefix[B] = total pages).  Invalid lengths count as 0 blocks and
// are reported once (by CTA (0,0)).
__device__ void page_prefix(const IdxArgs& a, int* prefix, int* scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int per = (a.B + nt - 1) / nt;
  const int lo = tid * per, hi = min(a.B, lo + per);
  int sum = 0;
  for (int b = lo; b < hi; ++b) {
    const int L = a.seq_lens[b];
    int nb = 0;
    if (L >= a.T && L <= a.max_pages * kBlock) {
      nb = (L + kBlock - 1) / kBlock;
    } else if (blockIdx.x == 0 && blockIdx.y == 0) {
      report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
    }
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
    const int L = a.seq_lens[b];
    run += (L >= a.T && L <= a.max_pages * kBlock) ? (L + kBlock - 1) / kBlock : 0;
  }
  __syncthreads();
}

__device__ __forceinline__ void sts128(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

template <int NQ, bool FP8IDX>
__global__ void __launch_bounds__(kIdxThreads, 4) indexer_kernel(const __grid_constant__ IdxArgs a) {
  constexpr int kND = NQ <= 64 ? 2 : 1;                      // accumulator buffers
  constexpr int kCols = pow2_at_least(kACols + kND * NQ);    // TMEM columns
  constexpr int kChunk = NQ < 32 ? NQ : 32;                  // columns per TMEM load
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
  const IdxLayout Ly = idx_layout(NQ, FP8IDX, a.B);
  uint8_t* qbuf = smem + Ly.qbuf;
  uint8_t* raw = smem + Ly.raw;
  uint2* lut = reinterpret_cast<uint2*>(smem + Ly.lut);
  float* red = reinterpret_cast<float*>(smem + Ly.red);            // [2][4][NQ]
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* raw_empty = raw_full + kIdxRawStages;
  uint64_t* a_full = raw_empty + kIdxRawStages;                    // workers -> MMA
  uint64_t* a_empty = a_full + 1;                                  // MMA -> workers
  uint64_t* acc_full = a_empty + 1;                                // MMA -> workers [2]
  uint64_t* acc_empty = acc_full + 2;                              // workers -> MMA [2]
  int* meta = reinterpret_cast<int*>(smem + Ly.meta);              // [stage][b, i, kind]
  int* tinfo = reinterpret_cast<int*>(smem + Ly.tinfo);            // [skip, qsel]
  int* cnt = reinterpret_cast<int*>(smem + Ly.cnt);                // [2]
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly.tslot);
  int* prefix = reinterpret_cast<int*>(smem + Ly.prefix);
  int* scratch = reinterpret_cast<int*>(smem + Ly.scratch);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (!FP8IDX) build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < kIdxRawStages; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], kIdxWorkers);
    }
    mbar_init(a_full, kIdxWorkers);
    mbar_init(a_empty, 1);
    for (int x = 0; x < 2; ++x) {
      mbar_init(&acc_full[x], 1);
      mbar_init(&acc_empty[x], kIdxWorkers);
      cnt[x] = 0;
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
  const int lo = (int)((long long)total * blockIdx.x / gridDim.x);
  const int hi = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
  const int n = hi - lo;
  const int qbase = blockIdx.y * NQ;           // first index query of this chunk
  const int t_first = qbase >> 2;
  const int t_last = min(a.T - 1, (qbase + NQ - 1) >> 2);
  const long long ctx = (long long)a.max_pages * kBlock;

  if (warp == kIdxProducerWarp) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      int b;
      {  // prefix[b] <= lo < prefix[b+1]
        int l = 0, r = a.B;
        while (r - l > 1) { const int m = (l + r) >> 1; if (prefix[m] <= lo) l = m; else r = m; }
        b = l;
      }
      int i = lo - prefix[b];
      for (int k = 0; k < n; ++k) {
        const int s = k % kIdxRawStages;
        if (k >= kIdxRawStages && !mbar_wait(&raw_empty[s], ((k / kIdxRawStages) - 1) & 1)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1);
          break;
        }
        while (i >= prefix[b + 1] - prefix[b]) { i -= prefix[b + 1] - prefix[b]; ++b; }
        const int L = a.seq_lens[b];
        int kind = kPageLoad;
        const long long p = a.page_table ? (long long)a.page_table[(long long)b * a.max_pages + i]
                                         : (long long)b * a.max_pages + i;
        if (i * kBlock > L - a.T + t_last) {
          kind = kPageMasked;
        } else if (p < 0 || p >= a.num_pages) {
          report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)p);
          kind = kPageBad;
        }
        meta[3 * s + 0] = b;
        meta[3 * s + 1] = i;
        meta[3 * s + 2] = kind;
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
        ++i;
      }
    }
  } else if (warp == kIdxMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc = idesc_e4m3_f32(128, NQ);
      constexpr uint32_t idesc_neg = idesc | (1u << 13);     // negate A
      for (int k = 0; k < n; ++k) {
        const int x = k % kND;
        if (!mbar_wait(a_full, k & 1)) { report(a.flags, 5, 2); break; }
        if (k >= kND && !mbar_wait(&acc_empty[x], ((k / kND) - 1) & 1)) { report(a.flags, 5, 3); break; }
        tc_fence_after();
        if (!tinfo[0]) {
          const uint32_t d = tmem + kACols + x * NQ;
          const uint32_t b0 = smem_u32(qbuf + tinfo[1] * NQ * 128);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            tc_mma_e4m3_ts(d, tmem + 8 * kk, desc_kmajor_sw128(b0 + 32 * kk), idesc, kk > 0);
          if (!FP8IDX) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              tc_mma_e4m3_ts(d, tmem + 32 + 8 * kk, desc_kmajor_sw128(b0 + 32 * kk), idesc_neg, 1);
          }
        }
        tc_commit(a_empty);
        tc_commit(&acc_full[x]);
      }
    }
  } else {
    // ------------------------------------------------------------ workers
    const uint32_t lane_base = tmem + ((uint32_t)(32 * warp) << 16);   // this warp's TMEM lanes
    const int row = 32 * warp + lane;                                   // key row of this thread
    // Epilogue of page kk (accumulator buffer kk % kND).
    auto epilogue = [&](int kk, int pb, int pi, int pkind, int pL) -> bool {
      const int xd = kk % kND, xe = kk & 1;
      if (!mbar_wait(&acc_full[xd], (kk / kND) & 1)) { report(a.flags, 5, 6); return false; }
      tc_fence_after();
      if (pkind == kPageLoad) {
        const int pos0 = pL - a.T;
        const bool need_mask = pi * kBlock + kBlock - 1 > pos0 + t_first;
        // 16x256b loads: thread (g, t) holds keys g, g+8 (first load) and
        // g+16, g+24 (second) of this warp's 32, columns 8c+2t and 8c+2t+1.
        constexpr int kR = kChunk / 8;                       // column groups per load
        const int g = lane >> 2, tq = lane & 3;
#pragma unroll 1
        for (int c0 = 0; c0 < NQ; c0 += kChunk) {
          float va[4 * kR], vb[4 * kR];
          tmem_ld_16x256b<kR>(lane_base + kACols + xd * NQ + c0, va);
          tmem_ld_16x256b<kR>(lane_base + (16u << 16) + kACols + xd * NQ + c0, vb);
          tmem_wait_ld();
          const int kb = pi * kBlock + 32 * warp + g;        // key of va[.][0..1]
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
            float* dst = red + (xe * kIdxWorkers + warp) * NQ + c0 + 2 * tq;
#pragma unroll
            for (int c = 0; c < kR; ++c) { dst[8 * c] = m[2 * c]; dst[8 * c + 1] = m[2 * c + 1]; }
          }
        }
      }
      tc_fence_before();
      __syncwarp();
      int last = 0;
      if (lane == 0) {
        mbar_arrive(&acc_empty[xd]);
        __threadfence_block();
        last = (atomicAdd(&cnt[xe], 1) == kIdxWorkers - 1);
      }
      last = __shfl_sync(0xffffffffu, last, 0);
      if (last) {   // the last warp of this page combines the four partial maxima
        __threadfence_block();
        if (pkind != kPageBad) {
          for (int col = lane; col < NQ; col += 32) {
            const int qg = qbase + col, t = qg >> 2;
            if (t >= a.T) continue;
            float m = -INFINITY;
            if (pkind == kPageLoad) {
#pragma unroll
              for (int w = 0; w < kIdxWorkers; ++w)
                m = fmaxf(m, red[(xe * kIdxWorkers + w) * NQ + col]);
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
        if (lane == 0) cnt[xe] = 0;
      }
      return true;
    };

    int cur_b = -1, qsel = 1, L = 0;
    int pb = 0, pi = 0, pkind = kPageBad, pL = 0;   // the page one behind
    for (int k = 0; k <= n; ++k) {
      int nb = 0, ni = 0, nkind = kPageBad;
      if (k < n) {
        // ---- decode page k into the A operand in TMEM
        const int s = k % kIdxRawStages;
        if (!mbar_wait(&raw_full[s], (k / kIdxRawStages) & 1)) { report(a.flags, 5, 5); break; }
        if (k >= 1 && !mbar_wait(a_empty, (k - 1) & 1)) { report(a.flags, 5, 4); break; }
        tc_fence_after();
        nb = meta[3 * s + 0];
        ni = meta[3 * s + 1];
        nkind = meta[3 * s + 2];
        if (nb != cur_b) {
          cur_b = nb;
          L = a.seq_lens[nb];
          qsel ^= 1;
          // B operand: the query rows of this chunk for sequence nb, swizzled
          // (its previous user, an MMA of page k-2 or earlier, has completed).
          uint8_t* qb = qbuf + qsel * NQ * 128;
          constexpr int kRowsPerWarp = NQ / kIdxWorkers;
          for (int idx = lane; idx < kRowsPerWarp * 8; idx += 32) {
            const int nrow = warp * kRowsPerWarp + idx / 8, c = idx % 8;
            const int qg = qbase + nrow, t = qg >> 2;
            uint4 v = make_uint4(0u, 0u, 0u, 0u);
            if (t < a.T)
              v = *reinterpret_cast<const uint4*>(
                  a.qi + (((long long)nb * a.T + t) * kG + (qg & 3)) * kDim + 16 * c);
            sts128(qb + nrow * 128 + ((c ^ (nrow & 7)) << 4), v);
          }
          fence_async_smem();
        }
        if (nkind == kPageLoad) {
          const uint8_t* rs = raw + s * Ly.raw_stride;
          if constexpr (FP8IDX) {
            // 128-byte rows loaded with the 128-byte swizzle: chunk c of row r
            // sits at chunk position c ^ (r % 8).
#pragma unroll
            for (int c2 = 0; c2 < 4; ++c2) {
              const uint4 x0 = lds128(rs + row * 128 + (((2 * c2) ^ (row & 7)) << 4));
              const uint4 x1 = lds128(rs + row * 128 + (((2 * c2 + 1) ^ (row & 7)) << 4));
              const uint32_t w8[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
              tmem_st8(lane_base + 8 * c2, w8);
            }
          } else {
            // 64-byte code rows loaded with the 64-byte swizzle: chunk c of
            // row r sits at chunk position c ^ ((r / 2) % 4).
            const uint2 sc = *reinterpret_cast<const uint2*>(rs + kPageCodes + row * kRowScales);
            const int sw = (row >> 1) & 3;
            // warp-uniform branch: tcgen05.st is a .sync.aligned warp instruction
            if (__all_sync(0xffffffffu, ((sc.x | sc.y) & 0x80808080u) == 0u)) {
              // every block scale of the warp's 32 rows is non-negative
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
                tmem_st8(lane_base + 8 * c, pw);
                tmem_st8(lane_base + 32 + 8 * c, nw);
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
                tmem_st8(lane_base + 8 * c, pw);
                tmem_st8(lane_base + 32 + 8 * c, nw);
              }
            }
          }
          tmem_wait_st();
        }
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          mbar_arrive(&raw_empty[s]);
          if (warp == 0) { tinfo[0] = (nkind != kPageLoad); tinfo[1] = qsel; }
          mbar_arrive(a_full);
        }
      }
      // ---- epilogue of page k-1 (its MMA ran while page k was decoded)
      if (k >= 1 && !epilogue(k - 1, pb, pi, pkind, pL)) break;
      pb = nb; pi = ni; pkind = nkind; pL = L;
    }
  }

  // ---- teardown: every role leaves its loop (normally or on a timeout)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kIdxMmaWarp) tmem_dealloc(tmem, kCols);
}

template <int NQ, bool FP8IDX>
static cudaError_t launch_nq(const IdxArgs& a, int num_sms, cudaStream_t st) {
  auto kern = indexer_kernel<NQ, FP8IDX>;
  const size_t smem = (size_t)idx_layout(NQ, FP8IDX, a.B).total;
  static size_t configured = 0;
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  const int per_sm = ctas_per_sm(reinterpret_cast<const void*>(kern), kIdxThreads, smem,
                                 pow2_at_least(kACols + (NQ <= 64 ? 2 : 1) * NQ));
  const int gy = (kG * a.T + NQ - 1) / NQ;
  const long long want = ((long long)num_sms * per_sm + gy - 1) / gy;
  const long long cap = (long long)a.B * a.max_pages;
  const int gx = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  kern<<<dim3(gx, gy), kIdxThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(const IdxArgs& a, bool fp8idx, int num_sms, cudaStream_t st) {
  const int nq = idx_nq(a.T);
#define MSA_IDX_CASE(NQV)                                                     \
  if (nq == NQV)                                                              \
    return fp8idx ? launch_nq<NQV, true>(a, num_sms, st) : launch_nq<NQV, false>(a, num_sms, st);
  MSA_IDX_CASE(8)
  MSA_IDX_CASE(16)
  MSA_IDX_CASE(32)
  MSA_IDX_CASE(64)
  MSA_IDX_CASE(128)
  MSA_IDX_CASE(256)
#undef MSA_IDX_CASE
  return cudaErrorInvalidValue;
}

}  // namespace msa
