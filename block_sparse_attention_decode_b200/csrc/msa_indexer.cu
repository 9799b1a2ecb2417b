// msa_indexer.cu -- indexer scores + block max-pool ([post, "MSA primer"]:
// one index query per GQA group scores every cached key against one shared
// index-key head; the scores are max-pooled to one score per 128-token block).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Work split.  The index-key pages of all sequences form one flat list
// (sequence-major); each CTA of the grid's x dimension takes one contiguous
// slice of it, so the load is even however ragged the lengths are.  The y
// dimension tiles the index queries (T tokens x 4 groups) in chunks of 8*NT.
//
// Per CTA: one producer warp streams whole pages (8 KB codes + 1 KB scales,
// or 16 KB FP8 keys) into a ring of shared-memory stages with bulk async
// copies completing on mbarriers; four consumer warps each own every fourth
// page.  A consumer decodes the page straight into FP8 MMA fragments (keys
// are the M side, 16 per fragment; queries the N side), runs
// m16n8k32 e4m3 MMAs, masks keys after each query's position, and reduces
// the 128 keys of the page to one block maximum in registers -- token scores
// never reach global memory unless the caller asks for them.
#include "msa_internal.h"

namespace msa {

template <bool FP8IDX>
struct IdxStage {
  static constexpr int kBytes = FP8IDX ? kBlock * kDim : kPageCodes + kPageScales;
};

// Per-page metadata handed from the producer to the consumer of a stage.
enum : int { kPageLoad = 0, kPageMasked = 1, kPageBad = 2 };

size_t indexer_smem_bytes(bool fp8idx, int batch) {
  const int stage = fp8idx ? IdxStage<true>::kBytes : IdxStage<false>::kBytes;
  return (size_t)kIdxStages * stage + 256 * sizeof(uint2) + 2 * kIdxStages * sizeof(uint64_t) +
         3 * kIdxStages * sizeof(int) + (size_t)(batch + 1) * sizeof(int) +
         kIdxThreads * sizeof(int) + 64;
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

template <int NT, bool FP8IDX>
__global__ void __launch_bounds__(kIdxThreads) indexer_kernel(IdxArgs a) {
  constexpr int kStage = IdxStage<FP8IDX>::kBytes;
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint2* lut = reinterpret_cast<uint2*>(smem + kIdxStages * kStage);
  uint64_t* full = reinterpret_cast<uint64_t*>(lut + 256);
  uint64_t* empty = full + kIdxStages;
  int* meta = reinterpret_cast<int*>(empty + kIdxStages);   // [stage][b, i, kind]
  int* prefix = meta + 3 * kIdxStages;                       // [B + 1]
  int* scratch = prefix + a.B + 1;                           // [kIdxThreads]

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;

  build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < kIdxStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], 1); }
    mbar_fence_init();
  }
  page_prefix(a, prefix, scratch);   // contains __syncthreads

  const int total = prefix[a.B];
  const int lo = (int)((long long)total * blockIdx.x / gridDim.x);
  const int hi = (int)((long long)total * (blockIdx.x + 1) / gridDim.x);
  const int n = hi - lo;
  const int qbase = blockIdx.y * 8 * NT;          // first index query of this chunk
  const int t_first = qbase >> 2;
  const int t_last = min(a.T - 1, (qbase + 8 * NT - 1) >> 2);

  if (warp == kIdxConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0 && n > 0) {
      int b = 0;
      {  // first sequence whose pages reach index lo: prefix[b] <= lo < prefix[b+1]
        int l = 0, r = a.B;
        while (r - l > 1) { const int m = (l + r) >> 1; if (prefix[m] <= lo) l = m; else r = m; }
        b = l;
      }
      int i = lo - prefix[b];
      for (int k = 0; k < n; ++k) {
        const int s = k % kIdxStages;
        if (k >= kIdxStages && !mbar_wait(&empty[s], ((k / kIdxStages) - 1) & 1)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, k);
          break;
        }
        while (i >= prefix[b + 1] - prefix[b]) { i -= prefix[b + 1] - prefix[b]; ++b; }
        const int L = a.seq_lens[b];
        const int max_pos = L - a.T + t_last;
        int kind = kPageLoad;
        long long p = a.page_table ? (long long)a.page_table[(long long)b * a.max_pages + i]
                                   : (long long)b * a.max_pages + i;
        if (i * kBlock > max_pos) {
          kind = kPageMasked;
        } else if (p < 0 || p >= a.num_pages) {
          report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)p);
          kind = kPageBad;
        }
        meta[3 * s + 0] = b;
        meta[3 * s + 1] = i;
        meta[3 * s + 2] = kind;
        uint8_t* dst = stages + s * kStage;
        if (kind == kPageLoad) {
          mbar_expect_tx(&full[s], kStage);
          if (FP8IDX) {
            bulk_g2s(dst, a.idx_data + p * (kBlock * kDim), kBlock * kDim, &full[s]);
          } else {
            bulk_g2s(dst, a.idx_data + p * kPageCodes, kPageCodes, &full[s]);
            bulk_g2s(dst + kPageCodes, a.idx_scale + p * kPageScales, kPageScales, &full[s]);
          }
        } else {
          mbar_arrive(&full[s]);
        }
        ++i;
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    uint32_t qf[NT][8];
    int cur_b = -1, L = 0;
    for (int k = warp; k < n; k += kIdxConsumers) {
      const int s = k % kIdxStages;
      if (!mbar_wait(&full[s], (k / kIdxStages) & 1)) {
        report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, k);
        break;
      }
      const int b = meta[3 * s + 0], i = meta[3 * s + 1], kind = meta[3 * s + 2];
      if (b != cur_b) {
        cur_b = b;
        L = a.seq_lens[b];
        // B fragments: column gid of n-tile j = index query qbase + 8j + gid;
        // this thread holds its elements 32*tig .. 32*tig+31.
#pragma unroll
        for (int j = 0; j < NT; ++j) {
          const int qg = qbase + 8 * j + gid;
          const int t = qg >> 2;
          if (t < a.T) {
            const uint8_t* src = a.qi + (((long long)b * a.T + t) * kG + (qg & 3)) * kDim + 32 * tig;
            const uint4 x0 = *reinterpret_cast<const uint4*>(src);
            const uint4 x1 = *reinterpret_cast<const uint4*>(src + 16);
            qf[j][0] = x0.x; qf[j][1] = x0.y; qf[j][2] = x0.z; qf[j][3] = x0.w;
            qf[j][4] = x1.x; qf[j][5] = x1.y; qf[j][6] = x1.z; qf[j][7] = x1.w;
          } else {
#pragma unroll
            for (int m = 0; m < 8; ++m) qf[j][m] = 0u;
          }
        }
      }
      const int pos0 = L - a.T;       // position of token 0
      const long long ctx = (long long)a.max_pages * kBlock;
      if (kind == kPageLoad) {
        const uint8_t* sd = stages + s * kStage;
        const bool need_mask = (i * kBlock + kBlock - 1) > (pos0 + t_first);
        float bm[NT][2];
#pragma unroll
        for (int j = 0; j < NT; ++j) { bm[j][0] = -INFINITY; bm[j][1] = -INFINITY; }
#pragma unroll 1
        for (int mt = 0; mt < kBlock / 16; ++mt) {
          const int r0 = 16 * mt + gid, r1 = r0 + 8;
          uint32_t k0[8], k1[8];
          if (FP8IDX) {
            const uint4 x0 = lds128(sd + r0 * kDim + 32 * tig), x1 = lds128(sd + r0 * kDim + 32 * tig + 16);
            const uint4 y0 = lds128(sd + r1 * kDim + 32 * tig), y1 = lds128(sd + r1 * kDim + 32 * tig + 16);
            k0[0] = x0.x; k0[1] = x0.y; k0[2] = x0.z; k0[3] = x0.w;
            k0[4] = x1.x; k0[5] = x1.y; k0[6] = x1.z; k0[7] = x1.w;
            k1[0] = y0.x; k1[1] = y0.y; k1[2] = y0.z; k1[3] = y0.w;
            k1[4] = y1.x; k1[5] = y1.y; k1[6] = y1.z; k1[7] = y1.w;
          } else {
            const uint8_t* ss = sd + kPageCodes;
            dq32(lut, lds128(sd + r0 * kRowCodes + 16 * tig), lds16(ss + r0 * kRowScales + 2 * tig), k0);
            dq32(lut, lds128(sd + r1 * kRowCodes + 16 * tig), lds16(ss + r1 * kRowScales + 2 * tig), k1);
          }
          float acc[NT][4];
#pragma unroll
          for (int j = 0; j < NT; ++j) { acc[j][0] = acc[j][1] = acc[j][2] = acc[j][3] = 0.f; }
#pragma unroll
          for (int ks = 0; ks < 4; ++ks) {
#pragma unroll
            for (int j = 0; j < NT; ++j)
              mma_e4m3(acc[j], k0[2 * ks], k1[2 * ks], k0[2 * ks + 1], k1[2 * ks + 1],
                       qf[j][2 * ks], qf[j][2 * ks + 1]);
          }
#pragma unroll
          for (int j = 0; j < NT; ++j) {
#pragma unroll
            for (int e = 0; e < 4; ++e) {
              const int row = (e < 2) ? r0 : r1;
              const int qg = qbase + 8 * j + 2 * tig + (e & 1);
              const int t = qg >> 2;
              const int key = i * kBlock + row;
              float v = acc[j][e];
              if (need_mask && (t >= a.T || key > pos0 + t)) v = -INFINITY;
              if (a.token_scores && t < a.T)
                a.token_scores[(((long long)cur_b * a.T + t) * kG + (qg & 3)) * ctx + key] =
                    v * a.score_scale;
              bm[j][e & 1] = fmaxf(bm[j][e & 1], v);
            }
          }
        }
        // max over the 8 lanes that share tig (rows gid = 0..7)
#pragma unroll
        for (int j = 0; j < NT; ++j) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            float v = bm[j][c];
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 4));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 8));
            v = fmaxf(v, __shfl_xor_sync(0xffffffffu, v, 16));
            bm[j][c] = v;
          }
        }
        if (gid == 0) {
#pragma unroll
          for (int j = 0; j < NT; ++j) {
#pragma unroll
            for (int c = 0; c < 2; ++c) {
              const int qg = qbase + 8 * j + 2 * tig + c;
              const int t = qg >> 2;
              if (t < a.T)
                a.block_scores[(((long long)cur_b * a.T + t) * kG + (qg & 3)) * a.max_pages + i] =
                    bm[j][c] * a.score_scale;
            }
          }
        }
      } else if (kind == kPageMasked) {
        // no key of this page is visible to any query of the chunk
        for (int c = lane; c < 8 * NT; c += 32) {
          const int qg = qbase + c, t = qg >> 2;
          if (t < a.T)
            a.block_scores[(((long long)cur_b * a.T + t) * kG + (qg & 3)) * a.max_pages + i] =
                -INFINITY;
        }
        if (a.token_scores) {
          for (int c = 0; c < 8 * NT; ++c) {
            const int qg = qbase + c, t = qg >> 2;
            if (t >= a.T) break;
            float* row = a.token_scores + (((long long)cur_b * a.T + t) * kG + (qg & 3)) * ctx;
            for (int r = lane; r < kBlock; r += 32) row[i * kBlock + r] = -INFINITY;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);
    }
  }
}

template <int NT, bool FP8IDX>
static cudaError_t launch_nt(const IdxArgs& a, int gx, int gy, size_t smem, cudaStream_t st) {
  auto kern = indexer_kernel<NT, FP8IDX>;
  static size_t configured = 0;
  if (configured < smem) {
    cudaError_t e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
    configured = smem;
  }
  kern<<<dim3(gx, gy), kIdxThreads, smem, st>>>(a);
  return cudaGetLastError();
}

int indexer_ntiles(int T) {
  const int nq = kG * T;
  return nq <= 8 ? 1 : (nq <= 16 ? 2 : 4);
}

cudaError_t launch_indexer(const IdxArgs& a, bool fp8idx, int num_sms, cudaStream_t st) {
  const int NT = indexer_ntiles(a.T);
  const int gy = (kG * a.T + 8 * NT - 1) / (8 * NT);
  const size_t smem = indexer_smem_bytes(fp8idx, a.B);
  // CTAs resident per SM for this shared-memory footprint (at most 3)
  int per_sm = (int)((220 * 1024) / smem);
  per_sm = per_sm < 1 ? 1 : (per_sm > 3 ? 3 : per_sm);
  long long want = ((long long)num_sms * per_sm + gy - 1) / gy;
  const long long cap = (long long)a.B * a.max_pages;
  int gx = (int)(want < 1 ? 1 : (want > cap ? cap : want));
  if (gx > 65535 * 32) gx = 65535 * 32;
  if (fp8idx) {
    if (NT == 1) return launch_nt<1, true>(a, gx, gy, smem, st);
    if (NT == 2) return launch_nt<2, true>(a, gx, gy, smem, st);
    return launch_nt<4, true>(a, gx, gy, smem, st);
  }
  if (NT == 1) return launch_nt<1, false>(a, gx, gy, smem, st);
  if (NT == 2) return launch_nt<2, false>(a, gx, gy, smem, st);
  return launch_nt<4, false>(a, gx, gy, smem, st);
}

}  // namespace msa
