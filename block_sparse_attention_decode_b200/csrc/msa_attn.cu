// msa_attn.cu -- exact attention over the selected blocks ([post, "MSA
// primer"] and its Figure 1 caption: every query head of a GQA group attends
// over that group's selected blocks) with NVFP4 K/V dequantised to E4M3 in
// the kernel and fed to FP8 MMA ([post, "NVIDIA Blackwell optimized MSA
// kernels"]).  post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援
// (hot.atechcom.net).
//
// Work unit: one (sequence, query token, group) = 16 query heads = one m16
// MMA tile, split over its <= 16 selected blocks into `splits` CTAs.
// Per CTA a producer warp gathers each selected block of the group's KV head
// through the page table with four bulk async copies (K codes, K scales,
// V codes, V scales = 18 KB) into a ring of stages; four consumer warps each
// take 32 keys of every block:
//   S  = Q K^T   A = Q (16 heads x 128 dims, registers, loaded once),
//                B = K decoded from the stage straight into fragments;
//   online softmax in the exp2 domain, masked beyond the query position;
//   O += P V     A = P rounded to E4M3 from the S accumulators (the key order
//                of S's columns is chosen so that each thread already holds
//                the P values its A fragment needs), B = V, which the warp
//                decodes and transposes (4x4 byte blocks) into a small
//                per-warp V^T tile so each B fragment is one 64-bit load.
// The four warps' (m, l, O) merge in shared memory; with one split the CTA
// writes bf16, otherwise it writes an fp32 partial and the last CTA of the
// unit to finish (atomic counter, no waiting) combines the partials.
#include "msa_internal.h"

#include <cuda_bf16.h>

namespace msa {

constexpr int kAttStageBytes = 2 * (kPageCodes + kPageScales);   // K + V of one KV head
constexpr int kVtWords = kDim * 8 + 32;                           // per warp: [128 dims][8 words] + pad

size_t attn_smem_bytes() {
  return (size_t)kAttStages * kAttStageBytes + kAttConsumers * kVtWords * 4 + 4 * 32 * 16 +
         256 * sizeof(uint2) + 2 * kAttStages * sizeof(uint64_t) + 4 * kTopk * sizeof(int) + 64;
}

int attn_splits(long long units, int num_sms) {
  int s = 1;
  while (s < kTopk && units * s < 2LL * num_sms) s *= 2;
  return s;
}

// Key (within a warp's 32) held as S column n of n-tile j:
//   pi(j, n) = 4*(2j + n%2) + n/2.
// Thread tig then holds the keys congruent to tig mod 4, which is exactly the
// set its P A-fragment needs when the V^T word of key quad q holds keys
// q, q+8, q+16, q+24; and each K or V load instruction of the warp covers 8
// consecutive rows of the stage (bank-conflict free).
__device__ __forceinline__ int key_of(int j, int n) {
  return 4 * (2 * j + (n & 1)) + (n >> 1);
}

// 4x4 byte transpose: x[r] byte e -> y[e] byte r.
__device__ __forceinline__ void transpose4x4(uint32_t x0, uint32_t x1, uint32_t x2, uint32_t x3,
                                             uint32_t& y0, uint32_t& y1, uint32_t& y2,
                                             uint32_t& y3) {
  const uint32_t t0 = __byte_perm(x0, x1, 0x5140), t1 = __byte_perm(x0, x1, 0x7362);
  const uint32_t t2 = __byte_perm(x2, x3, 0x5140), t3 = __byte_perm(x2, x3, 0x7362);
  y0 = __byte_perm(t0, t2, 0x5410);
  y1 = __byte_perm(t0, t2, 0x7632);
  y2 = __byte_perm(t1, t3, 0x5410);
  y3 = __byte_perm(t1, t3, 0x7632);
}

// V^T word index of (dim d, key quad q): rows of 8 words, 8 words of padding
// every 32 dims so the transposing writers hit 32 distinct banks.
__device__ __forceinline__ int vt_index(int d, int q) {
  return d * 8 + 8 * (d >> 5) + 2 * (q & 3) + (q >> 2);
}

__global__ void __launch_bounds__(kAttThreads, 3) attn_kernel(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint32_t* vt_all = reinterpret_cast<uint32_t*>(smem + kAttStages * kAttStageBytes);
  uint32_t* qfrag = vt_all + kAttConsumers * kVtWords;                  // [4][32][4]
  uint2* lut = reinterpret_cast<uint2*>(qfrag + 4 * 32 * 4);
  uint64_t* full = reinterpret_cast<uint64_t*>(lut + 256);
  uint64_t* empty = full + kAttStages;
  int* list = reinterpret_cast<int*>(empty + kAttStages);   // [16] block ids
  int* pages = list + kTopk;                                 // [16] page ids (-1 = bad)
  int* misc = pages + kTopk;                                 // [0] = count, [1] = is_last

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int gid = lane >> 2, tig = lane & 3;
  const long long unit = blockIdx.x / a.splits;
  const int sp = blockIdx.x % a.splits;
  const int b = (int)(unit / (kG * a.T));
  const int t = (int)((unit / kG) % a.T);
  const int g = (int)(unit % kG);
  const int L = a.seq_lens[b];
  const bool len_ok = L >= a.T && L <= a.max_pages * kBlock;
  const int pos = L - a.T + t;

  build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < kAttStages; ++s) { mbar_init(&full[s], 1); mbar_init(&empty[s], kAttConsumers); }
    mbar_fence_init();
    int cnt = 0;
    if (!len_ok) {
      if (sp == 0 && g == 0 && t == 0) report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
    } else {
      const int nvis = pos / kBlock + 1;
      const int k0 = kTopk * sp / a.splits, k1 = kTopk * (sp + 1) / a.splits;
      for (int k = k0; k < k1; ++k) {
        const int blk = a.sel[unit * kTopk + k];
        if (blk < 0) continue;
        if (blk >= nvis) { report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, blk); continue; }
        const long long p = a.page_table ? (long long)a.page_table[(long long)b * a.max_pages + blk]
                                         : (long long)b * a.max_pages + blk;
        if (p < 0 || p >= a.num_pages) { report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)p); continue; }
        list[cnt] = blk;
        pages[cnt] = (int)p;
        ++cnt;
      }
    }
    misc[0] = cnt;
  }
  __syncthreads();
  const int nlist = misc[0];

  // per-warp softmax state for heads 16g+gid (row 0) and 16g+gid+8 (row 1)
  float m_run[2] = {-INFINITY, -INFINITY}, l_run[2] = {0.f, 0.f};
  float o[16][4];
#pragma unroll
  for (int nt = 0; nt < 16; ++nt) o[nt][0] = o[nt][1] = o[nt][2] = o[nt][3] = 0.f;

  if (warp == kAttConsumers) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      for (int k = 0; k < nlist; ++k) {
        const int s = k % kAttStages;
        if (k >= kAttStages && !mbar_wait(&empty[s], ((k / kAttStages) - 1) & 1)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, k);
          break;
        }
        const long long row0 = ((long long)pages[k] * kG + g) * kBlock;   // first (page, head, token) row
        uint8_t* dst = stages + s * kAttStageBytes;
        mbar_expect_tx(&full[s], kAttStageBytes);
        bulk_g2s(dst, a.k_data + row0 * kRowCodes, kPageCodes, &full[s]);
        bulk_g2s(dst + kPageCodes, a.k_scale + row0 * kRowScales, kPageScales, &full[s]);
        bulk_g2s(dst + kPageCodes + kPageScales, a.v_data + row0 * kRowCodes, kPageCodes, &full[s]);
        bulk_g2s(dst + 2 * kPageCodes + kPageScales, a.v_scale + row0 * kRowScales, kPageScales,
                 &full[s]);
      }
    }
  } else {
    // ------------------------------------------------------------ consumers
    // Q A-fragments live in shared memory (qfrag[k-step][lane] = a0..a3), so
    // they cost no registers across the block loop: row gid/gid+8 = heads
    // 16g+gid / 16g+gid+8, k-step st covers dims 32tig+8st..+7.
    if (warp == 0) {
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int h = g * kHpg + gid + 8 * r;
        const uint8_t* src = a.q + (((long long)b * a.T + t) * kHq + h) * kDim + 32 * tig;
        const uint4 x0 = *reinterpret_cast<const uint4*>(src);
        const uint4 x1 = *reinterpret_cast<const uint4*>(src + 16);
        const uint32_t w[8] = {x0.x, x0.y, x0.z, x0.w, x1.x, x1.y, x1.z, x1.w};
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          qfrag[(st * 32 + lane) * 4 + r] = w[2 * st];          // a0 / a1
          qfrag[(st * 32 + lane) * 4 + 2 + r] = w[2 * st + 1];  // a2 / a3
        }
      }
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kAttConsumers * 32) : "memory");
    uint32_t* vt = vt_all + warp * kVtWords;
    const float sc = a.logit_scale_log2;
    for (int k = 0; k < nlist; ++k) {
      const int s = k % kAttStages;
      if (!mbar_wait(&full[s], (k / kAttStages) & 1)) {
        report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, k);
        break;
      }
      const uint8_t* kc = stages + s * kAttStageBytes;
      const uint8_t* ks_ = kc + kPageCodes;
      const uint8_t* vc = ks_ + kPageScales;
      const uint8_t* vs = vc + kPageCodes;
      const int key0 = list[k] * kBlock + 32 * warp;   // global position of this warp's key 0

      // ---- S = Q K^T over this warp's 32 keys
      float sacc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
        const int kk = 32 * warp + key_of(j, gid);
        uint32_t kw[8];
        dq32(lut, lds128(kc + kk * kRowCodes + 16 * tig), lds16(ks_ + kk * kRowScales + 2 * tig), kw);
#pragma unroll
        for (int st = 0; st < 4; ++st) {
          const uint4 qa = *reinterpret_cast<const uint4*>(&qfrag[(st * 32 + lane) * 4]);
          mma_e4m3(sacc[j], qa.x, qa.y, qa.z, qa.w, kw[2 * st], kw[2 * st + 1]);
        }
      }

      // ---- V^T tile: lane (kq, dc) decodes keys kq + 8r (r = 0..3), dims
      // 32dc..32dc+31, in two halves of 16 dims (one scale byte each)
      {
        const int kq = lane >> 2, dc = lane & 3;
#pragma unroll
        for (int hf = 0; hf < 2; ++hf) {
          uint32_t vw[4][4];
#pragma unroll
          for (int r = 0; r < 4; ++r) {
            const int kk = 32 * warp + kq + 8 * r;
            const uint2 c = *reinterpret_cast<const uint2*>(vc + kk * kRowCodes + 16 * dc + 8 * hf);
            const uint2 row = lut[vs[kk * kRowScales + 2 * dc + hf]];
            dq8(c.x, row, vw[r][0], vw[r][1]);
            dq8(c.y, row, vw[r][2], vw[r][3]);
          }
#pragma unroll
          for (int m = 0; m < 4; ++m) {
            uint32_t y0, y1, y2, y3;
            transpose4x4(vw[0][m], vw[1][m], vw[2][m], vw[3][m], y0, y1, y2, y3);
            const int d = 32 * dc + 16 * hf + 4 * m;
            vt[vt_index(d + 0, kq)] = y0;
            vt[vt_index(d + 1, kq)] = y1;
            vt[vt_index(d + 2, kq)] = y2;
            vt[vt_index(d + 3, kq)] = y3;
          }
        }
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[s]);   // stage no longer read by this warp

      // ---- mask, online softmax (exp2 domain)
      float mb[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + key_of(j, 2 * tig + (e & 1));
          float v = sacc[j][e] * sc;
          if (key > pos) v = -INFINITY;
          sacc[j][e] = v;
          mb[e >> 1] = fmaxf(mb[e >> 1], v);
        }
      }
      float alpha[2], mu[2];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        mb[r] = fmaxf(mb[r], __shfl_xor_sync(0xffffffffu, mb[r], 1));
        mb[r] = fmaxf(mb[r], __shfl_xor_sync(0xffffffffu, mb[r], 2));
        const float m_new = fmaxf(m_run[r], mb[r]);
        mu[r] = (m_new == -INFINITY) ? 0.f : m_new;
        alpha[r] = exp2f(m_run[r] - mu[r]);
        m_run[r] = m_new;
      }
      float ps[2] = {0.f, 0.f};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const float p = exp2f(sacc[j][e] - mu[e >> 1]);
          sacc[j][e] = p;
          ps[e >> 1] += p;
        }
      }
#pragma unroll
      for (int r = 0; r < 2; ++r) l_run[r] = l_run[r] * alpha[r] + ps[r];
      if (__any_sync(0xffffffffu, alpha[0] != 1.f || alpha[1] != 1.f)) {
#pragma unroll
        for (int nt = 0; nt < 16; ++nt) {
          o[nt][0] *= alpha[0]; o[nt][1] *= alpha[0];
          o[nt][2] *= alpha[1]; o[nt][3] *= alpha[1];
        }
      }
      // ---- P fragments: logical k 4tig+e <-> key tig+8e (S n-tile e, column
      // 2tig), logical 16+4tig+e <-> key tig+4+8e (n-tile e, column 2tig+1).
      // P = Ph + Pl, both E4M3, so the FP8 MMA sees P to ~8 significant bits
      // (one E4M3 term alone moves the weights of a few-key softmax by ~3%).
      uint32_t ph0, pl0, ph1, pl1, ph2, pl2, ph3, pl3;
      split_e4m3x4(sacc[0][0], sacc[1][0], sacc[2][0], sacc[3][0], ph0, pl0);
      split_e4m3x4(sacc[0][2], sacc[1][2], sacc[2][2], sacc[3][2], ph1, pl1);
      split_e4m3x4(sacc[0][1], sacc[1][1], sacc[2][1], sacc[3][1], ph2, pl2);
      split_e4m3x4(sacc[0][3], sacc[1][3], sacc[2][3], sacc[3][3], ph3, pl3);
      // ---- O += Ph V + Pl V
#pragma unroll
      for (int nt = 0; nt < 16; ++nt) {
        const int d = 8 * nt + gid;
        const uint2 bb = *reinterpret_cast<const uint2*>(vt + vt_index(d, tig));
        mma_e4m3(o[nt], ph0, ph1, ph2, ph3, bb.x, bb.y);
        mma_e4m3(o[nt], pl0, pl1, pl2, pl3, bb.x, bb.y);
      }
      __syncwarp();   // V^T tile reused by the next block
    }
    // full row sums: add the 4 lanes of a row
#pragma unroll
    for (int r = 0; r < 2; ++r) {
      l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 1);
      l_run[r] += __shfl_xor_sync(0xffffffffu, l_run[r], 2);
    }
  }

  // ---------------------------------------------- merge the 4 warps' states
  __syncthreads();   // all stages consumed: reuse the stage ring as scratch
  float* ow = reinterpret_cast<float*>(stages);                // [4][16][128]
  float* mw = ow + kAttConsumers * kHpg * kDim;                // [4][16]
  float* lw = mw + kAttConsumers * kHpg;                       // [4][16]
  if (warp < kAttConsumers) {
    if (tig == 0) {
      mw[warp * kHpg + gid] = m_run[0];
      mw[warp * kHpg + gid + 8] = m_run[1];
      lw[warp * kHpg + gid] = l_run[0];
      lw[warp * kHpg + gid + 8] = l_run[1];
    }
#pragma unroll
    for (int nt = 0; nt < 16; ++nt) {
      float* r0 = ow + (warp * kHpg + gid) * kDim + 8 * nt + 2 * tig;
      float* r1 = r0 + 8 * kDim;
      r0[0] = o[nt][0]; r0[1] = o[nt][1];
      r1[0] = o[nt][2]; r1[1] = o[nt][3];
    }
  }
  __syncthreads();
  // 128 threads: thread -> head row tid/8, 16 dims starting at (tid%8)*16
  const int hr = tid >> 3, d0 = (tid & 7) * 16;
  float acc[16];
  float M = -INFINITY, Lsum = 0.f;
  if (tid < 128) {
#pragma unroll
    for (int w = 0; w < kAttConsumers; ++w) M = fmaxf(M, mw[w * kHpg + hr]);
    const float Mu = (M == -INFINITY) ? 0.f : M;
#pragma unroll
    for (int c = 0; c < 16; ++c) acc[c] = 0.f;
#pragma unroll
    for (int w = 0; w < kAttConsumers; ++w) {
      const float f = exp2f(mw[w * kHpg + hr] - Mu);
      Lsum += lw[w * kHpg + hr] * f;
      const float* src = ow + (w * kHpg + hr) * kDim + d0;
#pragma unroll
      for (int c = 0; c < 16; ++c) acc[c] += src[c] * f;
    }
  }
  const int h = g * kHpg + hr;
  uint16_t* dst = a.out + (((long long)b * a.T + t) * kHq + h) * kDim + d0;
  if (a.splits == 1) {
    if (tid < 128) {
      const float inv = Lsum > 0.f ? a.out_scale / Lsum : 0.f;
      uint32_t packed[8];
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const __nv_bfloat162 v = __floats2bfloat162_rn(acc[2 * c] * inv, acc[2 * c + 1] * inv);
        packed[c] = *reinterpret_cast<const uint32_t*>(&v);
      }
      reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
      reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
    }
    return;
  }
  // split-K: write this CTA's partial, the last CTA of the unit combines
  float* part = a.partials + ((long long)unit * a.splits + sp) * kPartialFloats;
  if (tid < 128) {
#pragma unroll
    for (int c = 0; c < 16; ++c) part[hr * kDim + d0 + c] = acc[c];
    if ((tid & 7) == 0) {
      part[kHpg * kDim + hr] = M;
      part[kHpg * kDim + kHpg + hr] = Lsum;
    }
  }
  __threadfence();
  __syncthreads();
  if (tid == 0) {
    const int prev = atomicAdd(&a.counters[unit], 1);
    misc[1] = (prev == a.splits - 1);
  }
  __syncthreads();
  if (!misc[1]) return;
  __threadfence();
  if (tid < 128) {
    const float* base = a.partials + (long long)unit * a.splits * kPartialFloats;
    float Mx = -INFINITY;
    for (int s2 = 0; s2 < a.splits; ++s2)
      Mx = fmaxf(Mx, __ldcg(base + s2 * kPartialFloats + kHpg * kDim + hr));
    const float Mu = (Mx == -INFINITY) ? 0.f : Mx;
    float tot[16];
#pragma unroll
    for (int c = 0; c < 16; ++c) tot[c] = 0.f;
    float Lt = 0.f;
    for (int s2 = 0; s2 < a.splits; ++s2) {
      const float* ps2 = base + s2 * kPartialFloats;
      const float f = exp2f(__ldcg(ps2 + kHpg * kDim + hr) - Mu);
      Lt += __ldcg(ps2 + kHpg * kDim + kHpg + hr) * f;
#pragma unroll
      for (int c = 0; c < 16; ++c) tot[c] += __ldcg(ps2 + hr * kDim + d0 + c) * f;
    }
    const float inv = Lt > 0.f ? a.out_scale / Lt : 0.f;
    uint32_t packed[8];
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const __nv_bfloat162 v = __floats2bfloat162_rn(tot[2 * c] * inv, tot[2 * c + 1] * inv);
      packed[c] = *reinterpret_cast<const uint32_t*>(&v);
    }
    reinterpret_cast<uint4*>(dst)[0] = make_uint4(packed[0], packed[1], packed[2], packed[3]);
    reinterpret_cast<uint4*>(dst)[1] = make_uint4(packed[4], packed[5], packed[6], packed[7]);
  }
  if (tid == 0) a.counters[unit] = 0;   // ready for the next call
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = attn_smem_bytes();
  static bool configured = false;
  if (!configured) {
    cudaError_t e = cudaFuncSetAttribute(attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (e != cudaSuccess) return e;
    configured = true;
  }
  const long long units = (long long)a.B * a.T * kG;
  const long long grid = units * a.splits;
  if (grid > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  attn_kernel<<<(unsigned)grid, kAttThreads, smem, st>>>(a);
  return cudaGetLastError();
}

// ----------------------------------------------------- parity debug hook --
__global__ void nvfp4_table_kernel(uint8_t* out) {
  __shared__ uint2 lut[256];
  build_nvfp4_lut(lut, threadIdx.x, blockDim.x);
  __syncthreads();
  const int s = threadIdx.x;   // 256 threads, one scale byte each
  const uint2 r = lut[s];
  uint32_t o[4];
  dq8(0x76543210u, r, o[0], o[1]);   // codes 0..7 in element order
  dq8(0xFEDCBA98u, r, o[2], o[3]);   // codes 8..15
  uint4* dst = reinterpret_cast<uint4*>(out + s * 16);
  *dst = make_uint4(o[0], o[1], o[2], o[3]);
}

cudaError_t launch_nvfp4_table(uint8_t* out, cudaStream_t st) {
  nvfp4_table_kernel<<<1, 256, 0, st>>>(out);
  return cudaGetLastError();
}

}  // namespace msa
