// msa_attn.cu -- exact attention over the selected blocks ([post, "MSA
// primer"] and its Figure 1 caption: every query head of a GQA group attends
// over that group's selected blocks) with NVFP4 K/V dequantised to E4M3 in
// the kernel ([post, "NVIDIA Blackwell optimized MSA kernels"]).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Work unit: one (sequence, query token, group) = 16 query heads = one m16
// tile, split over its <= 16 selected blocks into `splits` CTAs.  A producer
// warp gathers each selected block of the group's KV head through the page
// table with four bulk async copies (K codes, K scales, V codes, V scales =
// 18 KB) into a ring of stages; four consumer warps each take 32 keys of
// every block.
//
// Arithmetic: K and V are decoded to their E4M3 values (the FP8 operands the
// method prescribes) and widened exactly to f16, and both contractions run on
// f16 tensor-core MMA with fp32 accumulation (m16n8k16).  On sm_100a the
// warp-level FP8 MMA is not native (it costs about twenty issue slots per
// instruction, measured), while the f16 one is; the products of E4M3 values
// are exact in either, so the result is the FP8 contraction's.
//   S  = Q K^T   A = Q (f16 fragments staged once in shared memory),
//                B = K decoded from the stage straight into fragments;
//   online softmax in the exp2 domain, masked beyond the query position;
//   O += P V     A = P (f16, from the S accumulators, FlashAttention-2
//                layout), B = V decoded into a swizzled 16-key f16 tile and
//                read transposed with ldmatrix.
// The four warps' (m, l, O) merge in shared memory; with one split the CTA
// writes bf16, otherwise it writes an fp32 partial and the last CTA of the
// unit to finish (atomic counter, no waiting) combines the partials.
#include "msa_internal.h"

#include <cuda_bf16.h>

namespace msa {

constexpr int kAttStageBytes = 2 * (kPageCodes + kPageScales);   // K + V of one KV head
constexpr int kVtBytes = 16 * kDim * 2;                           // per warp: 16 keys x 128 f16

size_t attn_smem_bytes() {
  return (size_t)kAttStages * kAttStageBytes + kAttConsumers * kVtBytes + 8 * 32 * 16 +
         256 * sizeof(uint2) + 2 * kAttStages * sizeof(uint64_t) + 4 * kTopk * sizeof(int) + 64;
}

int attn_splits(long long units, int num_sms) {
  int s = 1;
  while (s < kTopk && units * s < 2LL * num_sms) s *= 2;
  return s;
}

__global__ void __launch_bounds__(kAttThreads, 3) attn_kernel(AttnArgs a) {
  extern __shared__ __align__(128) uint8_t smem[];
  uint8_t* stages = smem;
  uint8_t* vt_all = smem + kAttStages * kAttStageBytes;                // [4 warps][16][256 B]
  uint32_t* qfrag = reinterpret_cast<uint32_t*>(vt_all + kAttConsumers * kVtBytes);   // [8][32][4]
  uint2* lut = reinterpret_cast<uint2*>(qfrag + 8 * 32 * 4);
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
    // Q A-fragments (f16), k-step ks: a0/a1 = rows gid/gid+8, dims
    // 32tig+4ks+{0,1}; a2/a3 = dims 32tig+4ks+{2,3}.  Staged once by warp 0.
    if (warp == 0) {
      uint32_t w[2][8];
#pragma unroll
      for (int r = 0; r < 2; ++r) {
        const int h = g * kHpg + gid + 8 * r;
        const uint8_t* src = a.q + (((long long)b * a.T + t) * kHq + h) * kDim + 32 * tig;
        const uint4 x0 = *reinterpret_cast<const uint4*>(src);
        const uint4 x1 = *reinterpret_cast<const uint4*>(src + 16);
        w[r][0] = x0.x; w[r][1] = x0.y; w[r][2] = x0.z; w[r][3] = x0.w;
        w[r][4] = x1.x; w[r][5] = x1.y; w[r][6] = x1.z; w[r][7] = x1.w;
      }
#pragma unroll
      for (int ks = 0; ks < 8; ++ks)
        *reinterpret_cast<uint4*>(&qfrag[(ks * 32 + lane) * 4]) =
            make_uint4(e4m3x2_to_f16x2(w[0][ks]), e4m3x2_to_f16x2(w[1][ks]),
                       e4m3x2_to_f16x2(w[0][ks] >> 16), e4m3x2_to_f16x2(w[1][ks] >> 16));
    }
    asm volatile("bar.sync 1, %0;\n" ::"n"(kAttConsumers * 32) : "memory");
    uint8_t* vt = vt_all + warp * kVtBytes;     // this warp's 16-key f16 V tile
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

      // ---- S = Q K^T over this warp's 32 keys (n-tile j = keys 8j..8j+7)
      float sacc[4][4];
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        sacc[j][0] = sacc[j][1] = sacc[j][2] = sacc[j][3] = 0.f;
        const int kk = 32 * warp + 8 * j + gid;
        uint32_t kw[8];
        dq32(lut, lds128(kc + kk * kRowCodes + 16 * tig), lds16(ks_ + kk * kRowScales + 2 * tig), kw);
#pragma unroll
        for (int st = 0; st < 8; ++st) {
          const uint4 qa = *reinterpret_cast<const uint4*>(&qfrag[(st * 32 + lane) * 4]);
          mma_f16(sacc[j], qa.x, qa.y, qa.z, qa.w, e4m3x2_to_f16x2(kw[st]),
                  e4m3x2_to_f16x2(kw[st] >> 16));
        }
      }

      // ---- mask, online softmax (exp2 domain)
      float mb[2] = {-INFINITY, -INFINITY};
#pragma unroll
      for (int j = 0; j < 4; ++j) {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int key = key0 + 8 * j + 2 * tig + (e & 1);
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

      // ---- O += P V, 16 keys at a time (PV k-step kk = S n-tiles 2kk, 2kk+1)
#pragma unroll
      for (int kk = 0; kk < 2; ++kk) {
        const uint32_t pa0 = f32x2_to_f16x2(sacc[2 * kk][0], sacc[2 * kk][1]);
        const uint32_t pa1 = f32x2_to_f16x2(sacc[2 * kk][2], sacc[2 * kk][3]);
        const uint32_t pa2 = f32x2_to_f16x2(sacc[2 * kk + 1][0], sacc[2 * kk + 1][1]);
        const uint32_t pa3 = f32x2_to_f16x2(sacc[2 * kk + 1][2], sacc[2 * kk + 1][3]);
        // V tile: rows = the 16 keys 32w+16kk+0..15 (256 B of f16 each);
        // 16-byte chunk c of row r at chunk position c ^ (r % 8).
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const int r = 8 * p + gid, vk = 32 * warp + 16 * kk + r;
          uint32_t vw[8];
          dq32(lut, lds128(vc + vk * kRowCodes + 16 * tig), lds16(vs + vk * kRowScales + 2 * tig), vw);
#pragma unroll
          for (int i = 0; i < 4; ++i)   // dims 32tig + 8i .. +7 = chunk 4tig + i
            *reinterpret_cast<uint4*>(vt + r * 256 + (((4 * tig + i) ^ (r & 7)) << 4)) =
                make_uint4(e4m3x2_to_f16x2(vw[2 * i]), e4m3x2_to_f16x2(vw[2 * i] >> 16),
                           e4m3x2_to_f16x2(vw[2 * i + 1]), e4m3x2_to_f16x2(vw[2 * i + 1] >> 16));
        }
        __syncwarp();
        // ldmatrix.x4.trans: matrix mi (lanes 8mi..8mi+7) = keys 8(mi&1)..+7 x dims 16n2+8(mi>>1)..+7
        const int mi = lane >> 3, lr = (mi & 1) * 8 + (lane & 7);
#pragma unroll
        for (int n2 = 0; n2 < 8; ++n2) {
          const int chunk = 2 * n2 + (mi >> 1);
          uint32_t b0, b1, b2, b3;
          ldsm_x4_trans(vt + lr * 256 + ((chunk ^ (lr & 7)) << 4), b0, b1, b2, b3);
          mma_f16(o[2 * n2], pa0, pa1, pa2, pa3, b0, b1);
          mma_f16(o[2 * n2 + 1], pa0, pa1, pa2, pa3, b2, b3);
        }
        __syncwarp();   // the tile is rewritten by the next 16 keys
      }
      if (lane == 0) mbar_arrive(&empty[s]);   // stage no longer read by this warp
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
