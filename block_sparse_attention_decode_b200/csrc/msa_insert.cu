// msa_insert.cu -- write the new tokens into the cache: quantise each
// token's K and V (4 KV heads) and its index key to NVFP4 (index keys to FP8
// when the cache holds FP8 index keys) at the token's page and slot.  The
// step before the decode path ([post, "What is new in the MiniMax-M3.1
// architecture"]: NVFP4 KV cache for the indexer and the attention; [post,
// "QKV GEMM + norm + RoPE + KV insert fusion"] names the insertion).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Quantiser (the pages name the formats only; the reading is stated in the
// design notes): per 16 elements the scale byte is E4M3 (nearest-even,
// saturating) of amax / (6 s_t); each code is the nearest E2M1 magnitude of
// x / (scale s_t), ties to the even code, saturating at 6, sign bit only for
// a non-zero magnitude; FP8 keys are E4M3 of x / s_t.  The quotients that
// decide codes are IEEE fp32 divisions (__fdiv_rn), products __fmul_rn.
//
// One warp per (token, row): rows 0-3 the K heads, 4-7 the V heads, 8 the
// index key.  Lane l holds elements 4l..4l+3 (one 8-byte load of bf16); the
// 16-element block max takes two shuffles inside each group of 4 lanes; the
// warp writes the row's 64 code bytes in one 2-byte store per lane.
#include "msa_internal.h"

#include <cuda_fp8.h>

namespace msa {

constexpr int kInsRows = 9;                 // per token: 4 K heads, 4 V heads, index key

// Nearest E2M1 magnitude code of m >= 0, ties to the even code, saturating:
// the midpoints 0.25 0.75 1.25 1.75 2.5 3.5 5 between the grid values
// 0 0.5 1 1.5 2 3 4 6 round down (>) or up (>=) towards the even code.
__device__ __forceinline__ unsigned e2m1_code(float m) {
  return (unsigned)(m > 0.25f) + (unsigned)(m >= 0.75f) + (unsigned)(m > 1.25f) +
         (unsigned)(m >= 1.75f) + (unsigned)(m > 2.5f) + (unsigned)(m >= 3.5f) + (unsigned)(m > 5.f);
}

__device__ __forceinline__ float bf16_bits_to_float(uint32_t h) { return __uint_as_float(h << 16); }

__global__ void __launch_bounds__(256) insert_kernel(const InsArgs a) {
  const long long gw = ((long long)blockIdx.x * blockDim.x + threadIdx.x) >> 5;
  const int lane = threadIdx.x & 31;
  const long long ntok = (long long)a.B * a.T;
  if (gw >= ntok * kInsRows) return;
  const long long tok = gw / kInsRows;
  const int r = (int)(gw % kInsRows);
  const int b = (int)(tok / a.T), t = (int)(tok % a.T);
  const int L = a.seq_lens[b];
  if (L < a.T || L > a.max_pages * kBlock) {
    if (lane == 0 && r == 0 && t == 0) report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
    return;
  }
  const int pos = L - a.T + t;
  const int slot = pos % kBlock;
  const long long p = a.page_table ? (long long)a.page_table[(long long)b * a.max_pages + pos / kBlock]
                                   : (long long)b * a.max_pages + pos / kBlock;
  if (p < 0 || p >= a.num_pages) {
    if (lane == 0 && r == 0) report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)p);
    return;
  }
  const uint16_t* src;
  uint8_t* codes;
  uint8_t* scales = nullptr;
  float s_t;
  if (r < 2 * kG) {
    const int g = r & 3;
    const long long row = (p * kG + g) * kBlock + slot;
    src = (r < kG ? a.k_new : a.v_new) + (tok * kG + g) * kDim;
    codes = (r < kG ? a.k_data : a.v_data) + row * kRowCodes;
    scales = (r < kG ? a.k_scale : a.v_scale) + row * kRowScales;
    s_t = r < kG ? a.s_k : a.s_v;
  } else {
    const long long row = p * kBlock + slot;
    src = a.idx_new + tok * kDim;
    codes = a.idx_data + row * (a.idx_fp8 ? kDim : kRowCodes);
    if (!a.idx_fp8) scales = a.idx_scale + row * kRowScales;
    s_t = a.s_idx;
  }
  const uint2 raw = *reinterpret_cast<const uint2*>(src + 4 * lane);
  const float x[4] = {bf16_bits_to_float(raw.x & 0xFFFFu), bf16_bits_to_float(raw.x >> 16),
                      bf16_bits_to_float(raw.y & 0xFFFFu), bf16_bits_to_float(raw.y >> 16)};
  if (scales == nullptr) {   // FP8 index key
    uint32_t out = 0;
#pragma unroll
    for (int i = 0; i < 4; ++i)
      out |= (uint32_t)__nv_cvt_float_to_fp8(__fdiv_rn(x[i], s_t), __NV_SATFINITE, __NV_E4M3) << (8 * i);
    *reinterpret_cast<uint32_t*>(codes + 4 * lane) = out;
    return;
  }
  float am = fmaxf(fmaxf(fabsf(x[0]), fabsf(x[1])), fmaxf(fabsf(x[2]), fabsf(x[3])));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 1));
  am = fmaxf(am, __shfl_xor_sync(0xffffffffu, am, 2));   // max of the lane group's 16 elements
  const float r6 = __fdiv_rn(am, __fmul_rn(6.f, s_t));
  const __nv_fp8_storage_t sb = __nv_cvt_float_to_fp8(r6, __NV_SATFINITE, __NV_E4M3);
  __nv_fp8_e4m3 sdv;
  sdv.__x = sb;
  const float u = __fmul_rn(float(sdv), s_t);
  unsigned c[4];
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    c[i] = 0u;
    if (u != 0.f) {
      const unsigned m = e2m1_code(fabsf(__fdiv_rn(x[i], u)));
      c[i] = (m != 0u && x[i] < 0.f) ? (m | 8u) : m;
    }
  }
  *reinterpret_cast<uint16_t*>(codes + 2 * lane) =
      (uint16_t)(c[0] | (c[1] << 4) | (c[2] << 8) | (c[3] << 12));
  if ((lane & 3) == 0) scales[lane >> 2] = (uint8_t)sb;
}

cudaError_t launch_insert(const InsArgs& a, cudaStream_t st) {
  const long long warps = (long long)a.B * a.T * kInsRows;
  const long long ctas = (warps + 7) / 8;
  if (ctas > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  insert_kernel<<<(unsigned)ctas, 256, 0, st>>>(a);
  return cudaGetLastError();
}

}  // namespace msa
