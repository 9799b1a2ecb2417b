// msa_topk.cu -- block selection ([post, "MSA primer"]: attention runs over
// the top 16 blocks and the most recent block is always kept).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// One CTA per (sequence, token, group) row.  The latest visible block is
// kept; the other 15 are the best of blocks 0 .. latest-1 ranked by (score
// descending, block id ascending).  Selection is an exact radix select over
// order-preserving 32-bit keys of the fp32 scores (4 passes of 8 bits) that
// finds the 15th key value and how many blocks equal to it are still needed;
// a final pass in id order keeps every block above that value and the lowest
// ids among the equal ones, which also emits the ids in ascending order.
// No sort, no inter-CTA communication, and the result does not depend on how
// the indexer split its work (the selection stays exact, as in the post's
// "NVFP4 indexer DCP" section).
#include "msa_internal.h"

namespace msa {

constexpr int kTopkThreads = 128;
constexpr int kTopkWarps = kTopkThreads / 32;

// Exclusive block-wide prefix count of `pred`; *total receives the sum.
__device__ __forceinline__ int block_excl_count(bool pred, int* warp_sums, int* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const unsigned bal = __ballot_sync(0xffffffffu, pred);
  const int in_warp = __popc(bal & ((1u << lane) - 1u));
  if (lane == 0) warp_sums[warp] = __popc(bal);
  __syncthreads();
  int before = 0, sum = 0;
#pragma unroll
  for (int w = 0; w < kTopkWarps; ++w) {
    const int v = warp_sums[w];
    if (w < warp) before += v;
    sum += v;
  }
  __syncthreads();
  *total = sum;
  return before + in_warp;
}

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int B, int T,
            int max_pages, int32_t* __restrict__ sel, Flags* flags) {
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix;
  __shared__ int s_need;
  __shared__ int warp_sums[kTopkWarps];

  const long long row = blockIdx.x;          // (b * T + t) * 4 + g
  const int b = (int)(row / (kG * T));
  const int t = (int)((row / kG) % T);
  const int tid = threadIdx.x;
  int32_t* out = sel + row * kTopk;
  const int L = seq_lens[b];
  if (L < T || L > max_pages * kBlock) {
    if (tid == 0 && (row % kG) == 0 && t == 0) report(flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
    if (tid < kTopk) out[tid] = -1;
    return;
  }
  const int pos = L - T + t;
  const int nb = pos / kBlock + 1;           // visible blocks; the latest is nb-1
  if (nb <= kTopk) {
    if (tid < kTopk) out[tid] = tid < nb ? tid : -1;
    return;
  }
  const float* S = scores + row * max_pages;
  const int n = nb - 1;                      // candidates 0 .. nb-2
  unsigned prefix = 0;
  int need = kTopk - 1;
  for (int pass = 3; pass >= 0; --pass) {
    const int shift = 8 * pass;
    for (int d = tid; d < 256; d += kTopkThreads) hist[d] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const unsigned k = float_key(S[i]);
      if (pass == 3 || (k >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid == 0) {
      int above = 0;
      for (int d = 255; d >= 0; --d) {
        const int c = (int)hist[d];
        if (above + c >= need) {
          s_prefix = prefix | ((unsigned)d << shift);
          s_need = need - above;
          break;
        }
        above += c;
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
    __syncthreads();
  }
  // prefix = key of the 15th best candidate; take `need` of the blocks equal
  // to it (lowest ids first) and every block above it.
  int eq_seen = 0, emitted = 0;
  for (int base = 0; base < n; base += kTopkThreads) {
    const int i = base + tid;
    const unsigned k = i < n ? float_key(S[i]) : 0u;
    const bool gt = i < n && k > prefix;
    const bool eq = i < n && k == prefix;
    int eq_total, take_total;
    const int eq_rank = eq_seen + block_excl_count(eq, warp_sums, &eq_total);
    const bool take = gt || (eq && eq_rank < need);
    const int slot = emitted + block_excl_count(take, warp_sums, &take_total);
    if (take && slot < kTopk - 1) out[slot] = i;
    eq_seen += eq_total;
    emitted += take_total;
  }
  if (tid == 0) out[kTopk - 1] = nb - 1;
}

__global__ void maxpool_kernel(const float* __restrict__ ts, const int32_t* __restrict__ seq_lens,
                               int B, int T, int max_pages, float* __restrict__ bs) {
  const long long row = blockIdx.x;          // (b * T + t) * 4 + g
  const int i = blockIdx.y * blockDim.x + threadIdx.x;
  if (i >= max_pages) return;
  const int b = (int)(row / (kG * T)), t = (int)((row / kG) % T);
  const int L = seq_lens[b];
  if (L < T || L > max_pages * kBlock) return;
  const int pos = L - T + t;
  const int nblk = (L + kBlock - 1) / kBlock;
  if (i >= nblk) return;
  const float* r = ts + row * (long long)max_pages * kBlock + (long long)i * kBlock;
  float m = -INFINITY;
  for (int j = 0; j < kBlock && i * kBlock + j <= pos; ++j) m = fmaxf(m, r[j]);
  bs[row * max_pages + i] = m;
}

cudaError_t launch_topk(const float* block_scores, const int32_t* seq_lens, int B, int T,
                        int max_pages, int32_t* sel, Flags* flags, cudaStream_t st) {
  const long long rows = (long long)B * T * kG;
  if (rows > 0x7FFFFFFFLL) return cudaErrorInvalidValue;
  topk_kernel<<<(unsigned)rows, kTopkThreads, 0, st>>>(block_scores, seq_lens, B, T, max_pages,
                                                        sel, flags);
  return cudaGetLastError();
}

cudaError_t launch_maxpool(const float* token_scores, const int32_t* seq_lens, int B, int T,
                           int max_pages, float* block_scores, Flags* flags, cudaStream_t st) {
  (void)flags;
  const long long rows = (long long)B * T * kG;
  if (rows > 0x7FFFFFFFLL || max_pages > 65535 * 128) return cudaErrorInvalidValue;
  dim3 grid((unsigned)rows, (max_pages + 127) / 128);
  maxpool_kernel<<<grid, 128, 0, st>>>(token_scores, seq_lens, B, T, max_pages, block_scores);
  return cudaGetLastError();
}

}  // namespace msa
