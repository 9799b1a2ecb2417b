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
constexpr int kTopkCache = 4096;   // rows up to this many candidates are cached in smem

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int B, int T,
            int max_pages, int32_t* __restrict__ sel, Flags* flags) {
  __shared__ unsigned keys[kTopkCache];
  __shared__ unsigned hist[256];
  __shared__ unsigned s_prefix;
  __shared__ int s_need;

  const long long row = blockIdx.x;          // (b * T + t) * 4 + g
  const int b = (int)(row / (kG * T));
  const int t = (int)((row / kG) % T);
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
  const bool cached = n <= kTopkCache;
  if (cached)
    for (int i = tid; i < n; i += kTopkThreads) keys[i] = float_key(S[i]);
  auto key_at = [&](int i) -> unsigned { return cached ? keys[i] : float_key(S[i]); };

  // Radix select, 8 bits per pass from the top: after the passes `prefix`
  // is the key of the 15th best candidate and `need` how many candidates
  // equal to it belong to the selection.
  unsigned prefix = 0;
  int need = kTopk - 1;
  for (int pass = 3; pass >= 0; --pass) {
    const int shift = 8 * pass;
    for (int d = tid; d < 256; d += kTopkThreads) hist[d] = 0;
    __syncthreads();
    for (int i = tid; i < n; i += kTopkThreads) {
      const unsigned k = key_at(i);
      if (pass == 3 || (k >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (warp == 0) {   // digit search: lane l owns bins 255-8l .. 248-8l (descending)
      unsigned c[8], sum = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) { c[j] = hist[255 - 8 * lane - j]; sum += c[j]; }
      unsigned incl = sum;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const unsigned v = __shfl_up_sync(0xffffffffu, incl, off);
        if (lane >= off) incl += v;
      }
      const unsigned hit = __ballot_sync(0xffffffffu, incl >= (unsigned)need);
      if (lane == __ffs(hit) - 1) {
        unsigned above = incl - sum;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (above + c[j] >= (unsigned)need) {
            s_prefix = prefix | ((unsigned)(255 - 8 * lane - j) << shift);
            s_need = need - (int)above;
            break;
          }
          above += c[j];
        }
      }
    }
    __syncthreads();
    prefix = s_prefix;
    need = s_need;
  }
  // One warp emits the selection in id order: every candidate above the
  // threshold key and the `need` lowest ids equal to it, then the latest.
  if (warp == 0) {
    int eq_seen = 0, emitted = 0;
    for (int base = 0; base < n && emitted < kTopk - 1; base += 32) {
      const int i = base + lane;
      const unsigned k = i < n ? key_at(i) : 0u;
      const bool gt = i < n && k > prefix;
      const bool eq = i < n && k == prefix;
      const unsigned lt = (1u << lane) - 1u;
      const unsigned beq = __ballot_sync(0xffffffffu, eq);
      const bool take = gt || (eq && eq_seen + __popc(beq & lt) < need);
      const unsigned btake = __ballot_sync(0xffffffffu, take);
      const int slot = emitted + __popc(btake & lt);
      if (take && slot < kTopk - 1) out[slot] = i;
      eq_seen += __popc(beq);
      emitted += __popc(btake);
    }
    if (lane == 0) out[kTopk - 1] = nb - 1;
  }
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
