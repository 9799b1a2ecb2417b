// msa_topk.cu -- block selection ([post, "MSA primer"]: attention runs over
// the top 16 blocks and the most recent block is always kept).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// One warp per (sequence, token, group) row, four rows per CTA, no block-wide
// synchronisation.  The latest visible block is kept; the other 15 are the
// best of blocks 0 .. latest-1 ranked by (score descending, block id
// ascending), scores compared as order-preserving 32-bit keys of the fp32
// values (-0 taken as +0).
//
// Fast path: the keys are staged in shared memory; tau = the 15th largest of
// the 32 lanes' maxima is at most the 15th largest key (the 15 lanes with
// the largest maxima hold 15 keys >= tau), so every block of the selection
// has a key >= tau.  The blocks with key >= tau -- usually a few dozen -- are
// compacted (ballots) into a candidate list, ranked exactly against each
// other, and the 15 best are written in id order.  When more than
// kTopkCand blocks reach tau (heavy ties), the row falls back to an exact
// radix select over all keys (8-bit digits from the first byte where the
// keys differ) that finds the 15th key and how many blocks equal to it are
// needed, then keeps every block above it and the lowest ids among the equal
// ones.  No sort, no inter-CTA communication, and the result does not depend
// on how the indexer split its work (the selection stays exact, as in the
// post's "NVFP4 indexer DCP" section).
#include "msa_internal.h"

namespace msa {

constexpr int kTopkRows = 4;                  // rows (warps) per CTA
constexpr int kTopkThreads = 32 * kTopkRows;
constexpr int kTopkCache = 2048;              // candidates per row cached in shared memory
constexpr int kTopkCand = 64;                 // fast path: at most this many blocks reach tau

// Order-preserving key of a block score with -0 taken as +0 (the ranking
// compares values, and -0 == +0).
__device__ __forceinline__ unsigned score_key(float f) { return float_key(f + 0.0f); }

__global__ void __launch_bounds__(kTopkThreads)
topk_kernel(const float* __restrict__ scores, const int32_t* __restrict__ seq_lens, int B, int T,
            int max_pages, int32_t* __restrict__ sel, Flags* flags) {
  __shared__ unsigned keys_all[kTopkRows][kTopkCache];
  __shared__ unsigned hist_all[kTopkRows][256];
  __shared__ unsigned cand_key_all[kTopkRows][kTopkCand];
  __shared__ int cand_id_all[kTopkRows][kTopkCand];
  const int lane = threadIdx.x & 31, w = threadIdx.x >> 5;
  grid_dependency_wait();   // launched with programmatic serialisation: scores ready
  grid_launch_dependents(); // the attention may start its prologue
  const long long row = (long long)blockIdx.x * kTopkRows + w;   // (b * T + t) * 4 + g
  if (row >= (long long)B * T * kG) return;
  unsigned* keys = keys_all[w];
  unsigned* hist = hist_all[w];
  const int b = (int)(row / (kG * T));
  const int t = (int)((row / kG) % T);
  int32_t* out = sel + row * kTopk;
  const int L = seq_lens[b];
  if (L < T || L > max_pages * kBlock) {
    if (lane == 0 && (row % kG) == 0 && t == 0) report(flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
    if (lane < kTopk) out[lane] = -1;
    return;
  }
  const int pos = L - T + t;
  const int nb = pos / kBlock + 1;           // visible blocks; the latest is nb-1
  if (nb <= kTopk) {
    if (lane < kTopk) out[lane] = lane < nb ? lane : -1;
    return;
  }
  const float* S = scores + row * max_pages;
  const int n = nb - 1;                      // candidates 0 .. nb-2
  const bool cached = n <= kTopkCache;
  unsigned kmin = 0xFFFFFFFFu, kmax = 0u;
  // 32 loads in flight per lane (the scores come from L2 or HBM): a row of
  // up to 1,024 candidates is read in one round trip
  for (int base = 0; base < n; base += 32 * 32) {
    float v[32];
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = base + 32 * j + lane;
      v[j] = i < n ? __ldcg(S + i) : 0.f;
    }
#pragma unroll
    for (int j = 0; j < 32; ++j) {
      const int i = base + 32 * j + lane;
      if (i < n) {
        const unsigned k = score_key(v[j]);
        if (cached) keys[i] = k;
        kmin = min(kmin, k);
        kmax = max(kmax, k);
      }
    }
  }
  __syncwarp();
  auto key_at = [&](int i) -> unsigned { return cached ? keys[i] : score_key(S[i]); };

  // ---- fast path: candidates with key >= tau, ranked exactly
  {
    // tau = the 15th largest lane maximum (lanes without candidates hold 0,
    // below every key; n >= 16 lanes hold one)
    int above = 0;
#pragma unroll 8
    for (int m = 0; m < 32; ++m) {
      const unsigned x = __shfl_sync(0xffffffffu, kmax, m);
      above += (x > kmax) || (x == kmax && m < lane);
    }
    const unsigned tau = __shfl_sync(0xffffffffu, kmax, __ffs(__ballot_sync(0xffffffffu, above == kTopk - 2)) - 1);
    unsigned* ck = cand_key_all[w];
    int* cid = cand_id_all[w];
    int count = 0;                       // candidates so far (warp-uniform)
    for (int base = 0; base < n; base += 32) {
      const int i = base + lane;
      const bool c = i < n && key_at(i) >= tau;
      const unsigned bal = __ballot_sync(0xffffffffu, c);
      const int slot = count + __popc(bal & ((1u << lane) - 1u));
      if (c && slot < kTopkCand) { ck[slot] = key_at(i); cid[slot] = i; }
      count += __popc(bal);
    }
    __syncwarp();
    if (count <= kTopkCand) {
      // lane holds candidates lane and lane + 32 in registers; the others'
      // come by shuffle.  Rank of candidate j = how many candidates precede it
      // in (key desc, id asc); the 15 of rank < 15 are selected.
      const bool v0 = lane < count, v1 = lane + 32 < count;
      const unsigned k0 = v0 ? ck[lane] : 0u, k1 = v1 ? ck[lane + 32] : 0u;
      const int i0 = v0 ? cid[lane] : 0x7FFFFFFF, i1 = v1 ? cid[lane + 32] : 0x7FFFFFFF;
      int r0 = 0, r1 = 0;
      const int c0 = min(count, 32), c1 = count - c0;
      for (int m = 0; m < c0; ++m) {
        const unsigned km = __shfl_sync(0xffffffffu, k0, m);
        const int im = __shfl_sync(0xffffffffu, i0, m);
        r0 += (km > k0) || (km == k0 && im < i0);
        r1 += (km > k1) || (km == k1 && im < i1);
      }
      for (int m = 0; m < c1; ++m) {
        const unsigned km = __shfl_sync(0xffffffffu, k1, m);
        const int im = __shfl_sync(0xffffffffu, i1, m);
        r0 += (km > k0) || (km == k0 && im < i0);
        r1 += (km > k1) || (km == k1 && im < i1);
      }
      const bool s0 = v0 && r0 < kTopk - 1, s1 = v1 && r1 < kTopk - 1;
      // the 15 selected ids in ascending order: position = selected ids below
      const unsigned b0 = __ballot_sync(0xffffffffu, s0), b1 = __ballot_sync(0xffffffffu, s1);
      int p0 = 0, p1 = 0;
      for (unsigned bb = b0; bb; bb &= bb - 1u) {
        const int im = __shfl_sync(0xffffffffu, i0, __ffs(bb) - 1);
        p0 += im < i0;
        p1 += im < i1;
      }
      for (unsigned bb = b1; bb; bb &= bb - 1u) {
        const int im = __shfl_sync(0xffffffffu, i1, __ffs(bb) - 1);
        p0 += im < i0;
        p1 += im < i1;
      }
      if (s0) out[p0] = i0;
      if (s1) out[p1] = i1;
      if (lane == 0) out[kTopk - 1] = nb - 1;
      return;
    }
  }

  // ---- fallback: exact radix select over all keys (heavy ties)
  kmin = __reduce_min_sync(0xffffffffu, kmin);
  kmax = __reduce_max_sync(0xffffffffu, kmax);

  // Radix select, 8 bits per pass from the top: after the passes `prefix`
  // is the key of the 15th best candidate and `need` how many candidates
  // equal to it belong to the selection.
  // Bytes every candidate shares are known already: start at the highest
  // byte where the smallest and the largest key differ (the scores of a row
  // usually share their sign and top exponent bits, which would otherwise
  // send a whole pass's counts into one or two bins).
  const int top = (31 - __clz(kmin ^ kmax)) >> 3;           // -1 when all keys are equal
  unsigned prefix = top < 0 ? kmax : (top >= 3 ? 0u : (kmax & ~((1u << (8 * top + 8)) - 1u)));
  int need = kTopk - 1;
#pragma unroll 1
  for (int pass = top; pass >= 0; --pass) {
    const int shift = 8 * pass;
#pragma unroll
    for (int j = 0; j < 8; ++j) hist[lane * 8 + j] = 0;
    __syncwarp();
    for (int i = lane; i < n; i += 32) {
      const unsigned k = key_at(i);
      if (pass == 3 || (k >> (shift + 8)) == (prefix >> (shift + 8)))
        atomicAdd(&hist[(k >> shift) & 255u], 1u);
    }
    __syncwarp();
    // digit search: lane l owns bins 255-8l .. 248-8l (descending)
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
    const int src = __ffs(hit) - 1;
    unsigned np = 0;
    int nn = 0;
    if (lane == src) {
      unsigned above = incl - sum;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        if (above + c[j] >= (unsigned)need) {
          np = prefix | ((unsigned)(255 - 8 * lane - j) << shift);
          nn = need - (int)above;
          break;
        }
        above += c[j];
      }
    }
    prefix = __shfl_sync(0xffffffffu, np, src);
    need = __shfl_sync(0xffffffffu, nn, src);
    __syncwarp();   // the histogram is rewritten by the next pass
  }
  // Emit the selection in id order: every candidate above the threshold key
  // and the `need` lowest ids equal to it, then the latest.
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
  const long long ctas = (rows + kTopkRows - 1) / kTopkRows;
  return launch_dependent(topk_kernel, dim3((unsigned)ctas), dim3(kTopkThreads), 0, st, block_scores,
                          seq_lens, B, T, max_pages, sel, flags);
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
