// msa_attn.cu -- exact attention over the selected blocks ([post, "MSA
// primer"] and its Figure 1 caption: every query head of a GQA group attends
// over that group's selected blocks) with NVFP4 K/V dequantised to E4M3 in
// the kernel and both contractions on the FP8 tensor core ([post, "NVIDIA
// Blackwell optimized MSA kernels"]).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Work item: one (sequence, query token, group) row -- its 16 query heads --
// or, for small batches, one of `splits` slices of that row's selected
// blocks.  Persistent CTAs (two per SM) claim items from a counter in the
// workspace header and stream their blocks through a pipeline:
//
//   warp 12 (producer): per item one TMA load of the 16 query rows (128-byte
//     swizzle: the B operand of S); per block, through the page table, two
//     tiled TMA loads of the K and V codes (64-byte swizzle) and two bulk
//     copies of their scales into a ring of shared-memory stages;
//   warps 0-3 (decoders): thread = key row, warp w decoding rows
//     32w..32w+31 (kKVSplit below: K here and V on warps 4-7).  K is decoded signed (dq8) straight into tensor memory
//     (dq8; one A operand: 4 MMAs per block rather than 8 for a split by sign --
//     the MMA-issuing thread is the scarcer resource here); V is decoded
//     signed into shared memory as E4M3 rows of 128
//     bytes with the 128-byte swizzle -- the A operand of O^T = V^T P^T in
//     MN-major form;
//   warp 13 (MMA, one thread): per block
//       S^T[128 keys x 16 heads]  = K Q^T   (4 MMAs, A from TMEM)
//       O^T[128 dims x 32]       += V^T [P_hi | P_lo]^T  (4 MMAs, A and B in
//                                   shared memory, both MN-major),
//     the two streams polled independently, so that the S of the next block
//     is issued while the softmax of this one runs;
//   warps 4-11 (softmax): warp 4+4j+q reads heads 8j..8j+7 of the S^T lanes
//     of quarter q (thread = key), masks keys after the query position,
//     takes the per-head block maximum (warp reduction, then across the four
//     quarters through shared memory), and writes P = 2^(s*c - m + 4) split
//     into two E4M3 terms through FP16 (P_hi + P_lo holds P to about 2^-8
//     relative) as 16-byte rows per key.
//     The running maximum m is raised lazily -- only when a block's maximum
//     exceeds it by more than 2^4 -- so that P stays below 2^8 (inside E4M3)
//     and O^T in tensor memory is rescaled rarely.  At the end of an item
//     the same warps (thread = dim) read O^T, divide by the row sums and
//     write bf16, or, with splits, an fp32 partial that the last CTA of the
//     row combines (atomic counter, no waiting).
// Every wait is a bounded mbarrier wait; on a timeout a thread records
// MSA_ERR_TIMEOUT and leaves its loop, and TMEM is freed before exit.
#include "msa_internal.h"

#include <cuda_bf16.h>
#include <cuda_fp8.h>

namespace msa {

// kKVSplit: K and V decoded by separate warps (K: 0-3, V: 4-7), so that a
// block's two decodes run side by side, the softmax then on four warps of 16
// heads (8-11).  Correct, but slower (0.211 against 0.202 ms at 64 x 128K,
// T = 8): off.
constexpr bool kKVSplit = false;
constexpr int kAttDecoders = 4;             // warps 0-3, one per TMEM lane quarter
constexpr int kAttVWarp0 = 4;               // V decoders (with the split): warps 4-7
constexpr int kAttSoft = kKVSplit ? 4 : 8;  // softmax warps: one or two per lane quarter
constexpr int kAttSoftWarp0 = kKVSplit ? 8 : 4;
constexpr int kHh = kHpg * 4 / kAttSoft;    // heads per softmax warp
static_assert(kHh % 8 == 0, "softmax warps hold whole groups of eight heads");
constexpr int kRing = 8;                    // block info slots (decoders -> MMA, softmax)
constexpr int kAttProducerWarp = 12;
constexpr int kAttMmaWarp = 13;
constexpr int kAttRawStride = 2 * (kPageCodes + kPageScales);   // 18432 = 18 x 1024
constexpr int kAttTmemCols = 256;           // A[2] 0..63, S[2] 64..95, O[2] 96..159
constexpr int kColA = 0, kColS = 64, kColO = 96;
constexpr float kPExp = 4.f;                // P carries a factor 2^4 (E4M3 normal range)
constexpr float kLazy = 4.f;                // raise m only when a block max exceeds it by 2^4
constexpr int kVB = 3;                      // V and P buffers (blocks between decode and O update)

enum : int { kBlkLoad = 0, kBlkEmpty = 1, kBlkEnd = 2 };

// Block info (producer -> decoders via the stage meta, decoders -> MMA and
// softmax via a ring of kRing): kind, block id, first, last, item sequence
// number, row, split, query position.
constexpr int kInfo = 8;

struct AttLayout {
  int raw, vbuf, pbuf, qbuf, lut, red, bc, lsum, bars, meta, binfo, tslot, misc, total;
};

// Decode-once mode: a stage holds the block's E4M3 K rows (the A operand of S),
// its V rows go straight to a V buffer
constexpr int kDkvTile = kBlock * kDim;         // 16 KB of E4M3 rows

template <bool PRE>
__host__ __device__ inline AttLayout att_layout() {
  AttLayout L;
  int off = 0;
  L.raw = off;   off += kAttStages * (PRE ? kDkvTile : kAttRawStride);
  L.vbuf = off;  off += kVB * kBlock * kDim;               // V rows, E4M3, 128-byte swizzle
  L.qbuf = off;  off += 2 * kHpg * kDim;                   // Q rows, E4M3, 128-byte swizzle
  L.pbuf = off;  off += kVB * 2 * kBlock * kHpg;           // [kVB][hi, lo][key][16 heads]
  L.lut = off;   off += 256 * 8;
  L.red = off;   off += 2 * 4 * kHpg * 4;                  // block maxima [parity][quarter][16]
  L.bc = off;    off += kAttSoft * 2 * kHh * 4;            // per softmax warp: offsets, alphas
  L.lsum = off;  off += 2 * 4 * kHpg * 4;                  // row sums [parity][quarter][16]
  L.bars = off;  off += (2 * kAttStages + 3 * kVB + 14) * 8;
  L.meta = off;  off += kAttStages * kInfo * 4;
  L.binfo = off; off += kRing * kInfo * 4;
  L.tslot = off; off += 16;
  L.misc = off;  off += 16;
  L.total = off + 1024;                                    // alignment slack
  return L;
}

size_t attn_smem_bytes() { return (size_t)att_layout<false>().total; }

int attn_splits(long long rows, int num_sms) {
  int s = 1;
  while (s < kTopk && rows * s < 4LL * num_sms) s *= 2;
  return s;
}

// Shared-memory descriptor, MN-major operand with the 128-byte swizzle: rows
// of 128 bytes (128 M elements) per K index, 8-row atoms `sbo` bytes apart.
__device__ __forceinline__ uint64_t desc_mn_sw128(uint32_t addr, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(16384 >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Shared-memory descriptor, MN-major operand without swizzle: core matrices
// of 8 K rows x 16 bytes (128 contiguous bytes), `lbo` bytes apart along K
// and `sbo` bytes apart along N.
__device__ __forceinline__ uint64_t desc_mn_plain(uint32_t addr, uint32_t lbo, uint32_t sbo) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)(lbo >> 4) << 16) |
         ((uint64_t)(sbo >> 4) << 32) | ((uint64_t)1 << 46);
}

// P (two values, 0 <= p <= 256) as the sum of two E4M3 terms, each pair
// packed in 16 bits (low byte = first value): P is rounded to FP16 (relative
// error 2^-11), hi = E4M3(P16); P16 - hi is exact in FP16 (hi lies within
// 2^-4 of P16) and lo = E4M3(P16 - hi), so hi + lo holds P to about 2^-8.
__device__ __forceinline__ void p_split_e4m3x2(float p0, float p1, uint32_t& hi, uint32_t& lo) {
  uint32_t p16, back, r16;
  uint16_t h8, l8;
  asm("cvt.rn.f16x2.f32 %0, %1, %2;\n" : "=r"(p16) : "f"(p1), "f"(p0));
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;\n" : "=h"(h8) : "r"(p16));
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(back) : "h"(h8));
  asm("sub.rn.f16x2 %0, %1, %2;\n" : "=r"(r16) : "r"(p16), "r"(back));
  asm("cvt.rn.satfinite.e4m3x2.f16x2 %0, %1;\n" : "=h"(l8) : "r"(r16));
  hi = h8;
  lo = l8;
}

// 2^x with the SFU's approximate exp2 (relative error below 2^-22).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;\n" : "=f"(y) : "f"(x));
  return y;
}


template <bool PRE>
__global__ void __launch_bounds__(kAttThreads, 2) attn_kernel(const __grid_constant__ AttnArgs a) {
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
  const AttLayout Ly = att_layout<PRE>();
  uint8_t* raw = smem + Ly.raw;
  uint8_t* vbuf = smem + Ly.vbuf;
  uint8_t* qbuf = smem + Ly.qbuf;
  uint8_t* pbuf = smem + Ly.pbuf;
  uint2* lut = reinterpret_cast<uint2*>(smem + Ly.lut);
  float* red = reinterpret_cast<float*>(smem + Ly.red);
  float* bc = reinterpret_cast<float*>(smem + Ly.bc);
  float* lsum = reinterpret_cast<float*>(smem + Ly.lsum);
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* raw_empty = raw_full + kAttStages;
  uint64_t* q_full = raw_empty + kAttStages;     // [2] producer (TMA) -> MMA
  uint64_t* q_empty = q_full + 2;                // [2] MMA -> producer
  uint64_t* kv_full = q_empty + 2;               // [2] decoders -> MMA
  uint64_t* s_full = kv_full + 2;                // [2] MMA -> softmax
  uint64_t* p_full = s_full + 2;                 // [kVB] softmax -> MMA
  uint64_t* pv_done = p_full + kVB;              // [kVB] MMA -> decoders, softmax
  uint64_t* o_free = pv_done + kVB;              // [2] softmax -> MMA
  uint64_t* red_full = o_free + 2;               // [1] softmax rendezvous
  uint64_t* misc_bar = red_full + 1;             // [1] softmax rendezvous (item end)
  uint64_t* s_free = misc_bar + 1;               // [2] softmax -> MMA: S buffer read
  uint64_t* v_full = s_free + 2;                 // [kVB] V decoders -> MMA (with the split)
  int* meta = reinterpret_cast<int*>(smem + Ly.meta);
  int* binfo = reinterpret_cast<int*>(smem + Ly.binfo);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly.tslot);
  int* misc = reinterpret_cast<int*>(smem + Ly.misc);

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const long long rows = (long long)a.B * a.T * kG;
  const long long items = rows * a.splits;

  build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < kAttStages; ++s) {
      mbar_init(&raw_full[s], 1);
      // decode-once: released by the S MMA; else by the K (and V) decoders
      mbar_init(&raw_empty[s], PRE ? 1 : kKVSplit ? 2 * kAttDecoders : kAttDecoders);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
      mbar_init(&kv_full[x], kAttDecoders);
      mbar_init(&s_full[x], 1);
      mbar_init(&o_free[x], kAttSoft);
    }
    for (int x = 0; x < kVB; ++x) {
      mbar_init(&p_full[x], kAttSoft);
      mbar_init(&pv_done[x], 1);
      mbar_init(&v_full[x], kAttDecoders);
    }
    mbar_init(red_full, kAttSoft);
    mbar_init(misc_bar, kAttSoft);
    for (int x = 0; x < 2; ++x) mbar_init(&s_free[x], kAttSoft);
    mbar_fence_init();
  }
  if (warp == kAttMmaWarp) {
    tmem_alloc(tslot, kAttTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem = *tslot;
  // launched with programmatic serialisation: the prologue above overlapped
  // the previous kernel; its outputs (the selection) are read from here on
  grid_dependency_wait();

  if (warp == kAttProducerWarp) {
    // ------------------------------------------------------------ producer
    // The whole warp sets up an item (lane kk checks selected block kk: its
    // id and page load in parallel); lane 0 issues the copies.  The next
    // item's selection is read while the current item's blocks are issued.
    int k = 0, ki = 0;            // block slot, item sequence number
    bool ok = true;
    auto emit = [&](int kind, int blk, int first, int last, long long row, int sp, int pos,
                    long long page, int g) -> bool {
      bool good = true;
      if (lane == 0) {
        if (k >= kAttStages && !mbar_wait(&raw_empty[k % kAttStages], ((k / kAttStages) - 1) & 1)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 20);
          good = false;
        } else if (PRE && k >= kVB && !mbar_wait(&pv_done[k % kVB], ((k / kVB) - 1) & 1)) {
          // decode-once: V buffer k % kVB and block info slot k % 8 are free
          // once block k-kVB's O update is done
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 23);
          good = false;
        } else if (PRE) {
          const int s = k % kAttStages;
          int* bi = binfo + (k & (kRing - 1)) * kInfo;
          bi[0] = kind; bi[1] = blk; bi[2] = first; bi[3] = last;
          bi[4] = ki; bi[5] = (int)row; bi[6] = sp; bi[7] = pos;
          if (kind == kBlkLoad) {
            const long long b = row / ((long long)kG * a.T);
            const long long r0 = ((b * a.max_pages + blk) * kG + g) * kBlock;   // first decoded row
            mbar_expect_tx(&raw_full[s], 2 * kDkvTile);
            tma_load_2d(raw + s * kDkvTile, &a.tmap_kd, 0, (int)r0, &raw_full[s]);
            tma_load_2d(vbuf + (k % kVB) * kDkvTile, &a.tmap_vd, 0, (int)r0, &raw_full[s]);
          } else {
            mbar_arrive(&raw_full[s]);
          }
        } else {
          const int s = k % kAttStages;
          int* m = meta + s * kInfo;
          m[0] = kind; m[1] = blk; m[2] = first; m[3] = last;
          m[4] = ki; m[5] = (int)row; m[6] = sp; m[7] = pos;
          if (kind == kBlkLoad) {
            uint8_t* dst = raw + s * kAttRawStride;
            const long long r0 = (page * kG + g) * kBlock;      // first (page, head, token) row
            mbar_expect_tx(&raw_full[s], kAttRawStride);
            tma_load_2d(dst, &a.tmap_k, 0, (int)r0, &raw_full[s]);
            tma_load_2d(dst + kPageCodes, &a.tmap_v, 0, (int)r0, &raw_full[s]);
            bulk_g2s(dst + 2 * kPageCodes, a.k_scale + r0 * kRowScales, kPageScales, &raw_full[s]);
            bulk_g2s(dst + 2 * kPageCodes + kPageScales, a.v_scale + r0 * kRowScales, kPageScales,
                     &raw_full[s]);
          } else {
            mbar_arrive(&raw_full[s]);
          }
        }
      }
      good = __shfl_sync(0xffffffffu, good, 0);
      ++k;
      return good;
    };
    // Item lookup, one lane per selected block of the item's slice, in two
    // steps one item apart, so that no global load is waited for right after
    // it is issued: lookup_sel reads the item's length and selected block id
    // (two items ahead), lookup_page its page-table entry (one item ahead).
    struct Look { long long it, row; int sp, b, t, g, L, blk; long long page; };
    auto lookup_sel = [&](long long it) -> Look {
      Look r{};
      r.it = it;
      r.page = -1;
      r.blk = -1;
      if (it >= items) return r;
      r.row = it / a.splits;
      r.sp = (int)(it % a.splits);
      r.b = (int)(r.row / (kG * a.T));
      r.t = (int)((r.row / kG) % a.T);
      r.g = (int)(r.row % kG);
      r.L = a.seq_lens[r.b];
      const int k0 = kTopk * r.sp / a.splits, k1 = kTopk * (r.sp + 1) / a.splits;
      if (lane >= k0 && lane < k1) r.blk = a.sel[r.row * kTopk + lane];
      return r;
    };
    auto lookup_page = [&](Look& r) {
      if (r.it >= items) return;
      const bool len_ok = r.L >= a.T && r.L <= a.max_pages * kBlock;
      if (!len_ok || r.blk < 0 || r.blk >= (r.L - a.T + r.t) / kBlock + 1) return;
      r.page = a.page_table ? (long long)a.page_table[(long long)r.b * a.max_pages + r.blk]
                            : (long long)r.b * a.max_pages + r.blk;
    };
    // Items are claimed three ahead: the claim of item n+3 is issued before
    // item n's blocks, and its value is only read one item later.
    long long c0 = 0, c1 = 0, nxt2 = 0, claim = 0;
    if (lane == 0) {
      c0 = atomicAdd(&a.work[0], 1);
      c1 = atomicAdd(&a.work[0], 1);
      nxt2 = atomicAdd(&a.work[0], 1);
    }
    Look cur = lookup_sel(__shfl_sync(0xffffffffu, c0, 0));
    lookup_page(cur);
    Look next = lookup_sel(__shfl_sync(0xffffffffu, c1, 0));
    long long item = cur.it;
    while (item < items && ok) {
      if (lane == 0) claim = atomicAdd(&a.work[0], 1);
      lookup_page(next);
      const Look next2 = lookup_sel(__shfl_sync(0xffffffffu, nxt2, 0));
      const long long row = cur.row;
      const int sp = cur.sp, b = cur.b, t = cur.t, g = cur.g, L = cur.L;
      const bool len_ok = L >= a.T && L <= a.max_pages * kBlock;
      const int pos = L - a.T + t;
      const int nvis = pos / kBlock + 1;
      const int k0 = kTopk * sp / a.splits, k1 = kTopk * (sp + 1) / a.splits;
      if (lane == 0 && !len_ok && sp == 0 && g == 0 && t == 0) report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
      // lane kk: selected block kk of this slice, validated
      int blk = -1;
      long long page = -1;
      bool valid = false;
      if (len_ok && lane >= k0 && lane < k1) {
        blk = cur.blk;
        if (blk >= nvis) {
          report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, blk);
        } else if (blk >= 0) {
          page = cur.page;                         // looked up one item ago
          if (page < 0 || page >= a.num_pages) report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)page);
          else valid = true;
        }
      }
      const unsigned vmask = __ballot_sync(0xffffffffu, valid);
      // the query rows of this item (previous user: item ki-2's last S MMA)
      const int qs = ki & 1;
      if (lane == 0) {
        if (ki >= 2 && !mbar_wait(&q_empty[qs], ((ki >> 1) - 1) & 1)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 21);
          ok = false;
        } else if (vmask != 0u) {
          mbar_expect_tx(&q_full[qs], kHpg * kDim);
          tma_load_2d(qbuf + qs * kHpg * kDim, &a.tmap_q, 0,
                      (int)(((long long)b * a.T + t) * kHq + kHpg * g), &q_full[qs]);
        } else {
          mbar_arrive(&q_full[qs]);   // keeps the phase count; nothing waits on it
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      if (!ok) break;
      if (vmask == 0u) {
        ok = emit(kBlkEmpty, 0, 1, 1, row, sp, pos, 0, g);
      } else {
        const int lastk = 31 - __clz(vmask);
        for (unsigned m = vmask; m != 0u && ok; m &= m - 1u) {
          const int kk = __ffs(m) - 1;
          const int bk = __shfl_sync(0xffffffffu, blk, kk);
          const long long pk = __shfl_sync(0xffffffffu, page, kk);
          ok = emit(kBlkLoad, bk, m == vmask, kk == lastk, row, sp, pos, pk, g);
        }
      }
      ++ki;
      cur = next;
      next = next2;
      item = cur.it;
      nxt2 = claim;                                   // lane 0's value, broadcast next time
    }
    if (ok) emit(kBlkEnd, 0, 0, 0, 0, 0, 0, 0, 0);
    // every CTA has made its last claim once all have arrived here
    if (lane == 0) {
      __threadfence();
      if (atomicAdd(&a.work[1], 1) == (int)gridDim.x - 1) {
        atomicExch(&a.work[0], 0);
        atomicExch(&a.work[1], 0);
      }
    }
  } else if (warp == kAttMmaWarp) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_e4m3_f32(128, kHpg);
      constexpr uint32_t idesc_o = idesc_e4m3_f32(128, 2 * kHpg) | (1u << 15) | (1u << 16);
      const uint64_t qd0 = desc_kmajor_sw128(smem_u32(qbuf));
      const uint64_t qd1 = desc_kmajor_sw128(smem_u32(qbuf + kHpg * kDim));
      // The S and O streams run independently: S of block ks as soon as its K
      // is decoded and the softmax has read S of block ks-2 (same buffer);
      // O of block ko as soon as its P is written.  Both are polled without
      // blocking, so neither waits behind the other.
      int ks = 0, ko = 0, s_end = -1;                 // next S, next O, index of the end block
      uint32_t idle = 0;
      for (;;) {
        bool did = false;
        if (s_end < 0) {
          const int x = ks & 1;
          const bool in = PRE ? mbar_test(&raw_full[ks % kAttStages], (ks / kAttStages) & 1)
                              : mbar_test(&kv_full[x], (ks >> 1) & 1);
          if (in && (ks < 2 || mbar_test(&s_free[x], ((ks >> 1) - 1) & 1))) {
            tc_fence_after();
            const int* bi = binfo + (ks & (kRing - 1)) * kInfo;
            const int kind = bi[0], first = bi[2], last = bi[3], ki = bi[4];
            if (kind != kBlkLoad || !first || mbar_test(&q_full[ki & 1], (ki >> 1) & 1)) {
              if (kind == kBlkLoad) {
                tc_fence_after();
                const uint32_t d = tmem + kColS + kHpg * x;
                const uint64_t bd = (ki & 1) ? qd1 : qd0;
                if constexpr (PRE) {   // A = the block's E4M3 K rows in the stage
                  const uint64_t ad = desc_kmajor_sw128(smem_u32(raw + (ks % kAttStages) * kDkvTile));
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk) tc_mma_ss(d, ad + 2 * kk, bd + 2 * kk, idesc_s, kk > 0);
                } else {
                  const uint32_t ta = tmem + kColA + 32 * x;
#pragma unroll
                  for (int kk = 0; kk < 4; ++kk) tc_mma_e4m3_ts(d, ta + 8 * kk, bd + 2 * kk, idesc_s, kk > 0);
                }
              }
              tc_commit(&s_full[x]);
              if (PRE) tc_commit(&raw_empty[ks % kAttStages]);   // the stage was the A operand
              if (kind != kBlkEnd && last) tc_commit(&q_empty[ki & 1]);
              if (kind == kBlkEnd) s_end = ks;
              ++ks;
              did = true;
            }
          }
        }
        if (ko < ks && (s_end < 0 || ko < s_end)) {
          // P of block ko: p_full[ko % kVB].  Its previous phase (block
          // ko-kVB) was taken here before the softmax, which waits for that
          // block's O update, could start block ko: phases never alias
          if (mbar_test(&p_full[ko % kVB], (ko / kVB) & 1) &&
              (PRE || !kKVSplit || mbar_test(&v_full[ko % kVB], (ko / kVB) & 1))) {
            tc_fence_after();
            const int* bi = binfo + (ko & (kRing - 1)) * kInfo;
            const int kind = bi[0], first = bi[2], ki = bi[4];
            const int ob = ki & 1;
            if (!(first && ki >= 2) || mbar_test(&o_free[ob], ((ki >> 1) - 1) & 1)) {
              tc_fence_after();
              if (kind == kBlkLoad) {
                const uint32_t d = tmem + kColO + 2 * kHpg * ob;
                const uint32_t va = smem_u32(vbuf + (ko % kVB) * kBlock * kDim);
                const uint32_t pa = smem_u32(pbuf + (ko % kVB) * 2 * kBlock * kHpg);
#pragma unroll
                for (int kk = 0; kk < 4; ++kk)   // 32 keys per slice
                  tc_mma_ss(d, desc_mn_sw128(va + kk * 32 * kDim, 1024),
                            desc_mn_plain(pa + kk * 32 * kHpg, 8 * kHpg, kBlock * kHpg), idesc_o,
                            (first && kk == 0) ? 0u : 1u);
              }
              tc_commit(&pv_done[ko % kVB]);
              ++ko;
              did = true;
            }
          }
        }
        if (s_end >= 0 && ko >= s_end) break;
        if (did) {
          idle = 0;
        } else if (++idle > kPollLimit) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 22);
          break;
        } else if (idle > 32) {
          __nanosleep(64);
        }
      }
    }
  } else if (warp >= kAttSoftWarp0) {
    // ------------------------------------------------------------ softmax
    // warp kAttSoftWarp0 + 4*hh + q: keys (TMEM lanes) 32q..32q+31, heads kHh*hh..kHh*hh+kHh-1
    const int q = warp & 3, hh = (warp - kAttSoftWarp0) >> 2, h0 = kHh * hh;
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    const float c = a.logit_scale_log2;               // softmax_scale * s_q * s_k * log2(e)
    float* mybc = bc + (warp - kAttSoftWarp0) * 2 * kHh;   // this warp's broadcast slot
    float lt[kHh];                                    // this key lane's share of the row sums
#pragma unroll
    for (int h = 0; h < kHh; ++h) lt[h] = 0.f;
    float m_used = -INFINITY;                         // lanes < kHh: running max of head h0+lane
    int nred = 0, nmisc = 0, nitem = 0;
    for (int k = 0;; ++k) {
      const int x = k & 1;
      if (!mbar_wait(&s_full[x], (k >> 1) & 1)) { report(a.flags, 5, 26); break; }
      tc_fence_after();
      const int* bi = binfo + (k & (kRing - 1)) * kInfo;
      const int kind = bi[0], blk = bi[1], first = bi[2], last = bi[3], ki = bi[4];
      const long long row = bi[5];
      const int sp = bi[6], pos = bi[7];
      if (kind == kBlkEnd) break;
      const int ob = ki & 1;
      const int vb = k % kVB;                          // P buffer (its last reader: block k-kVB's O)
      if (k >= kVB && !mbar_wait(&pv_done[vb], ((k / kVB) - 1) & 1)) { report(a.flags, 5, 27); break; }
      float s[kHh];
      if (kind == kBlkLoad) {
#pragma unroll
        for (int j = 0; j < kHh / 8; ++j)
          tmem_ld8(lane_base + kColS + kHpg * x + h0 + 8 * j, *reinterpret_cast<float(*)[8]>(s + 8 * j));
        tmem_wait_ld();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&s_free[x]);     // S buffer x may be overwritten (block k+2)
      if (kind == kBlkLoad) {
        if (blk * kBlock + 32 * q + lane > pos) {      // key after the query position
#pragma unroll
          for (int h = 0; h < kHh; ++h) s[h] = -INFINITY;
        }
        // block maximum per head: this warp's 32 keys, then the four quarters
        float* rq = red + ((nred & 1) * 4 + q) * kHpg + h0;
        float mh[kHh];
#pragma unroll
        for (int h = 0; h < kHh; ++h) mh[h] = warp_max(s[h]);
        if (lane == 0) {
#pragma unroll
          for (int j = 0; j < kHh / 4; ++j)
            reinterpret_cast<float4*>(rq)[j] = make_float4(mh[4 * j], mh[4 * j + 1], mh[4 * j + 2], mh[4 * j + 3]);
        }
        __syncwarp();
        if (lane == 0) mbar_arrive(red_full);
        if (!mbar_wait(red_full, nred & 1)) { report(a.flags, 5, 28); break; }
        int resc = 0;
        if (lane < kHh) {
          const float* rr = red + (nred & 1) * 4 * kHpg + h0 + lane;
          const float mb = fmaxf(fmaxf(rr[0], rr[kHpg]), fmaxf(rr[2 * kHpg], rr[3 * kHpg]));
          float alpha = 1.f;
          if (first) {
            m_used = mb;
          } else if ((mb - m_used) * c > kLazy) {
            alpha = ex2((m_used - mb) * c);
            m_used = mb;
            resc = 1;
          }
          mybc[lane] = m_used * c - kPExp;               // exponent offset of head h0+lane
          mybc[kHh + lane] = alpha;
        }
        ++nred;
        resc = __any_sync(0xffffffffu, resc);
        __syncwarp();
        if (resc) {   // raise m: rescale the row sums and O^T (after block k-1's update)
          const float* al = mybc + kHh;
#pragma unroll
          for (int h = 0; h < kHh; ++h) lt[h] *= al[h];
          if (!mbar_wait(&pv_done[(k - 1) % kVB], ((k - 1) / kVB) & 1)) { report(a.flags, 5, 29); break; }
          tc_fence_after();
          const uint32_t oa = lane_base + kColO + 2 * kHpg * ob + h0;
#pragma unroll 1
          for (int j = 0; j < 2 * (kHh / 8); ++j) {   // hi, lo columns of heads h0.., eight at a time
            const int hg = 8 * (j % (kHh / 8)), col = kHpg * (j / (kHh / 8)) + hg;
            float o8[8];
            tmem_ld8(oa + col, o8);
            tmem_wait_ld();
            uint32_t w8[8];
#pragma unroll
            for (int i = 0; i < 8; ++i) w8[i] = __float_as_uint(o8[i] * al[hg + i]);
            tmem_st8(oa + col, w8);
          }
          tmem_wait_st();
        }
        // P = 2^(s c - m c + 4) as hi + lo E4M3: bytes h0..h0+kHh-1 of the key's rows
        uint32_t ph[kHh / 4], pl[kHh / 4];
#pragma unroll
        for (int h2 = 0; h2 < kHh / 2; ++h2) {
          const float2 mo = *reinterpret_cast<const float2*>(mybc + 2 * h2);   // exponent offsets
          const float p0 = ex2(fmaf(s[2 * h2], c, -mo.x));
          const float p1 = ex2(fmaf(s[2 * h2 + 1], c, -mo.y));
          lt[2 * h2] += p0;
          lt[2 * h2 + 1] += p1;
          uint32_t hw, lw;
          p_split_e4m3x2(p0, p1, hw, lw);
          if (h2 & 1) { ph[h2 >> 1] |= hw << 16; pl[h2 >> 1] |= lw << 16; }
          else { ph[h2 >> 1] = hw; pl[h2 >> 1] = lw; }
        }
        uint8_t* pb = pbuf + vb * 2 * kBlock * kHpg + (32 * q + lane) * kHpg + h0;
        if constexpr (kHh == 16) {
          *reinterpret_cast<uint4*>(pb) = make_uint4(ph[0], ph[1], ph[2], ph[3]);
          *reinterpret_cast<uint4*>(pb + kBlock * kHpg) = make_uint4(pl[0], pl[1], pl[2], pl[3]);
        } else {
          *reinterpret_cast<uint2*>(pb) = make_uint2(ph[0], ph[1]);
          *reinterpret_cast<uint2*>(pb + kBlock * kHpg) = make_uint2(pl[0], pl[1]);
        }
        fence_async_smem();
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&p_full[vb]);
      if (!last) continue;

      // ---------------------------------------------------- end of the item
      // The item's last O update (for an empty item: the O stream's pass over
      // its block, which takes o_free's phase of item ki-2) before o_free's
      // phase of this item; then the row sums: this warp's 32 keys, then the
      // four quarters
      if (!mbar_wait(&pv_done[vb], (k / kVB) & 1)) { report(a.flags, 5, 30); break; }
      tc_fence_after();
#pragma unroll
      for (int h = 0; h < kHh; ++h) {
        float v = lt[h];
        v += __shfl_xor_sync(0xffffffffu, v, 16);
        v += __shfl_xor_sync(0xffffffffu, v, 8);
        v += __shfl_xor_sync(0xffffffffu, v, 4);
        v += __shfl_xor_sync(0xffffffffu, v, 2);
        v += __shfl_xor_sync(0xffffffffu, v, 1);
        if (lane == h) lsum[((nitem & 1) * 4 + q) * kHpg + h0 + h] = v;
        lt[h] = 0.f;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(misc_bar);
      if (!mbar_wait(misc_bar, (nmisc++) & 1)) { report(a.flags, 5, 31); break; }
      const float* ls = lsum + (nitem & 1) * 4 * kHpg + h0;   // [quarter][16] row sums
      const float mc = m_used * c;                     // lanes < kHh: m of head h0+lane, log2 units
      const int d = 32 * q + lane;                     // this thread's dimension
      const int b = (int)(row / (kG * a.T));
      const int t = (int)((row / kG) % a.T);
      const int g = (int)(row % kG);
      // O = O_hi + O_lo of heads h0..h0+kHh-1, then release O^T
      float o[kHh];
#pragma unroll
      for (int j = 0; j < kHh / 8; ++j) {
        float hi8[8], lo8[8];
        if (kind == kBlkLoad) {
          tmem_ld8(lane_base + kColO + 2 * kHpg * ob + h0 + 8 * j, hi8);
          tmem_ld8(lane_base + kColO + 2 * kHpg * ob + kHpg + h0 + 8 * j, lo8);
          tmem_wait_ld();
        } else {
#pragma unroll
          for (int i = 0; i < 8; ++i) hi8[i] = lo8[i] = 0.f;
        }
#pragma unroll
        for (int i = 0; i < 8; ++i) o[8 * j + i] = hi8[i] + lo8[i];
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&o_free[ob]);
      // lanes < kHh: the row sum of head h0+lane over the four quarters
      const float lrow = lane < kHh ? ls[lane] + ls[kHpg + lane] + ls[2 * kHpg + lane] + ls[3 * kHpg + lane]
                                    : 0.f;
      if (a.splits == 1) {
        const float f = lrow > 0.f ? a.out_scale / lrow : 0.f;   // lanes < kHh
        uint16_t* dst = a.out + (((long long)b * a.T + t) * kHq + kHpg * g + h0) * kDim + d;
#pragma unroll
        for (int h = 0; h < kHh; ++h) {
          const float v = o[h] * __shfl_sync(0xffffffffu, f, h);
          const __nv_bfloat16 bv = __float2bfloat16_rn(v);
          dst[(long long)h * kDim] = *reinterpret_cast<const uint16_t*>(&bv);
        }
      } else {
        // fp32 partial of this split: O (in units of 2^4 P), m (log2 units), l
        float* part = a.partials + (row * a.splits + sp) * kPartialFloats;
#pragma unroll
        for (int h = 0; h < kHh; ++h) part[(h0 + h) * kDim + d] = o[h];
        if (q == 0 && lane < kHh) {
          part[kHpg * kDim + h0 + lane] = kind == kBlkLoad ? mc : -INFINITY;
          part[kHpg * kDim + kHpg + h0 + lane] = lrow;
        }
        // all eight warps' partials written and fenced, then one thread counts
        // this split in; the result reaches the warps through shared memory
        __threadfence();
        __syncwarp();
        if (lane == 0) mbar_arrive(misc_bar);
        if (!mbar_wait(misc_bar, (nmisc++) & 1)) { report(a.flags, 5, 32); break; }
        if (warp == kAttSoftWarp0 && lane == 0)
          misc[nitem & 1] = (atomicAdd(&a.counters[row], 1) == a.splits - 1);
        __syncwarp();
        if (lane == 0) mbar_arrive(misc_bar);
        if (!mbar_wait(misc_bar, (nmisc++) & 1)) { report(a.flags, 5, 35); break; }
        if (misc[nitem & 1]) {
          __threadfence();
          // kAttSoft x 32 threads: head hr, kDpt dims from d0
          constexpr int kDpt = kHpg * kDim / (kAttSoft * 32), kTph = kDim / kDpt;   // dims / thread, threads / head
          const int tq = (warp - kAttSoftWarp0) * 32 + lane, hr = tq / kTph, d0 = (tq % kTph) * kDpt;
          const float* base = a.partials + row * a.splits * kPartialFloats;
          float Mx = -INFINITY;
          for (int s2 = 0; s2 < a.splits; ++s2)
            Mx = fmaxf(Mx, __ldcg(base + s2 * kPartialFloats + kHpg * kDim + hr));
          const float Mu = (Mx == -INFINITY) ? 0.f : Mx;
          float tot[kDpt];
#pragma unroll
          for (int cc = 0; cc < kDpt; ++cc) tot[cc] = 0.f;
          float Lt = 0.f;
          for (int s2 = 0; s2 < a.splits; ++s2) {
            const float* ps2 = base + s2 * kPartialFloats;
            const float f = exp2f(__ldcg(ps2 + kHpg * kDim + hr) - Mu);
            Lt += __ldcg(ps2 + kHpg * kDim + kHpg + hr) * f;
#pragma unroll
            for (int cc = 0; cc < kDpt; ++cc) tot[cc] += __ldcg(ps2 + hr * kDim + d0 + cc) * f;
          }
          const float inv = Lt > 0.f ? a.out_scale / Lt : 0.f;
          uint32_t packed[kDpt / 2];
#pragma unroll
          for (int cc = 0; cc < kDpt / 2; ++cc) {
            const __nv_bfloat162 v = __floats2bfloat162_rn(tot[2 * cc] * inv, tot[2 * cc + 1] * inv);
            packed[cc] = *reinterpret_cast<const uint32_t*>(&v);
          }
          uint4* op = reinterpret_cast<uint4*>(a.out + (((long long)b * a.T + t) * kHq + kHpg * g + hr) * kDim + d0);
#pragma unroll
          for (int cc = 0; cc < kDpt / 8; ++cc)
            op[cc] = make_uint4(packed[4 * cc], packed[4 * cc + 1], packed[4 * cc + 2], packed[4 * cc + 3]);
          if (tq == 0) a.counters[row] = 0;   // ready for the next call
        }
      }
      ++nitem;
      m_used = -INFINITY;
    }
  } else if (!PRE) {
    // ------------------------------------------------------------ decoders
    // warps 0-3 decode K (and, without the split, V); warps 4-7 decode V
    const bool vdec = kKVSplit && warp >= kAttVWarp0;
    const bool kdec = !vdec;
    const int qd = warp & 3;                         // row block = TMEM lane quarter
    const uint32_t lane_base = tmem + ((uint32_t)(32 * qd) << 16);
    const int row = 32 * qd + lane;                  // key row of this thread
    const int sw = (row >> 1) & 3;                   // 64-byte swizzle of the code rows
    for (int k = 0;; ++k) {
      const int s = k % kAttStages, x = k & 1;
      if (!mbar_wait(&raw_full[s], (k / kAttStages) & 1)) { report(a.flags, 5, 33); break; }
      // A[x] was last read by block k-2's S; V buffer k % kVB by block k-kVB's O
      if (kdec && k >= 2 && !mbar_wait(&s_full[x], ((k >> 1) - 1) & 1)) { report(a.flags, 5, 34); break; }
      if ((vdec || !kKVSplit) && k >= kVB && !mbar_wait(&pv_done[k % kVB], ((k / kVB) - 1) & 1)) {
        report(a.flags, 5, 36);
        break;
      }
      tc_fence_after();
      const int* m = meta + s * kInfo;
      const int kind = m[0];
      if (kind == kBlkLoad) {
        const uint8_t* rs = raw + s * kAttRawStride;
        const uint8_t* kc = rs;
        const uint8_t* vc = rs + kPageCodes;
        const uint8_t* ks = rs + 2 * kPageCodes;
        const uint8_t* vs = ks + kPageScales;
        if (kdec) {
          // K signed, as E4M3 into A[x] (row = TMEM lane, 32 columns)
          const uint32_t abase = lane_base + kColA + 32 * x;
          const uint2 ksc = *reinterpret_cast<const uint2*>(ks + row * kRowScales);
#pragma unroll
          for (int cix = 0; cix < 4; ++cix) {
            const uint4 w4 = lds128(kc + row * kRowCodes + ((cix ^ sw) << 4));
            const uint32_t sb = (cix < 2 ? ksc.x : ksc.y) >> (16 * (cix & 1));
            const uint2 r0 = lut[sb & 0xFFu], r1 = lut[(sb >> 8) & 0xFFu];
            uint32_t o[8];
            dq8(w4.x, r0, o[0], o[1]);
            dq8(w4.y, r0, o[2], o[3]);
            dq8(w4.z, r1, o[4], o[5]);
            dq8(w4.w, r1, o[6], o[7]);
            tmem_st8(abase + 8 * cix, o);
          }
          tmem_wait_st();
        }
        if (vdec || !kKVSplit) {
          // V signed, as E4M3 into the 128-byte V row of this key (16-byte
          // chunk j at chunk position j ^ (key % 8))
          const uint2 vsc = *reinterpret_cast<const uint2*>(vs + row * kRowScales);
          uint8_t* vrow = vbuf + (k % kVB) * kBlock * kDim + row * kDim;
#pragma unroll
          for (int cix = 0; cix < 4; ++cix) {
            const uint4 w4 = lds128(vc + row * kRowCodes + ((cix ^ sw) << 4));
            const uint32_t sb = (cix < 2 ? vsc.x : vsc.y) >> (16 * (cix & 1));
            const uint2 r0 = lut[sb & 0xFFu], r1 = lut[(sb >> 8) & 0xFFu];
            uint32_t o[8];
            dq8(w4.x, r0, o[0], o[1]);
            dq8(w4.y, r0, o[2], o[3]);
            dq8(w4.z, r1, o[4], o[5]);
            dq8(w4.w, r1, o[6], o[7]);
            // code chunk cix = dims 32cix..32cix+31 = V chunks 2cix, 2cix+1
            *reinterpret_cast<uint4*>(vrow + (((2 * cix) ^ (row & 7)) << 4)) = make_uint4(o[0], o[1], o[2], o[3]);
            *reinterpret_cast<uint4*>(vrow + (((2 * cix + 1) ^ (row & 7)) << 4)) =
                make_uint4(o[4], o[5], o[6], o[7]);
          }
          fence_async_smem();
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) {
        // the block info leaves the stage before the stage is released (the
        // producer rewrites it for block k + kAttStages right after); the
        // ring of kRing slots outlives every reader: slot k is rewritten at
        // block k + kRing, after block k + kRing - 2's S, hence after the
        // softmax of block k + kRing - 4 began, which waited for block
        // k + kRing - 4 - kVB's O update (and the O stream runs in order)
        if (warp == 0) {
          int* bi = binfo + (k & (kRing - 1)) * kInfo;
#pragma unroll
          for (int i = 0; i < kInfo; ++i) bi[i] = m[i];
        }
        mbar_arrive(&raw_empty[s]);
        if (vdec) mbar_arrive(&v_full[k % kVB]);
        else mbar_arrive(&kv_full[x]);
      }
      if (kind == kBlkEnd) break;
    }
  }

  // ---- teardown: every role leaves its loop (normally or on a timeout)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kAttMmaWarp) tmem_dealloc(tmem, kAttTmemCols);
}

// Decode-once pass: every visible block of every sequence, K and V of each
// KV head, decoded to E4M3 (the same dq8 rounding as the attention's own
// decoders) into the workspace rows the decode-once attention loads.  One
// thread per key row; tiles (sequence, block, head, K or V) grid-strided.
__global__ void __launch_bounds__(kBlock) dkv_kernel(const __grid_constant__ AttnArgs a) {
  __shared__ uint2 lut[256];
  build_nvfp4_lut(lut, threadIdx.x, blockDim.x);
  __syncthreads();
  const int row = threadIdx.x;
  const long long tiles = (long long)a.B * a.max_pages * kG * 2;
  for (long long tile = blockIdx.x; tile < tiles; tile += gridDim.x) {
    const int kv = (int)(tile & 1);
    const long long r = tile >> 1;
    const int g = (int)(r % kG);
    const int blk = (int)((r / kG) % a.max_pages);
    const int b = (int)(r / ((long long)kG * a.max_pages));
    const int L = a.seq_lens[b];
    // invalid lengths and page ids are reported by the attention itself
    if (L < a.T || L > a.max_pages * kBlock || blk * kBlock >= L) continue;
    const long long page = a.page_table ? (long long)a.page_table[(long long)b * a.max_pages + blk]
                                        : (long long)b * a.max_pages + blk;
    if (page < 0 || page >= a.num_pages) continue;
    const long long src = (page * kG + g) * kBlock + row;              // (page, head, token) row
    const uint8_t* codes = (kv ? a.v_data : a.k_data) + src * kRowCodes;
    const uint2 sc = *reinterpret_cast<const uint2*>((kv ? a.v_scale : a.k_scale) + src * kRowScales);
    uint8_t* dst = (kv ? a.vd : a.kd) + ((((long long)b * a.max_pages + blk) * kG + g) * kBlock + row) * kDim;
#pragma unroll
    for (int c = 0; c < 4; ++c) {   // 32 codes under scale bytes 2c, 2c+1
      const uint4 w4 = *reinterpret_cast<const uint4*>(codes + 16 * c);
      const uint32_t sb = (c < 2 ? sc.x : sc.y) >> (16 * (c & 1));
      const uint2 r0 = lut[sb & 0xFFu], r1 = lut[(sb >> 8) & 0xFFu];
      uint32_t o[8];
      dq8(w4.x, r0, o[0], o[1]);
      dq8(w4.y, r0, o[2], o[3]);
      dq8(w4.z, r1, o[4], o[5]);
      dq8(w4.w, r1, o[6], o[7]);
      *reinterpret_cast<uint4*>(dst + 32 * c) = make_uint4(o[0], o[1], o[2], o[3]);
      *reinterpret_cast<uint4*>(dst + 32 * c + 16) = make_uint4(o[4], o[5], o[6], o[7]);
    }
  }
}

template <bool PRE>
static cudaError_t launch_attn_mode(const AttnArgs& a, cudaStream_t st) {
  const size_t smem = (size_t)att_layout<PRE>().total;
  int grid = 0;
  cudaError_t e = persistent_grid(reinterpret_cast<const void*>(attn_kernel<PRE>), kAttThreads, smem,
                                  kAttTmemCols, &grid);
  if (e != cudaSuccess) return e;
  return launch_dependent(attn_kernel<PRE>, dim3(grid), dim3(kAttThreads), smem, st, a);
}

cudaError_t launch_attn(const AttnArgs& a, cudaStream_t st) {
  if (!a.dkv) return launch_attn_mode<false>(a, st);
  int dev = 0, sms = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e == cudaSuccess) e = cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  if (e != cudaSuccess) return e;
  const long long tiles = (long long)a.B * a.max_pages * kG * 2;
  const int grid = (int)std::min<long long>(tiles, 8LL * sms);
  dkv_kernel<<<grid, kBlock, 0, st>>>(a);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return launch_attn_mode<true>(a, st);
}

// ----------------------------------------------------- parity debug hook --
// The kernels' NVFP4 -> E4M3 table through the signed decode every kernel
// uses (dq8): out[s*16 + c] for scale byte s and code c.
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
