// msa_indexer.cu -- indexer scores + block max-pool on the 5th-generation
// tensor core ([post, "MSA primer"]: one index query per GQA group scores
// every cached key against one shared index-key head; the scores are
// max-pooled to one score per 128-token block).
// post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援 (hot.atechcom.net).
//
// Per page (= one 128-token block) the scores are one dense contraction
//   D[M queries x 128 keys] = Qi[M x 128] * K_page[128 keys x 128]^T
// with a tile of index queries as the M side (T tokens x 4 groups; M = 64
// when the tile holds at most 64 index queries, else tiles of 128) and the
// page's keys as the N side.  Each query's row of D then sits in one TMEM
// lane, so the block max is a reduction along the lane's columns: inside the
// thread, plus two shuffles when a 16x256b load spreads a row over four
// threads.  With M = 64 the accumulator occupies lanes 0-15 of each 32-lane
// quarter (rows 16q..16q+15 in quarter q).
//
// Work split: the pages of all sequences form one flat list, cut into chunks
// of kChunkPages; a work item is (query tile, chunk).  A launch may score
// only part `part` of `nparts` of every sequence's blocks (the context split
// of [post, "NVFP4 indexer DCP"]); the flat list then holds only those
// blocks.  Persistent CTAs take items from a counter in the workspace header
// as they go (ragged batches and CTAs sharing an SM still finish together);
// the last CTA to finish resets the counter.  Warp roles, a few pages apart:
//   warp 12 (producer): the whole warp looks up the pages of the next work
//     item (one lane per page: sequence, logical block, page table entry)
//     and issues the current item's pages, lane j page j, as their stages
//     free: per page one tiled TMA load of the codes (64-byte swizzle, so
//     that row-per-thread reads are bank-conflict free) and one bulk copy of
//     the scales into a ring of shared-memory stages (FP8 index keys: one TMA
//     load with the 128-byte swizzle, which is already the MMA's B operand);
//     and, per item, the TMA load of the item's index-query tile;
//   warps 0-3 (decoders): thread = key row.  NVFP4 is decoded to signed E4M3
//     (dq8: a table row per scale byte, byte permutes for magnitudes and
//     signs) and stored as 128-byte rows with the 128-byte swizzle -- the
//     K-major B operand -- into one of two buffers, so that page k+1 is
//     decoded while page k's MMAs run (FP16 mode: they also stage the
//     tile's index queries, the A operand, when the tile changes);
//   warp 13 (MMA): one thread issues per page 4 tcgen05.mma of K = 32 (E4M3;
//     8 of K = 16 for FP16) into TMEM accumulator k % 2;
//   warps 4-11 (epilogue): warp w reads the accumulator lanes of quarter
//     w % 4 for the pages of parity (w - 4) / 4, so that two pages are read
//     out at once; it masks keys after each query's position, takes each
//     query's maximum over the page's keys and writes the block score.  The
//     producer ends the page stream with two end markers, one per parity.
// Every wait is a bounded mbarrier wait; on a timeout a thread records
// MSA_ERR_TIMEOUT and leaves its loop, and TMEM is freed before exit.
//
// Modes (the template parameter MODE):
//   kIdxNvfp4  NVFP4 keys re-rounded to E4M3, FP8 MMA (the decode above);
//   kIdxFp8    E4M3 keys, scored from the TMA buffer as they are;
//   kIdxF16    NVFP4 keys decoded exactly to FP16 (e2m1 x scale needs no
//              rounding in FP16) and scored with FP16 MMA against the index
//              queries widened to FP16 -- the exact scores of [post, "NVIDIA
//              Rubin optimized MSA"].  Query and key rows are 256 bytes, held
//              as two 128-byte K-halves; 8 MMAs of K = 16 per page.
#include "msa_internal.h"

namespace msa {

constexpr int kIdxDecWarps = 4;             // warps 0-3: one key row per thread
constexpr int kIdxEpiWarp0 = 4;             // warps 4-11: lane quarter warp % 4, pages of parity (warp - 4) / 4
constexpr int kIdxProducerWarp = 12;
constexpr int kIdxMmaWarp = 13;
static_assert(kIdxThreads == 14 * 32, "warp roles");

enum : int { kPageLoad = 0, kPageMasked = 1, kPageBad = 2, kPageEnd = 3 };
constexpr int kChunkPages = 8;              // pages per work item
constexpr int kInfoRing = 8;                // per-page info slots (decoders -> MMA, epilogue)
constexpr int kIdxTmemCols = 256;           // two accumulators of 128 columns

template <int MODE, int M>
struct IdxCfg {
  static constexpr bool kFp8 = MODE == kIdxFp8;
  static constexpr bool kF16 = MODE == kIdxF16;
  static constexpr int kRow = kF16 ? 256 : 128;            // bytes per query / key row
  static constexpr int kRaw = kFp8 ? kBlock * kDim : kPageCodes + kPageScales;
  static constexpr int kRawStride = (kRaw + 1023) / 1024 * 1024;
  // raw pages in flight, as many as leave room for two CTAs per SM: 6 (FP8
  // pages, twice as large: 5), 4 with 128-row query tiles
  static constexpr int kStages = kF16 ? 3 : M == 128 ? 4 : kFp8 ? 5 : 6;
  static constexpr int kNB = kFp8 ? 0 : 2;                 // decoded key pages (B operand), page k in k % kNB
  static constexpr int kBR = kFp8 ? 2 : kNB;               // page-ready barriers (FP8: the raw stage is B)
  static constexpr int kBBytes = kBlock * kRow;
};

struct IdxLayout {
  int qbuf, raw, bbuf, lut, bars, meta, pinfo, tslot, prefix, scratch, total;
};

template <int MODE, int M>
__host__ __device__ inline IdxLayout idx_layout(int batch) {
  using C = IdxCfg<MODE, M>;
  IdxLayout L;
  int off = 0;
  L.qbuf = off;    off += (C::kF16 ? 1 : 2) * M * C::kRow;  // query tiles (multiples of 1024)
  L.raw = off;     off += C::kStages * C::kRawStride;
  L.bbuf = off;    off += C::kNB * C::kBBytes;
  L.lut = off;     off += MODE == kIdxNvfp4 ? 256 * 8 : 0;
  L.bars = off;    off += (2 * C::kStages + 2 * C::kBR + 8) * 8;
  L.meta = off;    off += C::kStages * 8 * 4;              // per stage: ptrow, i, kind, row0, row1, minpos
  L.pinfo = off;   off += kInfoRing * 8 * 4;               // per page: the same
  L.tslot = off;   off += 16;
  L.prefix = off;  off += (5 * batch + 2) * 4;           // item prefix [E+1], lengths [B], skip [B], groups
  L.scratch = off; off += kIdxThreads * 4;
  L.total = off + 1024;                                   // alignment slack
  return L;
}

// Index queries per tile: a tile is the M side of the MMA.
int idx_tile_queries(int T) { return kG * T <= 64 ? 64 : 128; }

bool idx_spread_rows(int T, int mode, int shared) { return !shared && mode != kIdxF16 && kG * T <= 32; }

size_t indexer_smem_bytes(int mode, int batch, int T) {
  const bool m64 = idx_tile_queries(T) == 64;
  if (mode == kIdxFp8) return (size_t)(m64 ? idx_layout<kIdxFp8, 64>(batch) : idx_layout<kIdxFp8, 128>(batch)).total;
  if (mode == kIdxF16) return (size_t)(m64 ? idx_layout<kIdxF16, 64>(batch) : idx_layout<kIdxF16, 128>(batch)).total;
  return (size_t)(m64 ? idx_layout<kIdxNvfp4, 64>(batch) : idx_layout<kIdxNvfp4, 128>(batch)).total;
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

// A work entity: logical blocks [lo, hi) of page-table row `ptrow`, scored
// against the index-query rows [r0, r1) (row = (b*T + t)*4 + g, the row of
// qi and of the block scores).  Without groups (or with shared = 0) entity b
// is sequence b: its blocks of this launch's part from its group's prefix
// on, against its own 4T rows.  With shared = 1 entity g is prefix group g:
// its shared blocks (the group's first sequence's page-table row) against
// the rows of all the group's sequences.
struct Ent { int lo, hi, r0, r1, ptrow; };

// Shared-memory tables (built by build_items): lengths, each sequence's own
// first block, and the prefix groups clamped to the batch and the page table.
struct Tabs { const int* lens; const int* skip; const int* gstart; const int* gpre; };

__device__ __forceinline__ Ent entity(const IdxArgs& a, int e, const Tabs& tb) {
  const int nq = kG * a.T;
  Ent r;
  if (a.shared) {
    const int s0 = tb.gstart[e], s1 = max(tb.gstart[e + 1], s0);
    r.lo = 0;
    r.hi = tb.gpre[e];
    r.r0 = s0 * nq;
    r.r1 = s1 * nq;
    r.ptrow = s0;
  } else {
    int first;
    const int nb = part_blocks(a, tb.lens[e], &first);
    r.lo = max(first, tb.skip[e]);
    r.hi = max(r.lo, first + nb);
    r.r0 = e * nq;
    r.r1 = r.r0 + nq;
    r.ptrow = e;
  }
  return r;
}

// Items (query tile x chunk of kChunkPages blocks) of an entity, M rows per tile.
template <int M>
__device__ __forceinline__ int entity_items(const Ent& E) {
  return ((E.r1 - E.r0 + M - 1) / M) * ((E.hi - E.lo + kChunkPages - 1) / kChunkPages);
}

// Shared-memory tables built by every CTA at start: the lengths lens[B], the
// first block of each sequence's own part skip[B] (its group's prefix), and
// the exclusive prefix over the entities' item counts (prefix[E] = items).
// Invalid lengths count as 0 blocks and are reported once (by CTA 0); so are
// prefix groups whose shared blocks are not entirely visible to every query
// of the group, or whose sequences do not map them to the same pages.
template <int M>
__device__ int build_items(const IdxArgs& a, int* prefix, int* lens, int* skip, int* gstart, int* gpre,
                           int* scratch) {
  const int tid = threadIdx.x, nt = blockDim.x;
  const int E = a.shared ? a.ngroups : a.B;
  for (int b = tid; b < a.B; b += nt) {
    const int L = a.seq_lens[b];
    lens[b] = L;
    skip[b] = 0;
    if ((L < a.T || L > a.max_pages * kBlock) && blockIdx.x == 0)
      report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, L);
  }
  if (a.grp_start != nullptr) {
    // clamped so that any group array stays inside the batch and the page
    // table; inconsistent arrays are reported (by CTA 0)
    for (int g = tid; g < a.ngroups; g += nt) {
      const int g0 = a.grp_start[g], g1 = a.grp_start[g + 1], gp = a.grp_prefix[g];
      const int s0 = min(max(g0, 0), a.B);
      gstart[g] = s0;
      gpre[g] = min(max(gp, 0), a.max_pages);
      if (g == a.ngroups - 1) gstart[g + 1] = min(max(g1, s0), a.B);
      if (blockIdx.x == 0 && (g0 != s0 || g1 < g0 || g1 > a.B || gp != gpre[g] ||
                              (g == 0 && g0 != 0) || (g == a.ngroups - 1 && g1 != a.B)))
        report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, g);
    }
  }
  __syncthreads();
  if (a.grp_start != nullptr) {
    for (int g = tid; g < a.ngroups; g += nt) {
      const int s0 = gstart[g], s1 = max(gstart[g + 1], s0), pre = gpre[g];
      for (int b = s0; b < s1; ++b) {
        skip[b] = pre;
        if (blockIdx.x == 0 && (long long)pre * kBlock > (long long)lens[b] - a.T)
          report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, b);
      }
    }
    // the shared blocks' page-table entries, each checked by one CTA
    if (a.shared && a.page_table != nullptr) {
      for (int g = 0; g < a.ngroups; ++g) {
        const int s0 = gstart[g], s1 = max(gstart[g + 1], s0), pre = gpre[g];
        if (s1 - s0 < 2 || pre == 0) continue;
        const long long n = (long long)(s1 - s0 - 1) * pre;
        for (long long x = (long long)blockIdx.x * nt + tid; x < n; x += (long long)gridDim.x * nt) {
          const int b = s0 + 1 + (int)(x / pre), i = (int)(x % pre);
          if (a.page_table[(long long)b * a.max_pages + i] != a.page_table[(long long)s0 * a.max_pages + i])
            report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, b);
        }
      }
    }
    __syncthreads();
  }
  const Tabs tb{lens, skip, gstart, gpre};
  const int per = (E + nt - 1) / nt;
  const int lo = tid * per, hi = min(E, lo + per);
  int sum = 0;
  for (int e = lo; e < hi; ++e) sum += entity_items<M>(entity(a, e, tb));
  scratch[tid] = sum;
  __syncthreads();
  if (tid < 32) {   // exclusive scan of the per-thread counts: lane l owns a run of them
    const int per_lane = (nt + 31) / 32;
    const int k0 = tid * per_lane, k1 = min(nt, k0 + per_lane);
    int own = 0;
    for (int k = k0; k < k1; ++k) own += scratch[k];
    int incl = own;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int v = __shfl_up_sync(0xffffffffu, incl, o);
      if (tid >= o) incl += v;
    }
    int run = incl - own;
    for (int k = k0; k < k1; ++k) { const int v = scratch[k]; scratch[k] = run; run += v; }
    if (tid == 31) prefix[E] = incl;
  }
  __syncthreads();
  int run = scratch[tid];
  for (int e = lo; e < hi; ++e) {
    prefix[e] = run;
    run += entity_items<M>(entity(a, e, tb));
  }
  __syncthreads();
  return E;
}

__device__ __forceinline__ void sts128(void* p, uint4 v) { *reinterpret_cast<uint4*>(p) = v; }

// Instruction descriptor of the page MMA: M x 128, fp32 accumulate, both
// operands K-major; E4M3 (kind::f8f6f4) or FP16 (kind::f16), whose format
// fields both read 0.
template <int M>
__host__ __device__ constexpr uint32_t idx_idesc() { return idesc_e4m3_f32(M, kBlock); }

template <int MODE, int M>
__global__ void __launch_bounds__(kIdxThreads, 2) indexer_kernel(const __grid_constant__ IdxArgs a) {
  using C = IdxCfg<MODE, M>;
  constexpr bool FP8 = C::kFp8, F16 = C::kF16;
  constexpr int S = C::kStages;
  extern __shared__ uint8_t smem_dyn[];
  uint8_t* smem = smem_dyn + ((1024u - (smem_u32(smem_dyn) & 1023u)) & 1023u);
  const IdxLayout Ly = idx_layout<MODE, M>(a.B);
  uint8_t* qbuf = smem + Ly.qbuf;
  uint8_t* raw = smem + Ly.raw;
  uint8_t* bbuf = smem + Ly.bbuf;
  uint2* lut = reinterpret_cast<uint2*>(smem + Ly.lut);
  uint64_t* raw_full = reinterpret_cast<uint64_t*>(smem + Ly.bars);
  uint64_t* raw_empty = raw_full + S;
  constexpr int BR = C::kBR;
  uint64_t* b_full = raw_empty + S;      // [BR] decoders -> MMA: page k ready (k % BR)
  uint64_t* b_empty = b_full + BR;       // [BR] MMA -> decoders: page k consumed
  uint64_t* d_full = b_empty + BR;       // [2] MMA -> epilogue
  uint64_t* d_empty = d_full + 2;        // [2] epilogue -> MMA
  uint64_t* q_full = d_empty + 2;        // [2] producer (TMA) -> MMA: an item's query tile
  uint64_t* q_empty = q_full + 2;        // [2] MMA -> producer: the item's last MMA done
  int* meta = reinterpret_cast<int*>(smem + Ly.meta);
  int* pinfo = reinterpret_cast<int*>(smem + Ly.pinfo);
  uint32_t* tslot = reinterpret_cast<uint32_t*>(smem + Ly.tslot);
  int* prefix = reinterpret_cast<int*>(smem + Ly.prefix);
  int* lens = prefix + a.B + 1;
  int* skip = lens + a.B;
  int* gstart = skip + a.B;          // [ngroups + 1] (ngroups <= B)
  int* gpre = gstart + a.B + 1;      // [ngroups]
  int* scratch = reinterpret_cast<int*>(smem + Ly.scratch);
  const Tabs tabs{lens, skip, gstart, gpre};

  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;

  if (MODE == kIdxNvfp4) build_nvfp4_lut(lut, tid, blockDim.x);
  if (tid == 0) {
    for (int s = 0; s < S; ++s) {
      mbar_init(&raw_full[s], 1);
      mbar_init(&raw_empty[s], FP8 ? 1 : kIdxDecWarps);   // FP8: released by the MMA
    }
    for (int x = 0; x < BR; ++x) {
      mbar_init(&b_full[x], kIdxDecWarps);
      mbar_init(&b_empty[x], 1);
    }
    for (int x = 0; x < 2; ++x) {
      mbar_init(&d_full[x], 1);
      mbar_init(&d_empty[x], 4);
      mbar_init(&q_full[x], 1);
      mbar_init(&q_empty[x], 1);
    }
    mbar_fence_init();
  }
  if (warp == kIdxMmaWarp) {
    tmem_alloc(tslot, kIdxTmemCols);
    tmem_relinquish();
  }
  tc_fence_before();
  const int nent = build_items<M>(a, prefix, lens, skip, gstart, gpre, scratch);   // ends with __syncthreads
  tc_fence_after();
  // the next kernel on the stream (the top-16) may start launching: its CTAs
  // take SMs as this kernel's persistent CTAs leave, and wait for its end
  grid_launch_dependents();
  const uint32_t tmem = *tslot;

  const int items = prefix[nent];
  const int nq_all = kG * a.T;                                // index queries per sequence
  const long long ctx = (long long)a.max_pages * kBlock;

  if (warp == kIdxProducerWarp) {
    // ------------------------------------------------------------ producer
    int k = 0;                                    // page slot (stage k % S)
    bool ok = true;
    auto slot = [&](int kk) -> bool {             // wait until stage kk % S is free
      return kk < S || mbar_wait(&raw_empty[kk % S], ((kk / S) - 1) & 1);
    };
    // Item `it` -> entity, query tile (rows [row0, row1)) and chunk; lane
    // j < np looks up the chunk's block j: logical block, page-table entry,
    // kind.  The page-table loads are issued here and consumed one item
    // later, while the previous item's pages are issued.
    struct Look { int np, ptrow, row0, row1, minpos, i, kind; long long p; };
    auto lookup = [&](int it) -> Look {
      Look r{};
      r.np = 0;
      if (it >= items) return r;
      int e = 0;
      {  // prefix[e] <= it < prefix[e+1]
        int l = 0, rr = nent;
        while (rr - l > 1) { const int m = (l + rr) >> 1; if (prefix[m] <= it) l = m; else rr = m; }
        e = l;
      }
      const Ent E = entity(a, e, tabs);
      const int local = it - prefix[e];
      const int tiles = (E.r1 - E.r0 + M - 1) / M;
      const int chunks = (E.hi - E.lo + kChunkPages - 1) / kChunkPages;
      // shared prefix: the tiles of one chunk are consecutive items, so the
      // CTAs working on them at the same time read the same pages (from L2
      // after the first); a sequence's own blocks: its chunks are consecutive
      const int y = a.shared ? local % tiles : local / chunks;
      const int c = a.shared ? local / tiles : local % chunks;
      const int i0 = E.lo + c * kChunkPages;
      r.np = min(E.hi - i0, kChunkPages);
      r.ptrow = E.ptrow;
      r.row0 = E.r0 + y * M;
      r.row1 = min(r.row0 + M, E.r1);
      // position of the tile's first and last query (a sequence's own rows;
      // shared prefix blocks are visible to every query of the group)
      const int L = lens[E.ptrow];
      r.minpos = a.shared ? 0x7FFFFFFF : L - a.T + ((r.row0 - E.r0) >> 2);
      const int maxpos = L - a.T + ((r.row1 - 1 - E.r0) >> 2);
      if (lane < r.np) {
        r.i = i0 + lane;                          // logical block
        r.p = a.page_table ? (long long)a.page_table[(long long)E.ptrow * a.max_pages + r.i]
                           : (long long)E.ptrow * a.max_pages + r.i;
        r.kind = (!a.shared && r.i * kBlock > maxpos) ? kPageMasked : kPageLoad;
      }
      return r;
    };
    // Items are claimed two ahead: the claim of item n+2 (an atomic whose
    // latency is a microsecond or more) is issued before item n's pages, and
    // its value is only read one item later.
    int item = 0, nxt = 0, claim = 0, ki = 0;      // ki: items of this CTA so far
    if (lane == 0) {
      item = atomicAdd(&a.work[0], 1);
      nxt = atomicAdd(&a.work[0], 1);
    }
    item = __shfl_sync(0xffffffffu, item, 0);
    Look cur = lookup(item);
    while (item < items && ok) {
      if (lane == 0) claim = atomicAdd(&a.work[0], 1);
      nxt = __shfl_sync(0xffffffffu, nxt, 0);
      const Look next = lookup(nxt);
      // page ids outside the pool: skipped and reported (kind Bad)
      if (lane < cur.np && cur.kind == kPageLoad && (cur.p < 0 || cur.p >= a.num_pages)) {
        report(a.flags, 4 /*MSA_ERR_DEVICE_BOUNDS*/, (int)cur.p);
        cur.kind = kPageBad;
      }
      // the item's query tile (E4M3 modes): one TMA load of its rows into
      // buffer ki % 2 once the MMAs of item ki-2 are done; rows past the
      // tile's end are read too (zero past the end of qi) and never used
      const int qx = ki & 1;
      if (!F16 && lane == 0) {
        if (ki >= 2 && !mbar_wait(&q_empty[qx], ((ki >> 1) - 1) & 1)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 8);
          ok = false;
        } else if (M == 64 && a.spread) {
          // boxes of 8 rows at MMA rows 16j.. (one 1 KB swizzle atom each)
          const int nbox = (cur.row1 - cur.row0 + 7) >> 3;
          mbar_expect_tx(&q_full[qx], nbox * 8 * 128);
          for (int j = 0; j < nbox; ++j)
            tma_load_2d(qbuf + qx * M * 128 + j * 16 * 128, &a.tmap_qi, 0, cur.row0 + 8 * j, &q_full[qx]);
        } else {
          mbar_expect_tx(&q_full[qx], M * 128);
          tma_load_2d(qbuf + qx * M * 128, &a.tmap_qi, 0, cur.row0, &q_full[qx]);
        }
      }
      ok = __shfl_sync(0xffffffffu, (int)ok, 0) != 0;
      // The item's pages, lane j: page j, stage (k + j) % S, issued in passes.
      // Stages are freed in page order (the decoders release them in order),
      // so the free stages of the pending pages are a prefix: each pass
      // issues that prefix at once, or waits for the first pending page's
      // stage when it is empty.  A lane only tests its stage once the page S
      // before it has been issued, so no barrier it reads is two phases behind.
      for (int jn = 0; jn < cur.np && ok;) {
        const int jend = min(cur.np, jn + S);
        const int kk = k + lane;                    // this lane's page slot
        const bool mine = lane >= jn && lane < jend;
        const bool fr = mine && (kk < S || mbar_test(&raw_empty[kk % S], ((kk / S) - 1) & 1));
        const unsigned pend = (jend >= 32 ? 0xffffffffu : (1u << jend) - 1u) & ~((1u << jn) - 1u);
        const unsigned busy = pend & ~__ballot_sync(0xffffffffu, fr);
        const int jx = busy ? __ffs(busy) - 1 : jend;   // pages [jn, jx) have free stages
        if (lane >= jn && lane < jx) {
          const int s = kk % S;
          int4* m4 = reinterpret_cast<int4*>(meta + 8 * s);
          m4[0] = make_int4(cur.ptrow, cur.i, cur.kind, cur.row0);
          m4[1] = make_int4(cur.row1, cur.minpos, ki, (lane == 0) | ((lane == cur.np - 1) << 1));
          uint8_t* dst = raw + s * C::kRawStride;
          if (cur.kind == kPageLoad) {
            mbar_expect_tx(&raw_full[s], C::kRaw);
            tma_load_2d(dst, &a.tmap_idx, 0, (int)(cur.p * kBlock), &raw_full[s]);
            if (!FP8) bulk_g2s(dst + kPageCodes, a.idx_scale + cur.p * kPageScales, kPageScales, &raw_full[s]);
          } else {
            mbar_arrive(&raw_full[s]);
          }
        }
        if (jx == jn) {   // no free stage: wait for page jn's (its slot is >= S)
          bool good = true;
          if (lane == jn) good = mbar_wait(&raw_empty[kk % S], ((kk / S) - 1) & 1);
          if (!__shfl_sync(0xffffffffu, (int)good, jn)) {
            if (lane == 0) report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1);
            ok = false;
          }
        }
        jn = jx;
      }
      k += cur.np;
      cur = next;
      item = nxt;
      nxt = claim;                                  // lane 0's value, broadcast next time
      ++ki;
    }
    if (lane == 0) {
      // two end markers, one for each of the epilogue's two page parities
      for (int e = 0; e < 2 && ok; ++e, ++k) {
        if (!slot(k)) {
          report(a.flags, 5 /*MSA_ERR_TIMEOUT*/, 1);
          ok = false;
        } else {
          meta[8 * (k % S) + 2] = kPageEnd;
          mbar_arrive(&raw_full[k % S]);
        }
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
      constexpr uint32_t idesc = idx_idesc<M>();
      int nend = 0;
      for (int k = 0;; ++k) {
        const int x = k & 1;                       // accumulator and page-ready barrier
        if (!mbar_wait(&b_full[k % BR], (k / BR) & 1)) { report(a.flags, 5, 2); break; }
        if (k >= 2 && !mbar_wait(&d_empty[x], ((k >> 1) - 1) & 1)) { report(a.flags, 5, 3); break; }
        tc_fence_after();
        const int* pf = pinfo + 8 * (k % kInfoRing);
        const int kind = pf[2], ki = pf[6], flg = pf[7];
        const int qx = F16 ? 0 : (ki & 1);
        if (!F16 && kind != kPageEnd && (flg & 1) && !mbar_wait(&q_full[qx], (ki >> 1) & 1)) {
          report(a.flags, 5, 9);
          break;
        }
        tc_fence_after();
        if (kind == kPageLoad) {
          const uint32_t d = tmem + (uint32_t)(x * kBlock);
          const uint32_t qa = smem_u32(qbuf + qx * M * 128);
          const uint32_t kb = FP8 ? smem_u32(raw + (k % S) * C::kRawStride)
                                  : smem_u32(bbuf + (k % BR) * C::kBBytes);
          if constexpr (F16) {
            // K-half h of the queries starts M rows further, of the keys 128 rows further
#pragma unroll
            for (int kk = 0; kk < 8; ++kk)
              tc_mma_ss_f16(d, desc_kmajor_sw128(qa + (kk >> 2) * M * 128) + 2 * (kk & 3),
                            desc_kmajor_sw128(kb + (kk >> 2) * kBlock * 128) + 2 * (kk & 3), idesc, kk > 0);
          } else {
            const uint64_t ad = desc_kmajor_sw128(qa), bd = desc_kmajor_sw128(kb);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) tc_mma_ss(d, ad + 2 * kk, bd + 2 * kk, idesc, kk > 0);
          }
        }
        tc_commit(&d_full[x]);
        if (kind == kPageEnd) {
          if (++nend == 2) break;
          continue;
        }
        if (FP8) tc_commit(&raw_empty[k % S]);   // the stage was the B operand
        tc_commit(&b_empty[k % BR]);              // page k consumed (and its B buffer free)
        if (!F16 && (flg & 2)) tc_commit(&q_empty[qx]);   // the item's query tile is free
      }
    }
  } else if (warp >= kIdxEpiWarp0) {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;                         // TMEM lane quarter
    const int par = (warp - kIdxEpiWarp0) >> 2;     // pages k with k % 2 == par (accumulator par)
    const uint32_t lane_base = tmem + ((uint32_t)(32 * q) << 16);
    // rows of the tile this warp reads: M = 64: 16q..16q+15 (spread: 8q..8q+7);
    // M = 128: 32q..32q+31
    const bool spread = M == 64 && a.spread;
    const int kRows = M == 64 ? (spread ? 8 : 16) : 32;
    for (int k = par;; k += 2) {
      const int x = par;
      if (!mbar_wait(&d_full[x], (k >> 1) & 1)) { report(a.flags, 5, 6); break; }
      tc_fence_after();
      const int* pf = pinfo + 8 * (k % kInfoRing);
      const int pi = pf[1], pkind = pf[2], prow0 = pf[3], prow1 = pf[4], pminpos = pf[5];
      if (pkind == kPageEnd) break;
      const int rbase = prow0 + kRows * q;           // first query row of this warp's lanes
      const bool active = rbase < prow1;             // warp-uniform
      // a key j is visible to query row r when j <= pos(r) = L_b - T + t
      const bool need_mask = pi * kBlock + kBlock - 1 > pminpos;
      auto last_key = [&](int r) -> int {    // rows past the last sequence hold no query
        if (r >= a.B * nq_all) return -1;
        const int b = r / nq_all;
        return lens[b] - a.T + (r - b * nq_all) / kG;
      };
      if (active && pkind == kPageLoad) {
        const uint32_t dcol = (uint32_t)(x * kBlock);
        if constexpr (M == 64) {
          // 16x256b: thread (g, t) holds rows g and g+8 of the quarter, columns
          // 8c+2t, 8c+2t+1 (spread: the rows g+8 hold no query)
          const int g = lane >> 2, t = lane & 3;
          float m0 = -INFINITY, m1 = -INFINITY;
          const int qa0 = rbase + g, qa1 = spread ? 0x7FFFFFFF : qa0 + 8;
          const int lim0 = need_mask ? last_key(qa0) : 0, lim1 = (need_mask && !spread) ? last_key(qa1) : 0;
#pragma unroll 1
          for (int h = 0; h < 2; ++h) {                // columns 64h .. 64h+63
            float v[32];
            tmem_ld_16x256b_x8(lane_base + dcol + 64 * h, v);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int i = 0; i < 32; ++i) {
                const int key = pi * kBlock + 64 * h + 8 * (i >> 2) + 2 * t + (i & 1);
                if (key > ((i & 2) ? lim1 : lim0)) v[i] = -INFINITY;
              }
            }
            if (a.token_scores != nullptr) {
#pragma unroll
              for (int i = 0; i < 32; i += 2) {
                const int qa = (i & 2) ? qa1 : qa0;
                if (qa < prow1) {
                  float* rowp = a.token_scores + (long long)qa * ctx;
                  const int col = pi * kBlock + 64 * h + 8 * (i >> 2) + 2 * t;
                  rowp[col] = v[i] * a.score_scale;
                  rowp[col + 1] = v[i + 1] * a.score_scale;
                }
              }
            }
            float r0[16], r1[16];
#pragma unroll
            for (int c = 0; c < 8; ++c) {
              r0[2 * c] = v[4 * c]; r0[2 * c + 1] = v[4 * c + 1];
              r1[2 * c] = v[4 * c + 2]; r1[2 * c + 1] = v[4 * c + 3];
            }
            m0 = fmaxf(m0, max_of<16>(r0));
            if (!spread) m1 = fmaxf(m1, max_of<16>(r1));
          }
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 1));
          m0 = fmaxf(m0, __shfl_xor_sync(0xffffffffu, m0, 2));
          if (!spread) {
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 1));
            m1 = fmaxf(m1, __shfl_xor_sync(0xffffffffu, m1, 2));
          }
          if (t < 2) {
            const int qa = t == 0 ? qa0 : qa1;
            if (qa < prow1) a.block_scores[(long long)qa * a.max_pages + pi] = (t == 0 ? m0 : m1) * a.score_scale;
          }
        } else {
          // 32x32b: thread = query row rbase + lane, all 128 columns
          const int qa = rbase + lane;
          const int lim = (need_mask && qa < prow1) ? last_key(qa) : 0;
          float m = -INFINITY;
#pragma unroll 1
          for (int h = 0; h < 4; ++h) {
            float v[32];
            tmem_ld_32x32b_x32(lane_base + dcol + 32 * h, v);
            tmem_wait_ld();
            if (need_mask) {
#pragma unroll
              for (int i = 0; i < 32; ++i)
                if (pi * kBlock + 32 * h + i > lim) v[i] = -INFINITY;
            }
            if (a.token_scores != nullptr && qa < prow1) {
              float* rowp = a.token_scores + (long long)qa * ctx + pi * kBlock + 32 * h;
#pragma unroll
              for (int i = 0; i < 32; ++i) rowp[i] = v[i] * a.score_scale;
            }
            m = fmaxf(m, max_of<32>(v));
          }
          if (qa < prow1) a.block_scores[(long long)qa * a.max_pages + pi] = m * a.score_scale;
        }
      } else if (active && pkind == kPageMasked) {
        // no key of the block is visible to any query of the tile
        for (int r = lane; r < kRows; r += 32) {
          const int qa = rbase + r;
          if (qa >= prow1) continue;
          a.block_scores[(long long)qa * a.max_pages + pi] = -INFINITY;
          if (a.token_scores != nullptr)
            for (int j = 0; j < kBlock; ++j) a.token_scores[(long long)qa * ctx + pi * kBlock + j] = -INFINITY;
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(&d_empty[x]);
    }
  } else {
    // ------------------------------------------------------------ decoders
    const int d = 32 * warp + lane;                 // 0 .. 127
    const int row = d;                              // key row of this thread
    const int sw = (row >> 1) & 3;                  // 64-byte swizzle of the code rows
    int nend = 0;
    int cur_row0 = -1;
    int s = 0;                                      // stage of page k
    uint32_t sph = 0;                               // its phase parity
    for (int k = 0;; ++k) {
      if (!mbar_wait(&raw_full[s], sph)) { report(a.flags, 5, 5); break; }
      // page k-BR consumed by the MMA: its B buffer and page-ready barrier
      // (k % BR) are free, and every MMA of pages <= k-BR has completed
      if (k >= BR && !mbar_wait(&b_empty[k % BR], ((k / BR) - 1) & 1)) {
        report(a.flags, 5, 4);
        break;
      }
      const int* m = meta + 8 * s;
      const int nkind = m[2];
      if (F16 && nkind != kPageEnd && m[3] != cur_row0) {
        const int nr0 = m[3], nr1 = m[4];
        // FP16 A operand: the index-query rows [nr0, nr1) of the tile widened
        // to FP16, K-major, two 128-byte-swizzled K-halves, zero rows past
        // nr1.  The previous tile's last MMA (page k-1 at the latest) must be
        // done.  (E4M3 tiles are loaded by the producer's TMA.)
        if (k >= 1 && !mbar_wait(&b_empty[(k - 1) % BR], ((k - 1) / BR) & 1)) {
          report(a.flags, 5, 7);
          break;
        }
        cur_row0 = nr0;
        for (int idx = d; idx < M * 8; idx += kIdxDecWarps * 32) {
          const int nrow = idx >> 3, c = idx & 7;
          const int qg = nr0 + nrow;
          uint4 v = make_uint4(0u, 0u, 0u, 0u);
          if (qg < nr1) v = *reinterpret_cast<const uint4*>(a.qi + (long long)qg * kDim + 16 * c);
          // dims 16c..16c+15 -> FP16 chunks 2c, 2c+1 of 8 dims: K-half c / 4,
          // chunk positions (2c % 8, 2c % 8 + 1) ^ (row % 8) in its 128-byte row
          const uint4 lo = make_uint4(e4m3x2_to_f16x2(v.x), e4m3x2_to_f16x2(v.x >> 16),
                                      e4m3x2_to_f16x2(v.y), e4m3x2_to_f16x2(v.y >> 16));
          const uint4 hi = make_uint4(e4m3x2_to_f16x2(v.z), e4m3x2_to_f16x2(v.z >> 16),
                                      e4m3x2_to_f16x2(v.w), e4m3x2_to_f16x2(v.w >> 16));
          uint8_t* rowp = qbuf + (c >> 2) * M * 128 + nrow * 128;
          const int jj = (2 * c) & 7;
          sts128(rowp + ((jj ^ (nrow & 7)) << 4), lo);
          sts128(rowp + (((jj + 1) ^ (nrow & 7)) << 4), hi);
        }
      }
      if (!FP8 && nkind == kPageLoad) {
        const uint8_t* rs = raw + s * C::kRawStride;
        uint8_t* bb = bbuf + (k % BR) * C::kBBytes;
        // 64-byte code rows loaded with the 64-byte swizzle: chunk c of row r
        // sits at chunk position c ^ ((r / 2) % 4); chunk c = elements
        // 32c..32c+31 under scale bytes 2c and 2c+1.  This thread: the whole
        // row, as two halves (chunks 2h, 2h+1 under scale bytes 4h..4h+3).
        const uint2 sc8 = *reinterpret_cast<const uint2*>(rs + kPageCodes + row * kRowScales);
#pragma unroll
        for (int half = 0; half < 2; ++half) {
          const uint32_t sc4 = half ? sc8.y : sc8.x;
          if constexpr (F16) {
            // FP16 key row: 256 bytes as two 128-byte K-halves (rows 128 apart),
            // each with the 128-byte swizzle; chunk c -> 16-byte chunks 4(c%2)..
            // of K-half c / 2 (= half)
            uint8_t* rowp = bb + half * kBlock * 128 + row * 128;
  #pragma unroll
            for (int cc = 0; cc < 2; ++cc) {
              const int c = 2 * half + cc;
              const uint4 w4 = lds128(rs + row * kRowCodes + ((c ^ sw) << 4));
              const uint32_t s2 = e4m3x2_to_f16x2(sc4 >> (16 * cc));
              const uint32_t s_lo = prmt(s2, 0u, 0x1010u), s_hi = prmt(s2, 0u, 0x3232u);
              uint32_t o[16];
              e2m1x8_to_f16x2(w4.x, o + 0);
              e2m1x8_to_f16x2(w4.y, o + 4);
              e2m1x8_to_f16x2(w4.z, o + 8);
              e2m1x8_to_f16x2(w4.w, o + 12);
  #pragma unroll
              for (int mm = 0; mm < 16; ++mm) o[mm] = hmul2(o[mm], mm < 8 ? s_lo : s_hi);
  #pragma unroll
              for (int jj = 0; jj < 4; ++jj) {
                const int ch = 4 * cc + jj;
                sts128(rowp + ((ch ^ (row & 7)) << 4),
                       make_uint4(o[4 * jj], o[4 * jj + 1], o[4 * jj + 2], o[4 * jj + 3]));
              }
            }
          } else {
            // E4M3 key row: 128 bytes with the 128-byte swizzle; code chunk c ->
            // row chunks 2c, 2c+1
            uint8_t* rowp = bb + row * 128;
            const uint4 w0 = lds128(rs + row * kRowCodes + (((2 * half) ^ sw) << 4));
            const uint4 w1 = lds128(rs + row * kRowCodes + (((2 * half + 1) ^ sw) << 4));
            const uint2 r0 = lut[sc4 & 0xFFu], r1 = lut[(sc4 >> 8) & 0xFFu];
            const uint2 r2 = lut[(sc4 >> 16) & 0xFFu], r3 = lut[sc4 >> 24];
            uint32_t o[16];
            dq8(w0.x, r0, o[0], o[1]);
            dq8(w0.y, r0, o[2], o[3]);
            dq8(w0.z, r1, o[4], o[5]);
            dq8(w0.w, r1, o[6], o[7]);
            dq8(w1.x, r2, o[8], o[9]);
            dq8(w1.y, r2, o[10], o[11]);
            dq8(w1.z, r3, o[12], o[13]);
            dq8(w1.w, r3, o[14], o[15]);
            const int c0 = 4 * half;                   // first of this thread's 4 row chunks
  #pragma unroll
            for (int jj = 0; jj < 4; ++jj)
              sts128(rowp + (((c0 + jj) ^ (row & 7)) << 4),
                     make_uint4(o[4 * jj], o[4 * jj + 1], o[4 * jj + 2], o[4 * jj + 3]));
          }
        }
      }
      fence_async_smem();   // generic-proxy writes (queries, keys) -> the MMA
      __syncwarp();
      if (lane == 0) {
        if (warp == 0) {   // the page's info, for the MMA and the epilogue
          const int4* src = reinterpret_cast<const int4*>(m);
          int4* dst = reinterpret_cast<int4*>(pinfo + 8 * (k % kInfoRing));
          dst[0] = src[0];
          dst[1] = src[1];
        }
        if (!FP8) mbar_arrive(&raw_empty[s]);
        mbar_arrive(&b_full[k % BR]);
      }
      if (nkind == kPageEnd && ++nend == 2) break;
      if (++s == S) { s = 0; sph ^= 1u; }
    }
  }

  // ---- teardown: every role leaves its loop (normally or on a timeout)
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == kIdxMmaWarp) tmem_dealloc(tmem, kIdxTmemCols);
}

template <int MODE, int M>
static cudaError_t launch_mode(const IdxArgs& a, cudaStream_t st) {
  auto kern = indexer_kernel<MODE, M>;
  const size_t smem = (size_t)idx_layout<MODE, M>(a.B).total;
  int grid = 0;                                 // persistent: items are claimed in the kernel
  cudaError_t e = persistent_grid(reinterpret_cast<const void*>(kern), kIdxThreads, smem,
                                  kIdxTmemCols, &grid);
  if (e != cudaSuccess) return e;
  kern<<<grid, kIdxThreads, smem, st>>>(a);
  return cudaGetLastError();
}

cudaError_t launch_indexer(const IdxArgs& a, int mode, cudaStream_t st) {
  // shared-prefix tiles span the query rows of several sequences: 128 rows
  const bool m64 = !a.shared && idx_tile_queries(a.T) == 64;
  if (mode == kIdxFp8) return m64 ? launch_mode<kIdxFp8, 64>(a, st) : launch_mode<kIdxFp8, 128>(a, st);
  if (mode == kIdxF16) return m64 ? launch_mode<kIdxF16, 64>(a, st) : launch_mode<kIdxF16, 128>(a, st);
  return m64 ? launch_mode<kIdxNvfp4, 64>(a, st) : launch_mode<kIdxNvfp4, 128>(a, st);
}

}  // namespace msa
