// msa_device.cuh -- device helpers shared by the MSA kernels (sm_100a).
//
// NVFP4 -> E4M3 decode.  [post, "NVIDIA Blackwell optimized MSA kernels"]
// (post = vLLM 為 MiniMax-M3.1-Flash 提供 Day-0 支援, hot.atechcom.net) feeds
// an FP8 MMA, so each E2M1 code times its E4M3 block scale is rounded back to
// E4M3.  The toolkit here (CUDA 12.9) has no e2m1 x e4m3 scale-multiply
// instruction, so the rounding is tabulated: for each of the 256 scale bytes
// the 8 E2M1 magnitudes times the scale, rounded by the CUDA fp8 conversion
// (round-to-nearest-even, satfinite), make one 8-byte row of a 2 KB shared
// table (the table-lookup idea of [post, "AMD GPU support", "NVFP4 MSA
// kernel"], rebuilt for PTX `prmt`).  Four codes then decode with one byte
// permute for the magnitudes and one for the signs.
#pragma once

#include <cstdint>
#include <cuda_fp8.h>
#include <cuda_runtime.h>

namespace msa {

constexpr int kBlock = 128;      // tokens per block / page
constexpr int kDim = 128;        // head dim
constexpr int kG = 4;            // KV heads = GQA groups
constexpr int kHpg = 16;         // query heads per group
constexpr int kHq = kG * kHpg;   // query heads
constexpr int kTopk = 16;        // selected blocks
constexpr int kRowCodes = 64;    // bytes of NVFP4 codes per 128-vector
constexpr int kRowScales = 8;    // E4M3 scale bytes per 128-vector
constexpr int kPageCodes = kBlock * kRowCodes;    // 8192
constexpr int kPageScales = kBlock * kRowScales;  // 1024

// Workspace header (first 256 bytes of the workspace, zeroed by
// msa_workspace_init): the device error flags at offset 0, the indexer's
// work-distribution counters at kWorkOffset.
struct Flags {
  int code;     // first msa_status recorded on the device (0 = none)
  int detail;   // the offending value
};
constexpr int kWorkOffset = 64;   // int[2]: next work item, CTAs finished (0 between calls)

// Programmatic dependent launch: wait until the grids this one depends on
// have completed and their writes are visible (returns at once when the
// kernel was launched without programmatic serialisation), and let the next
// kernel on the stream start launching once every CTA of this one has called
// it or exited.
__device__ __forceinline__ void grid_dependency_wait() {
  asm volatile("griddepcontrol.wait;\n" ::: "memory");
}
__device__ __forceinline__ void grid_launch_dependents() {
  asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory");
}

__device__ __forceinline__ void report(Flags* f, int code, int detail) {
  if (atomicCAS(&f->code, 0, code) == 0) atomicExch(&f->detail, detail);
}

// ----------------------------------------------------------- NVFP4 table --
// lut[s] = {E4M3(m*e4m3(s)) for m = 0..3 in .x, m = 4..7 in .y}, m indexing
// the E2M1 magnitudes {0, 0.5, 1, 1.5, 2, 3, 4, 6} (OCP MX v1.0).
__device__ __forceinline__ void build_nvfp4_lut(uint2* lut, int tid, int nthreads) {
  for (int i = tid; i < 512; i += nthreads) {
    const int s = i >> 1, half = i & 1;
    __nv_fp8_e4m3 sc;
    sc.__x = (__nv_fp8_storage_t)s;
    const float scale = float(sc);
    uint32_t word = 0;
#pragma unroll
    for (int k = 0; k < 4; ++k) {
      // the product of a 2-bit and a 4-bit significand is exact in fp32
      const int m = 4 * half + k;                       // E2M1 magnitude code
      const float mag = (m < 2) ? 0.5f * (float)m
                                : (1.0f + 0.5f * (float)(m & 1)) * (float)(1 << ((m >> 1) - 1));
      const float prod = mag * scale;
      const uint32_t b = __nv_cvt_float_to_fp8(prod, __NV_SATFINITE, __NV_E4M3);
      word |= (b & 0xFFu) << (8 * k);
    }
    if (half) lut[s].y = word; else lut[s].x = word;
  }
}

// -------------------------------------------- mbarrier + bulk async copy --
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

__device__ __forceinline__ void mbar_fence_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

// One bulk copy global -> shared (16-byte aligned, size a multiple of 16).
__device__ __forceinline__ void bulk_g2s(void* dst, const void* src, uint32_t bytes,
                                         uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Bounded wait on an mbarrier phase.  Each try_wait suspends the thread until
// the phase completes or the suspend-time hint (about 0.5 ms) runs out, so a
// waiting warp does not spin; after kSpinLimit attempts (a few seconds at
// most) the wait gives up and returns false.
constexpr uint32_t kSpinLimit = 1u << 13;
constexpr uint32_t kSuspendHintNs = 500000;

__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t it = 0; it < kSpinLimit; ++it) {
    uint32_t ok;
    asm volatile(
        "{\n.reg .pred P;\nmbarrier.try_wait.parity.shared::cta.b64 P, [%1], %2, %3;\n"
        "selp.b32 %0, 1, 0, P;\n}\n"
        : "=r"(ok)
        : "r"(a), "r"(parity), "r"(kSuspendHintNs)
        : "memory");
    if (ok) return true;
  }
  return false;
}

// Non-blocking test of an mbarrier phase (for a thread that polls several).
__device__ __forceinline__ bool mbar_test(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n.reg .pred P;\nmbarrier.test_wait.parity.shared::cta.b64 P, [%1], %2;\n"
      "selp.b32 %0, 1, 0, P;\n}\n"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}
// Polls without progress after which a polling thread gives up (with a
// 64 ns sleep per poll: a few seconds).
constexpr uint32_t kPollLimit = 1u << 26;

__device__ __forceinline__ uint4 lds128(const void* p) { return *reinterpret_cast<const uint4*>(p); }

// Order-preserving map float -> uint32 (larger float -> larger key).
__device__ __forceinline__ uint32_t float_key(float f) {
  const uint32_t u = __float_as_uint(f);
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

}  // namespace msa

// ------------------------------------------------------------- tcgen05 ----
// 5th-generation tensor core: MMAs issued by one thread, operands in shared
// memory described by 64-bit descriptors, fp32 accumulators in tensor memory.
namespace msa {

__device__ __forceinline__ void fence_async_smem() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}
// Warp-wide: allocate ncols (power of 2, >= 32) TMEM columns; address -> *dst.
__device__ __forceinline__ void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(smem_u32(dst)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// Shared-memory descriptor of a K-major operand tile stored with the 128-byte
// swizzle: rows of 128 bytes, 8-row atoms 1024 bytes apart, the 16-byte chunk
// c of row r at chunk position c ^ (r % 8); tile base 1024-byte aligned.
__device__ __forceinline__ uint64_t desc_kmajor_sw128(uint32_t smem_addr) {
  return (uint64_t)((smem_addr & 0x3FFFFu) >> 4)   // start address
         | ((uint64_t)1 << 16)                      // leading offset (unused with swizzle)
         | ((uint64_t)(1024 >> 4) << 32)            // stride between 8-row atoms
         | ((uint64_t)1 << 46)                      // descriptor version
         | ((uint64_t)2 << 61);                     // 128-byte swizzle
}

// Instruction descriptor: kind::f8f6f4, A = B = E4M3, fp32 accumulate,
// both operands K-major, shape M x N.
__host__ __device__ constexpr uint32_t idesc_e4m3_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// Arrive on *bar once every tcgen05 operation issued so far by this thread completes.
__device__ __forceinline__ void tc_commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
                   smem_u32(bar))
               : "memory");
}

__device__ __forceinline__ void tmem_wait_ld() {
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float (&v)[8]) {
  uint32_t r[8];
  asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                 "=r"(r[6]), "=r"(r[7])
               : "r"(taddr)
               : "memory");
#pragma unroll
  for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// Max of a float over the 32 lanes of the warp (result in every lane).
__device__ __forceinline__ float warp_max(float v) {
  float r;
  asm volatile("redux.sync.max.f32 %0, %1, 0xffffffff;\n" : "=f"(r) : "f"(v));
  return r;
}

}  // namespace msa

namespace msa {

// D[tmem] (+)= A[tmem] * B[smem]^T, one K = 32 slice (E4M3).  A: 128 TMEM
// lanes = rows, 8 consecutive 32-bit columns = 32 K-bytes of each row.
__device__ __forceinline__ void tc_mma_e4m3_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-wide: lane l writes 8 consecutive 32-bit columns of TMEM lane (taddr.lane + l).
__device__ __forceinline__ void tmem_st8(uint32_t taddr, const uint32_t (&r)[8]) {
  asm volatile("tcgen05.st.sync.aligned.32x32b.x8.b32 [%0], {%1,%2,%3,%4,%5,%6,%7,%8};\n" ::"r"(taddr),
               "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]),
               "r"(r[7])
               : "memory");
}

__device__ __forceinline__ void tmem_wait_st() {
  asm volatile("tcgen05.wait::st.sync.aligned;\n" ::: "memory");
}

// Tiled TMA load of a 2-D box at element coordinates (x, y) into shared memory.
__device__ __forceinline__ void tma_load_2d(void* dst, const void* tmap, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];\n" ::
          "r"(smem_u32(dst)),
      "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_u32(bar))
      : "memory");
}

// PTX prmt in its default mode (the top bit of each selector nibble
// replicates the sign of the selected byte, unlike __byte_perm).
__device__ __forceinline__ uint32_t prmt(uint32_t a, uint32_t b, uint32_t sel) {
  uint32_t d;
  asm("prmt.b32 %0, %1, %2, %3;\n" : "=r"(d) : "r"(a), "r"(b), "r"(sel));
  return d;
}

// x >> 16 as a multiply-high, which issues on the FMA pipe and leaves the
// integer ALU pipe (which also runs prmt and the logic ops) to the decode.
__device__ __forceinline__ uint32_t hi16(uint32_t x) {
  uint32_t d;
  asm("mul.hi.u32 %0, %1, 65536;\n" : "=r"(d) : "r"(x));
  return d;
}

// dq8_split for a non-negative block scale (the usual case).
__device__ __forceinline__ void dq8_split_pos(uint32_t w, uint2 r, uint32_t& p0, uint32_t& p1,
                                              uint32_t& n0, uint32_t& n1) {
  const uint32_t wn = w ^ 0x88888888u;
  p0 = prmt(r.x, r.y, w);
  p1 = prmt(r.x, r.y, hi16(w));
  n0 = prmt(r.x, r.y, wn);
  n1 = prmt(r.x, r.y, hi16(wn));
}

// max of three floats in one instruction (sm_100).
__device__ __forceinline__ float fmax3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;\n" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// NVFP4 -> E4M3 split by sign for 8 codes (element n in nibble n):
// pos = E4M3(|value|) of the positive elements (0 elsewhere), neg likewise for
// the negative ones, so value = pos - neg.  `r` is the table row of |scale|
// (all bytes < 0x80); a selector nibble with its top bit set makes prmt
// return 0x00 (the sign of a non-negative byte), which drops the elements of
// the other sign.  flip = 0x88888888 when the block scale is negative.
__device__ __forceinline__ void dq8_split(uint32_t w, uint2 r, uint32_t flip, uint32_t& p0,
                                          uint32_t& p1, uint32_t& n0, uint32_t& n1) {
  const uint32_t wp = w ^ flip;
  const uint32_t wn = wp ^ 0x88888888u;
  p0 = prmt(r.x, r.y, wp);
  p1 = prmt(r.x, r.y, wp >> 16);
  n0 = prmt(r.x, r.y, wn);
  n1 = prmt(r.x, r.y, wn >> 16);
}

}  // namespace msa

namespace msa {

// Two E4M3 values (low 16 bits of w, low byte first) -> f16x2 (exact).
__device__ __forceinline__ uint32_t e4m3x2_to_f16x2(uint32_t w) {
  uint32_t d;
  asm("cvt.rn.f16x2.e4m3x2 %0, %1;\n" : "=r"(d) : "h"((uint16_t)(w & 0xFFFFu)));
  return d;
}

// ----------------------------------------------- NVFP4 -> FP16 (exact) ----
// e2m1 x e4m3 has at most 5 significant bits and lies in [2^-10, 2688], so
// it is exact in FP16: no re-rounding ([post, "NVIDIA Rubin optimized MSA"]
// scores the index keys this way).

// Two E2M1 codes (the low byte of b, element 0 in the low nibble) -> f16x2
// (element 0 in the low half), unscaled.
__device__ __forceinline__ uint32_t e2m1x2_to_f16x2(uint32_t b) {
  uint32_t d;
  asm("{\n.reg .b8 c, z;\nmov.b16 {c, z}, %1;\ncvt.rn.f16x2.e2m1x2 %0, c;\n}\n"
      : "=r"(d)
      : "h"((uint16_t)(b & 0xFFFFu)));
  return d;
}

// The 8 codes of w (element n in nibble n) -> 4 f16x2 words o[0..3], o[m] =
// elements 2m (low half) and 2m+1, unscaled.
// Each byte is first moved to the bottom of a register of its own (prmt):
// unpacking the four bytes of one register through nested vector moves
// (32 -> 2 x 16 -> 4 x 8 bits) gave byte 0 in place of byte 2 on sm_100a.
__device__ __forceinline__ void e2m1x8_to_f16x2(uint32_t w, uint32_t* o) {
  o[0] = e2m1x2_to_f16x2(prmt(w, 0u, 0x4440u));
  o[1] = e2m1x2_to_f16x2(prmt(w, 0u, 0x4441u));
  o[2] = e2m1x2_to_f16x2(prmt(w, 0u, 0x4442u));
  o[3] = e2m1x2_to_f16x2(prmt(w, 0u, 0x4443u));
}

__device__ __forceinline__ uint32_t hmul2(uint32_t a, uint32_t b) {
  uint32_t d;
  asm("mul.rn.f16x2 %0, %1, %2;\n" : "=r"(d) : "r"(a), "r"(b));
  return d;
}

// Warp-wide: lane l writes 16 consecutive 32-bit columns of TMEM lane (taddr.lane + l).
__device__ __forceinline__ void tmem_st16(uint32_t taddr, const uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.st.sync.aligned.32x32b.x16.b32 [%0], "
      "{%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,%16};\n" ::"r"(taddr),
      "r"(r[0]), "r"(r[1]), "r"(r[2]), "r"(r[3]), "r"(r[4]), "r"(r[5]), "r"(r[6]), "r"(r[7]),
      "r"(r[8]), "r"(r[9]), "r"(r[10]), "r"(r[11]), "r"(r[12]), "r"(r[13]), "r"(r[14]),
      "r"(r[15])
      : "memory");
}

// Instruction descriptor: kind::f16, A = B = f16 (format code 0), fp32
// accumulate, both operands K-major, shape M x N.  The fields sit where they
// do for kind::f8f6f4, where format code 0 names E4M3.
__host__ __device__ constexpr uint32_t idesc_f16_f32(int M, int N) {
  return (1u << 4) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[tmem] * B[smem]^T, one K = 16 slice of FP16.  A: 8
// consecutive 32-bit TMEM columns = 16 K-elements of each row.
__device__ __forceinline__ void tc_mma_f16_ts(uint32_t d_tmem, uint32_t a_tmem, uint64_t bdesc,
                                              uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], [%1], %2, %3, p;\n}\n" ::"r"(d_tmem),
      "r"(a_tmem), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Warp-wide 16x256b TMEM load, R = 1, 2 or 4 repetitions along columns:
// thread (g = lane/4, t = lane%4) receives, for column group c < R,
//   v[4c+0] = (lane g,   col 8c+2t), v[4c+1] = (lane g,   col 8c+2t+1),
//   v[4c+2] = (lane g+8, col 8c+2t), v[4c+3] = (lane g+8, col 8c+2t+1),
// lanes relative to taddr's lane (which must be a multiple of 16 within the
// warp's 32-lane quarter).
template <int R>
__device__ __forceinline__ void tmem_ld_16x256b(uint32_t taddr, float (&v)[4 * R]) {
  uint32_t r[4 * R];
  if constexpr (R == 1) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x1.b32 {%0,%1,%2,%3}, [%4];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr)
                 : "memory");
  } else if constexpr (R == 2) {
    asm volatile("tcgen05.ld.sync.aligned.16x256b.x2.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];\n"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]),
                   "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr)
                 : "memory");
  } else {
    static_assert(R == 4, "16x256b repetitions");
    asm volatile(
        "tcgen05.ld.sync.aligned.16x256b.x4.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
          "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
          "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr)
        : "memory");
  }
#pragma unroll
  for (int i = 0; i < 4 * R; ++i) v[i] = __uint_as_float(r[i]);
}

}  // namespace msa

namespace msa {

// D[tmem] (+)= A[smem] * B[smem]^T (E4M3, kind::f8f6f4), one K = 32 slice.
__device__ __forceinline__ void tc_mma_ss(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                          uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate)
      : "memory");
}

// D[tmem] (+)= A[smem] * B[smem]^T (FP16, kind::f16), one K = 16 slice.
__device__ __forceinline__ void tc_mma_ss_f16(uint32_t d, uint64_t ad, uint64_t bd, uint32_t idesc,
                                              uint32_t accumulate) {
  asm volatile(
      "{\n.reg .pred p;\nsetp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n}\n" ::"r"(d),
      "l"(ad), "l"(bd), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Signed NVFP4 -> E4M3 decode of 8 codes w (element n in nibble n) with the
// table row r = lut[scale byte] (E4M3 of the 8 E2M1 magnitudes times the
// scale, sign of the scale included): o0 = elements 0..3, o1 = 4..7, low
// byte first.  The magnitudes come from one prmt per four codes.  The code
// signs sit in bit 3 of each nibble: those of the odd elements are already
// bit 7 of the bytes of w, those of the even elements bit 7 of the bytes of
// w << 4, and one byte permute per four codes interleaves them into bit 7 of
// the output bytes, where an xor applies them.  Nine operations per 8 codes.
__device__ __forceinline__ void dq8(uint32_t w, uint2 r, uint32_t& o0, uint32_t& o1) {
  const uint32_t mag = w & 0x77777777u;
  const uint32_t u = w << 4;
  const uint32_t s0 = prmt(u, w, 0x5140u);    // bytes: signs of elements 0, 1, 2, 3
  const uint32_t s1 = prmt(u, w, 0x7362u);    // elements 4, 5, 6, 7
  o0 = prmt(r.x, r.y, mag) ^ (s0 & 0x80808080u);
  o1 = prmt(r.x, r.y, mag >> 16) ^ (s1 & 0x80808080u);
}

// Warp-wide 16x256b TMEM load, 8 repetitions (64 columns): thread (g =
// lane/4, t = lane%4) receives for c < 8: v[4c+0] = (lane g, col 8c+2t),
// v[4c+1] = (lane g, col 8c+2t+1), v[4c+2] = (lane g+8, col 8c+2t),
// v[4c+3] = (lane g+8, col 8c+2t+1), lanes relative to taddr's lane.
__device__ __forceinline__ void tmem_ld_16x256b_x8(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.16x256b.x8.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Warp-wide 32x32b TMEM load of 32 consecutive columns: lane l receives
// columns c..c+31 of TMEM lane (taddr.lane + l).
__device__ __forceinline__ void tmem_ld_32x32b_x32(uint32_t taddr, float (&v)[32]) {
  uint32_t r[32];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]),
        "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]),
        "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 0; i < 32; ++i) v[i] = __uint_as_float(r[i]);
}

// Max of n floats (n a multiple of 2) with three-input max instructions.
template <int N>
__device__ __forceinline__ float max_of(const float* v) {
  float m = fmaxf(v[0], v[1]);
#pragma unroll
  for (int i = 2; i + 1 < N; i += 2) m = fmax3(m, v[i], v[i + 1]);
  return m;
}

}  // namespace msa
