// common.cuh -- device primitives for the sm_100a MoE kernels: status bits, bf16 packing,
// mbarrier waits with a time limit, TMA tile loads, and tcgen05 (UMMA / TMEM) wrappers.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <stdint.h>

namespace moe {

// ---------------------------------------------------------------- device status word bits
enum : uint32_t {
  DEV_ERR_TIMEOUT = 1u << 0,   // an mbarrier wait exceeded its time limit
  DEV_ERR_EXPERT = 1u << 1,    // an expert index outside [0, n)
  DEV_ERR_ROW = 1u << 2,       // a permuted row outside the workspace
};

// Roughly 2 s at the B200's 1.0-2.0 GHz SM clock.
constexpr long long WAIT_LIMIT_CYCLES = 4000000000LL;

__device__ __forceinline__ void set_status(uint32_t* status, uint32_t bits) {
  if (status) atomicOr(status, bits);
}

// ---------------------------------------------------------------- programmatic dependent launch
// Every kernel is launched so that it may start while the previous kernel of the stream is
// still finishing.  pdl_wait() blocks until that kernel has completed and its writes are
// visible, so it comes before any access to data it produced (and before any write another
// kernel of the previous call may still read); pdl_trigger() lets the next kernel launch.
__device__ __forceinline__ void pdl_wait() { asm volatile("griddepcontrol.wait;" ::: "memory"); }
__device__ __forceinline__ void pdl_trigger() {
  asm volatile("griddepcontrol.launch_dependents;" ::: "memory");
}

// ---------------------------------------------------------------- small helpers
__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&v);
}

__device__ __forceinline__ float bf16_lo(uint32_t v) { return __uint_as_float(v << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t v) { return __uint_as_float(v & 0xffff0000u); }

__device__ __forceinline__ float silu(float z) { return z / (1.0f + expf(-z)); }

// silu for the GEMM epilogues, where h is rounded to bf16 right after: fast exponential and
// division (a few fp32 ulps, far below bf16's half-ulp).  Large negative z gives exp = inf and
// a quotient of 0, the limit of silu.
__device__ __forceinline__ float silu_epilogue(float z) {
  return __fdividef(z, 1.0f + __expf(-z));
}

// ---------------------------------------------------------------- mbarrier
__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;" ::"r"(smem_u32(bar)), "r"(count));
}

__device__ __forceinline__ void fence_mbar_init() {
  asm volatile("fence.mbarrier_init.release.cluster;" ::: "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ void mbar_arrive_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.shared::cta.b64 _, [%0], %1;" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t ok;
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(ok)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return ok != 0;
}

// Wait until the barrier's phase with the given parity has completed.  Gives up after
// `limit` cycles (WAIT_LIMIT_CYCLES unless a caller passes a shorter one), or at once if
// *abort is set while waiting, records DEV_ERR_TIMEOUT and returns false; the caller then
// unwinds without issuing further work.
__device__ __forceinline__ bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t* status,
                                          volatile int* abort,
                                          long long limit = WAIT_LIMIT_CYCLES) {
  if (mbar_try_wait(bar, parity)) return true;
  const long long t0 = clock64();
  for (uint32_t it = 1;; ++it) {
    if (mbar_try_wait(bar, parity)) return true;
    if ((it & 255u) == 0u) {
      if (*abort) return false;
      if (clock64() - t0 > limit) {
        set_status(status, DEV_ERR_TIMEOUT);
        *abort = 1;
        return false;
      }
    }
  }
}

// Wait (at most WAIT_LIMIT_CYCLES / 16) for a phase on the unwind path of a kernel that
// already gave up, e.g. for its own copies in flight to land before it exits.
__device__ __forceinline__ bool wait_short(uint64_t* bar, uint32_t parity) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > (WAIT_LIMIT_CYCLES >> 4)) return false;
  return true;
}

// ---------------------------------------------------------------- TMA (no multicast)
__device__ __forceinline__ void tma_prefetch_desc(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

// 2-D tile load global -> shared, completion signalled on `bar` as transaction bytes.
// x (innermost, elements) must be a multiple of 16 bytes / element size.
__device__ __forceinline__ void tma_load_2d(void* smem_dst, const CUtensorMap* map,
                                            uint64_t* bar, int32_t x, int32_t y,
                                            uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)), "r"(x), "r"(y),
      "l"(cache_hint)
      : "memory");
}

// L2 cache policies for TMA loads (createpolicy fractional, fraction 1.0).
__device__ __forceinline__ uint64_t policy_evict_first() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_first.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_last() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_last.b64 %0, 1.0;" : "=l"(p));
  return p;
}
__device__ __forceinline__ uint64_t policy_evict_normal() {
  uint64_t p;
  asm volatile("createpolicy.fractional.L2::evict_normal.b64 %0, 1.0;" : "=l"(p));
  return p;
}

// ---------------------------------------------------------------- tcgen05 / TMEM
__device__ __forceinline__ void tmem_alloc(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tc_fence_after() {
  asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory");
}
__device__ __forceinline__ void tc_fence_before() {
  asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory");
}

// Shared-memory matrix descriptor for a K-major operand tile written by TMA with 128-byte
// swizzling: rows of 128 bytes (64 bf16), 8-row groups 1024 bytes apart.  Fields: start
// address >> 4 (bits 0-13), leading byte offset >> 4 (16-29, unused for this layout, 1),
// stride byte offset >> 4 (32-45), descriptor version 1 (46-47), swizzle mode 2 = 128B
// (61-63).  The tile must start on a 1024-byte boundary; advancing along K inside the
// 128-byte row is done by adding bytes >> 4 to the start address.
__device__ __forceinline__ uint64_t umma_desc_k128(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
         ((uint64_t)(1024 >> 4) << 32) | ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}

// Instruction descriptor, kind::f16 with bf16 A/B, fp32 accumulator, both K-major:
// D format F32 (bits 4-5 = 1), A format BF16 (7-9 = 1), B format BF16 (10-12 = 1),
// N >> 3 (17-22), M >> 4 (24-28).
__host__ __device__ constexpr uint32_t umma_idesc_bf16(int M, int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) |
         ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem]^T, single CTA, issued by one thread.
__device__ __forceinline__ void umma_bf16(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                          uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// ---------------------------------------------------------------- MXFP8 (block-scaled E4M3)
// Instruction descriptor, kind::mxf8f6f4 with E4M3 A and B (formats 0), both K-major, E8M0
// scale factors (bit 23), N >> 3 (17-22), M >> 4 (24-28); the byte of each 32-bit TMEM scale
// column that this MMA reads: B's in bits 4-5, A's in bits 29-30.
__host__ __device__ constexpr uint32_t umma_idesc_mx_e4m3(int M, int N, uint32_t sf_id) {
  return (sf_id << 4) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((uint32_t)(M >> 4) << 24) |
         (sf_id << 29);
}

// D[tmem] (+)= (A * SFA) (B * SFB)^T over K = 32 with E4M3 operands in shared memory and one
// E8M0 scale per row of A and per row of B in TMEM (scale_vec 1X: one per 32 elements).  The
// scale addresses carry the byte index in bits 30-31, like the descriptor's scale IDs.
__device__ __forceinline__ void umma_mx_e4m3(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                             uint32_t idesc, uint32_t sfa, uint32_t sfb,
                                             uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf8f6f4.block_scale [%0], %1, %2, %3, [%5], [%6], p;\n\t}"
      ::"r"(tmem_d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(sfa), "r"(sfb)
      : "memory");
}

// Shared-memory descriptor of a 32-row x 16-byte matrix stored row after row (no swizzle:
// 8-row core matrices of 128 bytes, 128 bytes apart), the source of tcgen05.cp below.
__device__ __forceinline__ uint64_t sdesc_rows16(uint32_t smem_addr) {
  return (uint64_t)((smem_addr >> 4) & 0x3FFFu) | ((uint64_t)1 << 16) |
         ((uint64_t)(128 >> 4) << 32) | ((uint64_t)1 << 46);
}

// Copy 32 rows x 128 bits from shared memory into TMEM lanes 0-31, columns taddr .. taddr + 3,
// and the same data into lanes 32-63, 64-95 and 96-127 (the scale-factor layout the MMA reads:
// lane i, column c holds the 4 scales of row 32c + i).  Ordered with this thread's later MMAs.
__device__ __forceinline__ void tmem_cp_32x128b_x4(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// Contiguous global -> shared copy of `bytes` (a multiple of 16; both addresses 16-byte
// aligned), completion signalled on `bar` as transaction bytes.  No multicast.
__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_u32(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// E8M0 code of a 32-element block's scale X = 2^E: the smallest E with amax <= 448 2^E, so
// that no element overflows E4M3 (amax = m 2^e, 1 <= m < 2: E = e - 8 for m <= 1.75, else
// e - 7), clamped to [-127, 127]; 127 (X = 1) for an all-zero block.  amax >= 0 and finite.
__device__ __forceinline__ uint32_t mx_scale_code(float amax) {
  if (amax == 0.f) return 127u;
  const uint32_t bits = __float_as_uint(amax);
  const int ex = (int)(bits >> 23);  // biased exponent (sign bit is 0)
  if (ex == 0) return 0u;  // subnormal: E would be below -127, so it is clamped there
  const int E = ex - 127 - 8 + ((bits & 0x7FFFFFu) > 0x600000u ? 1 : 0);  // 0x600000: m = 1.75
  return (uint32_t)(E < -127 ? 0 : E + 127);
}

// 1 / X for an E8M0 code c <= 253: 2^(127 - c), a normal binary32 (codes from mx_scale_code
// never exceed 247).
__device__ __forceinline__ float mx_inv_scale(uint32_t c) {
  return __uint_as_float((254u - c) << 23);
}

// Two binary32 values to OCP FP8 E4M3 codes (nearest, ties to even, saturating to +-448):
// lo's code in the low byte.
__device__ __forceinline__ uint16_t cvt_e4m3x2(float lo, float hi) {
  uint16_t r;
  asm("cvt.rn.satfinite.e4m3x2.f32 %0, %1, %2;" : "=h"(r) : "f"(hi), "f"(lo));
  return r;
}

// Four E4M3 codes of v * inv (inv a power of two), lowest address in the lowest byte.
__device__ __forceinline__ uint32_t e4m3x4_mul(float v0, float v1, float v2, float v3,
                                               float inv) {
  return (uint32_t)cvt_e4m3x2(v0 * inv, v1 * inv) |
         ((uint32_t)cvt_e4m3x2(v2 * inv, v3 * inv) << 16);
}

// Arrive on `bar` once every tcgen05 operation issued so far by this thread has completed.
__device__ __forceinline__ void umma_commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
          smem_u32(bar))
      : "memory");
}

// Each thread of the warp reads 32 consecutive fp32 columns of its own TMEM lane.
__device__ __forceinline__ void tmem_ld32(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]),
        "=r"(r[19]), "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]),
        "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]),
        "=r"(r[31])
      : "r"(taddr));
}

// 16 consecutive columns.
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, uint32_t (&r)[16]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]),
        "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
      : "r"(taddr));
}

__device__ __forceinline__ void tmem_ld_wait() {
  asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
}

// ---------------------------------------------------------------- CTA pairs (cluster of 2)
__device__ __forceinline__ uint32_t cluster_ctarank() {
  uint32_t r;
  asm volatile("mov.u32 %0, %%cluster_ctarank;" : "=r"(r));
  return r;
}

// Shared::cluster address of the same shared-memory object in CTA `rank` of the cluster.
__device__ __forceinline__ uint32_t map_to_rank(const void* p, uint32_t rank) {
  uint32_t out;
  asm volatile("mapa.shared::cluster.u32 %0, %1, %2;" : "=r"(out) : "r"(smem_u32(p)), "r"(rank));
  return out;
}

// Arrive on an mbarrier given by its shared::cluster address (possibly in the peer CTA).
__device__ __forceinline__ void mbar_arrive_cluster(uint32_t cluster_addr) {
  asm volatile("mbarrier.arrive.release.cluster.shared::cluster.b64 _, [%0];" ::"r"(cluster_addr)
               : "memory");
}

// Four floats from shared memory of a CTA of this cluster (16-byte aligned address).  Issue
// several of these back to back before using any: they complete in parallel.
__device__ __forceinline__ float4 ld_cluster_v4(uint32_t cluster_addr) {
  float4 v;
  asm volatile("ld.shared::cluster.v4.f32 {%0, %1, %2, %3}, [%4];"
               : "=f"(v.x), "=f"(v.y), "=f"(v.z), "=f"(v.w)
               : "r"(cluster_addr)
               : "memory");
  return v;
}

// Every thread of every CTA of the cluster: makes prior shared-memory writes (barrier
// initialisation included) visible cluster-wide.
__device__ __forceinline__ void cluster_sync_all() {
  asm volatile("barrier.cluster.arrive.release.aligned;\n\tbarrier.cluster.wait.acquire.aligned;"
               ::: "memory");
}

// 2-D tile load by either CTA of a pair; completion is counted on the mbarrier at
// `bar_cluster_addr` (the leader CTA's barrier).  No multicast.
__device__ __forceinline__ void tma_load_2d_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t x,
                                                 int32_t y, uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.mbarrier::complete_tx::bytes"
      ".L2::cache_hint [%0], [%1, {%3, %4}], [%2], %5;" ::"r"(smem_u32(smem_dst)),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr), "r"(x), "r"(y),
      "l"(cache_hint)
      : "memory");
}

// Four rows y0..y3 of a 2-D tensor whose map has a one-row box (64 bf16, 128-byte swizzle)
// into 512 consecutive bytes of this CTA's shared memory, completion on its barrier `bar`.
// Rows outside the tensor arrive as zeros.  No multicast.
__device__ __forceinline__ void tma_gather4(void* smem_dst, const CUtensorMap* map,
                                            uint64_t* bar, int32_t x, int32_t y0, int32_t y1,
                                            int32_t y2, int32_t y3, uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile::gather4"
      ".mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(smem_u32(bar)),
      "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "l"(cache_hint)
      : "memory");
}

// Four rows y0..y3 of a 2-D bf16 tensor whose map has a one-row box (64 elements, 128-byte
// swizzle) into 512 consecutive bytes of shared memory, by either CTA of a pair; completion
// is counted on the leader's barrier.  Rows outside the tensor (e.g. y = number of rows)
// arrive as zeros.  No multicast.
__device__ __forceinline__ void tma_gather4_pair(void* smem_dst, const CUtensorMap* map,
                                                 uint32_t bar_cluster_addr, int32_t x,
                                                 int32_t y0, int32_t y1, int32_t y2, int32_t y3,
                                                 uint64_t cache_hint) {
  asm volatile(
      "cp.async.bulk.tensor.2d.cta_group::2.shared::cluster.global.tile::gather4"
      ".mbarrier::complete_tx::bytes.L2::cache_hint [%0], [%1, {%3, %4, %5, %6, %7}], [%2], %8;"
      ::"r"(smem_u32(smem_dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(bar_cluster_addr),
      "r"(x), "r"(y0), "r"(y1), "r"(y2), "r"(y3), "l"(cache_hint)
      : "memory");
}

__device__ __forceinline__ void tmem_alloc_pair(uint32_t* dst_smem, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::2.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(
                   smem_u32(dst_smem)),
               "r"(ncols)
               : "memory");
}
__device__ __forceinline__ void tmem_relinquish_pair() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::2.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc_pair(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::2.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols)
               : "memory");
}

// D[tmem of both CTAs] (+)= A[rows of both CTAs] * B[columns split over both CTAs]^T, issued
// by one thread of the leader CTA; M = 256 (128 rows per CTA).
__device__ __forceinline__ void umma_bf16_pair(uint32_t tmem_d, uint64_t adesc, uint64_t bdesc,
                                               uint32_t idesc, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::2.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(tmem_d),
      "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
      : "memory");
}

// Arrive on the barrier at this shared-memory offset in every CTA of `cta_mask` once all
// prior tcgen05 operations of this thread (pair MMAs included) have completed.
__device__ __forceinline__ void umma_commit_pair(uint64_t* bar, uint16_t cta_mask) {
  asm volatile(
      "tcgen05.commit.cta_group::2.mbarrier::arrive::one.shared::cluster.multicast::cluster.b64"
      " [%0], %1;" ::"r"(smem_u32(bar)),
      "h"(cta_mask)
      : "memory");
}

}  // namespace moe
