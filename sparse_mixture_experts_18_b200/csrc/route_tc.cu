// route_tc.cu -- the router of large batches on the tensor cores.
//
// The router logits l = x . W_g ("Mixtral of Experts", method section, equation G(x)) are a
// dense contraction over the hidden dimension, T x d by d x n.  On sm_100a the CUDA cores
// reach barely the rate at which x streams from HBM at n = 8 (four multiply-adds per byte),
// so the contraction runs on the tensor cores, keeping the router exact in fp32:
//
//   * W_g (fp32) is split into three bf16 parts, w = hi + mid + lo, with hi = bf16(w),
//     mid = bf16(w - hi), lo = bf16(w - hi - mid): each step removes the leading 8
//     significant bits, so the three parts hold all 24 bits of w and the sum is exact
//     (wg_split_kernel, into [3n rounded up to 16][d] K-major rows);
//   * each product x_j * part_j of two bf16 values is exact in fp32, and the tensor core sums
//     them in fp32 (tcgen05.mma kind::f16, accumulator in TMEM); the logit of expert e is
//     (S_hi + S_mid) + S_lo of its three accumulator columns.
//
// One CTA per 128-token tile and K range: a cluster of CS CTAs (CS = 1, 2 or 4) splits the
// hidden dimension; each CTA then takes a share of the tile's tokens and adds all ranks'
// partial sums of them in rank order through distributed shared memory.  Warp 0 streams x
// and the W_g parts with TMA (no multicast), one thread of warp 1 issues the MMAs, warps 2-5
// read the accumulators (one token per thread) and run TopK (ties to the lower index) and the
// softmax over the kept logits, and write the token block histograms the scan kernel takes
// (8-token blocks, as router_topk_kernel).
#include "internal.h"

namespace moe {

constexpr int RTC_THREADS = 192;
constexpr int RTC_TILE = 128;         // tokens per tile (MMA M)
constexpr int RTC_MAX_STAGES = 12;
constexpr int RTC_MAX_N = 64;         // experts
// one CTA per SM with as many stages in flight as shared memory holds (two CTAs per SM with
// half the stages each measured slower)
constexpr uint32_t RTC_SMEM_BUDGET = 200 * 1024;

__host__ __device__ constexpr int rtc_npad(int n) { return (3 * n + 15) / 16 * 16; }
// floats per row of partial sums: 16-byte rows, and four banks apart from row to row so that
// the 16-byte accesses of eight consecutive rows fall in different banks
__host__ __device__ constexpr int rtc_pstride(int npad) { return npad + 4; }
__host__ __device__ constexpr uint32_t rtc_tmem_cols(int npad) {
  return npad <= 32 ? 32 : npad <= 64 ? 64 : npad <= 128 ? 128 : 256;
}

// W_g [d][n] fp32 -> parts [npad][d] bf16: row e = hi of column e, n + e = mid, 2n + e = lo,
// rows from 3n on are zero.
__global__ void __launch_bounds__(256)
    wg_split_kernel(const float* __restrict__ Wg, int d, int n, int npad,
                    __nv_bfloat16* __restrict__ parts) {
  // W_g is the caller's, but the parts buffer may still be read by the previous call's router
  pdl_wait();
  pdl_trigger();
  const int64_t total = (int64_t)npad * d;
  for (int64_t i = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; i < total;
       i += (int64_t)gridDim.x * blockDim.x) {
    const int r = (int)(i / d), j = (int)(i % d);
    float v = 0.f;
    if (r < 3 * n) {
      const int e = r % n, part = r / n;
      const float w = Wg[(int64_t)j * n + e];
      const __nv_bfloat16 hi = __float2bfloat16_rn(w);
      const float r1 = w - __bfloat162float(hi);  // exact: w and hi agree in the leading bits
      const __nv_bfloat16 mid = __float2bfloat16_rn(r1);
      const float r2 = r1 - __bfloat162float(mid);  // exact likewise; at most 8 bits remain
      v = part == 0 ? __bfloat162float(hi) : part == 1 ? __bfloat162float(mid) : r2;
    }
    parts[i] = __float2bfloat16_rn(v);  // hi and mid are bf16 already; lo = r2 fits in bf16
  }
}

struct RtcCtrl {
  uint64_t full[RTC_MAX_STAGES];
  uint64_t empty[RTC_MAX_STAGES];
  uint64_t tfull;
  uint64_t mma_done;
  uint32_t issued[RTC_MAX_STAGES];
  uint32_t tmem_slot;
  int abort;
};

// MAXN: 16 or 64, the most experts the instance handles (its TopK loops are unrolled to it)
template <int CS, int MAXN>
__global__ void __launch_bounds__(RTC_THREADS, 1)
    router_tc_kernel(const __grid_constant__ CUtensorMap tmX,
                     const __grid_constant__ CUtensorMap tmW, int64_t T, int n, int K,
                     int npad, int kb_per_cta, int stages, int64_t nblk,
                     int32_t* __restrict__ idx,
                     float* __restrict__ gate, int32_t* __restrict__ blk_counts,
                     uint32_t* status) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const uint32_t a_bytes = RTC_TILE * 128, b_bytes = (uint32_t)npad * 128;
  const uint32_t stage_bytes = (a_bytes + b_bytes + 1023u) & ~1023u;
  RtcCtrl* c = reinterpret_cast<RtcCtrl*>(smem + (size_t)stages * stage_bytes);
  // [RTC_TILE][pstride] partial sums, 16-byte aligned rows: in the stages' memory, which
  // is idle once the accumulator is complete (every load issued has been consumed by then)
  float* part = reinterpret_cast<float*>(smem);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = CS > 1 ? cluster_ctarank() : 0;
  const int64_t tile = blockIdx.x / CS;
  const int64_t t0 = tile * RTC_TILE;
  const int kb0 = (int)rank * kb_per_cta;

  if (threadIdx.x == 0) {
    for (int s = 0; s < stages; ++s) {
      mbar_init(&c->full[s], 1);
      mbar_init(&c->empty[s], 1);
      c->issued[s] = 0;
    }
    mbar_init(&c->tfull, 1);
    mbar_init(&c->mma_done, 1);
    c->abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW);
  }
  const uint32_t tmem_cols = rtc_tmem_cols(npad);
  const int pstride = rtc_pstride(npad);
  if (warp == 1) {
    tmem_alloc(&c->tmem_slot, tmem_cols);
    tmem_relinquish();
  }
  pdl_wait();  // x and the W_g parts come from the previous kernels
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = c->tmem_slot;

  if (warp == 0) {
    if (lane == 0) {  // ------------------------------------------------ TMA producer
      const uint64_t pol_x = policy_evict_first(), pol_w = policy_evict_last();
      for (int kb = 0; kb < kb_per_cta; ++kb) {
        const int stage = kb % stages;
        const uint32_t phase = (uint32_t)(kb / stages) & 1u;
        if (!mbar_wait(&c->empty[stage], phase ^ 1u, status, &c->abort)) break;
        uint8_t* st = smem + (size_t)stage * stage_bytes;
        mbar_arrive_expect_tx(&c->full[stage], a_bytes + b_bytes);
        const int k = (kb0 + kb) * 64;
        tma_load_2d(st, &tmX, &c->full[stage], k, (int32_t)t0, pol_x);  // rows >= T: zeros
        tma_load_2d(st + a_bytes, &tmW, &c->full[stage], k, 0, pol_w);
        c->issued[stage] += 1;
      }
      if (c->abort)  // let every issued copy land before the shared memory goes away
        for (int s = 0; s < stages; ++s)
          if (c->issued[s]) wait_short(&c->full[s], (c->issued[s] - 1u) & 1u);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {  // ------------------------------------------------ MMA issuer
      const uint32_t idesc = umma_idesc_bf16(RTC_TILE, npad);
      bool ok = true;
      for (int kb = 0; kb < kb_per_cta && ok; ++kb) {
        const int stage = kb % stages;
        const uint32_t phase = (uint32_t)(kb / stages) & 1u;
        if (!mbar_wait(&c->full[stage], phase, status, &c->abort)) { ok = false; break; }
        tc_fence_after();
        const uint32_t sb = smem_u32(smem + (size_t)stage * stage_bytes);
#pragma unroll
        for (int kk = 0; kk < 4; ++kk)
          umma_bf16(tmem_base, umma_desc_k128(sb + kk * 32),
                    umma_desc_k128(sb + a_bytes + kk * 32), idesc, (kb | kk) != 0);
        umma_commit(&c->empty[stage]);
      }
      if (ok) umma_commit(&c->tfull);
      if (c->abort) {
        umma_commit(&c->mma_done);
        wait_short(&c->mma_done, 0);
      }
    }
    __syncwarp();
  } else {  // ---------------------------------------------------------- epilogue, warps 2-5
    // this thread's token (TMEM lane / accumulator row r): its npad partial sums go to its
    // row of `part` (zeros if a wait ran out; the status word then reports it)
    const int q = warp & 3, r = q * 32 + lane;
    float4* mine = reinterpret_cast<float4*>(part + r * pstride);
    const bool ok = mbar_wait(&c->tfull, 0, status, &c->abort);
    if (__all_sync(0xffffffffu, ok)) {
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16);
      for (int c0 = 0; c0 < npad; c0 += 32) {  // npad is a multiple of 16
        if (c0 + 32 <= npad) {
          uint32_t v[32];
          tmem_ld32(tb + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 8; ++i)
            mine[c0 / 4 + i] =
                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        } else {
          uint32_t v[16];
          tmem_ld16(tb + c0, v);
          tmem_ld_wait();
#pragma unroll
          for (int i = 0; i < 4; ++i)
            mine[c0 / 4 + i] =
                make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                            __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
        }
      }
    } else {
      for (int i = 0; i < npad / 4; ++i) mine[i] = make_float4(0.f, 0.f, 0.f, 0.f);
    }
  }

  if (CS > 1) cluster_sync_all();  // every CTA's partial sums are in its shared memory
  // the tile's 32-token quarters are shared out over the cluster (quarter q to rank q % CS):
  // the CTA adds every rank's partial sums of its quarters' tokens in rank order, then runs
  // TopK, the softmax and the histograms for them
  if (warp >= 2 && (uint32_t)((warp & 3) % CS) == rank) {
    const int q = warp & 3, r = q * 32 + lane;
    const int64_t t = t0 + r;
    float* mine = part + r * pstride;
    if (CS > 1) {  // the K ranges in rank order, 48 columns per batch of loads
      float4* m4 = reinterpret_cast<float4*>(mine);
      constexpr int CH = 12;  // float4 per batch
      for (int c4 = 0; c4 < npad / 4; c4 += CH) {
        float4 sum[CH];
        {
          const uint32_t base0 = map_to_rank(mine, 0) + 16u * (uint32_t)c4;
#pragma unroll
          for (int i = 0; i < CH; ++i)
            if (c4 + i < npad / 4) sum[i] = ld_cluster_v4(base0 + 16u * (uint32_t)i);
        }
        for (uint32_t p = 1; p < (uint32_t)CS; ++p) {
          const uint32_t base = map_to_rank(mine, p) + 16u * (uint32_t)c4;
          float4 t4[CH];
#pragma unroll
          for (int i = 0; i < CH; ++i)
            if (c4 + i < npad / 4) t4[i] = ld_cluster_v4(base + 16u * (uint32_t)i);
#pragma unroll
          for (int i = 0; i < CH; ++i)
            if (c4 + i < npad / 4) {
              sum[i].x += t4[i].x; sum[i].y += t4[i].y; sum[i].z += t4[i].z; sum[i].w += t4[i].w;
            }
        }
#pragma unroll
        for (int i = 0; i < CH; ++i)
          if (c4 + i < npad / 4) m4[c4 + i] = sum[i];
      }
    }
    float l[MAXN];
#pragma unroll
    for (int e = 0; e < MAXN; ++e)
      l[e] = e < n ? (mine[e] + mine[n + e]) + mine[2 * n + e] : -INFINITY;
    // TopK by repeated arg-max (strict '>' keeps the lower index on ties), then Softmax over
    // the kept logits shifted by the largest, summed in slot order
    int sel[8];
    float kept[8];
    const bool valid = t < T;
    uint64_t used = 0;
    float top = 0.f, z = 0.f;
#pragma unroll
    for (int k = 0; k < 8; ++k) {
      sel[k] = -1;
      if (k >= K) continue;
      int best = 0;
      float bv = -INFINITY;
      bool any = false;
#pragma unroll
      for (int e = 0; e < MAXN; ++e) {
        if (e >= n || ((used >> e) & 1ull)) continue;
        if (!any || l[e] > bv) { best = e; bv = l[e]; any = true; }
      }
      used |= 1ull << best;
      if (k == 0) top = bv;
      z += expf(bv - top);
      sel[k] = best;
      kept[k] = bv;
    }
    if (valid) {
#pragma unroll
      for (int k = 0; k < 8; ++k)
        if (k < K) {
          idx[t * K + k] = sel[k];
          gate[t * K + k] = expf(kept[k] - top) / z;
        }
    }
    // histograms of the 8-token blocks of this warp's 32 tokens: lanes 8j .. 8j + 7 = block j
    const int j = lane >> 3;
    const int64_t b = t0 / 8 + q * 4 + j;
    for (int e = 0; e < n; ++e) {
      int cnt = 0;
#pragma unroll
      for (int k = 0; k < 8; ++k) {
        if (k >= K) continue;
        const uint32_t bal = __ballot_sync(0xffffffffu, valid && sel[k] == e);
        cnt += __popc(bal & (0xffu << (8 * j)));
      }
      if ((lane & 7) == (e & 7) && b < nblk) blk_counts[b * n + e] = cnt;
    }
  }
  if (CS > 1) cluster_sync_all();  // every rank has read the partial sums it needs

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, tmem_cols);
}

// ---------------------------------------------------------------- host side

bool router_tc_applies(const Plan& p) {
  return p.dt == 1 && p.T >= 1024 && p.n <= RTC_MAX_N && p.K <= 8 && p.d % 64 == 0;
}

size_t router_tc_parts_bytes(int64_t d, int n) { return (size_t)rtc_npad(n) * d * 2; }

// Pipeline stages and dynamic shared memory of the router for npad accumulator columns.
static size_t rtc_smem(int npad, int* stages_out) {
  const uint32_t stage_bytes = (uint32_t)((RTC_TILE * 128 + npad * 128 + 1023) / 1024 * 1024);
  const size_t fixed = sizeof(RtcCtrl) + 1024;
  int stages = (int)((RTC_SMEM_BUDGET - fixed) / stage_bytes);
  if (stages > RTC_MAX_STAGES) stages = RTC_MAX_STAGES;
  if (stages < 2) stages = 2;
  // the partial sums [RTC_TILE][pstride] reuse the stages' memory
  while ((size_t)stages * stage_bytes < (size_t)RTC_TILE * rtc_pstride(npad) * 4) ++stages;
  *stages_out = stages;
  return (size_t)stages * stage_bytes + fixed;
}

template <int CS, int MAXN>
static cudaError_t launch_rtc(const CUtensorMap& mx, const CUtensorMap& mw, const Plan& p,
                              int npad, int64_t tiles, const Workspace& w, cudaStream_t s) {
  int stages = 0;
  const size_t smem = rtc_smem(npad, &stages);
  auto kern = router_tc_kernel<CS, MAXN>;
  static int configured[MAX_DEVICES] = {0};
  const cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  attr[1].id = cudaLaunchAttributeClusterDimension;
  attr[1].val.clusterDim.x = CS;
  attr[1].val.clusterDim.y = 1;
  attr[1].val.clusterDim.z = 1;
  cfg.gridDim = dim3((unsigned)(tiles * CS), 1, 1);
  cfg.blockDim = dim3(RTC_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = CS > 1 ? 2 : 1;
  const int kb_per_cta = (int)(p.d / 64 / CS);
  return cudaLaunchKernelEx(&cfg, kern, mx, mw, p.T, p.n, p.K, npad, kb_per_cta, stages, p.nblk,
                            w.idx, w.gate, w.blk_counts, w.status);
}

cudaError_t launch_router_tc(const Plan& p, const void* x, const float* Wg, const Workspace& w,
                             cudaStream_t s) {
  const int npad = rtc_npad(p.n);
  const int d = (int)p.d;
  const int64_t total = (int64_t)npad * d;
  int64_t blocks = (total + 255) / 256;
  if (blocks > 4 * (int64_t)num_sms()) blocks = 4 * (int64_t)num_sms();
  pdl(wg_split_kernel, (unsigned)blocks, 256, 0, s)(Wg, d, p.n, npad, w.wparts);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  CUtensorMap mx, mw;
  if (!make_map_bf16(&mx, x, (uint64_t)d, (uint64_t)p.T, RTC_TILE) ||
      !make_map_bf16(&mw, w.wparts, (uint64_t)d, (uint64_t)npad, (uint32_t)npad))
    return cudaErrorInvalidValue;
  // cluster size c of 1, 2 or 4 (dividing d / 64) minimising the estimated time: waves of
  // CTAs (two per SM when their shared memory allows) times (1/c of a tile's stream + a fixed
  // cost per CTA of 0.15 of it)
  const int64_t tiles = (p.T + RTC_TILE - 1) / RTC_TILE;
  int stages = 0;
  const size_t smem = rtc_smem(npad, &stages);
  const int64_t slots = (2 * (smem + 1024) <= 228 * 1024 ? 2 : 1) * (int64_t)num_sms();
  int cs = 1;
  double best = 1e30;
  for (int c = 1; c <= 4; c <<= 1) {
    if ((d / 64) % c) break;
    const double t = (double)((tiles * c + slots - 1) / slots) * (1.0 / c + 0.15);
    if (t < best * 0.99) { best = t; cs = c; }
  }
  if (p.n <= 16) {
    switch (cs) {
      case 1: return launch_rtc<1, 16>(mx, mw, p, npad, tiles, w, s);
      case 2: return launch_rtc<2, 16>(mx, mw, p, npad, tiles, w, s);
      default: return launch_rtc<4, 16>(mx, mw, p, npad, tiles, w, s);
    }
  }
  switch (cs) {
    case 1: return launch_rtc<1, 64>(mx, mw, p, npad, tiles, w, s);
    case 2: return launch_rtc<2, 64>(mx, mw, p, npad, tiles, w, s);
    default: return launch_rtc<4, 64>(mx, mw, p, npad, tiles, w, s);
  }
}

}  // namespace moe
