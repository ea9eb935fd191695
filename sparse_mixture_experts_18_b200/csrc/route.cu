// route.cu -- routing kernels of the MoE block forward.
//
//  router_topk:   l = x . W_g (fp32 accumulation), TopK (ties -> lower expert index) and
//                 Softmax over the K kept logits ("Mixtral of Experts", method section,
//                 equation G(x)); also a per-block expert histogram.
//  route_scan:    per-expert exclusive prefix over router blocks and the row offsets of each
//                 expert's group (each group padded to `row_align` rows).
//  permute:       stable placement of every (token, slot) in its expert's group, the
//                 inverse map token -> row, and the gather of x rows into that order.  This
//                 is how experts with zero gate are skipped (Indonesian news summary,
//                 section on how the MoE layer is computed) while each expert sees a
//                 variable number of tokens (same page, implementation notes).
#include "internal.h"

namespace moe {

constexpr int ROUTE_THREADS = 256;  // 8 warps split the hidden dimension of a token block

template <typename Tin>
struct Vec8;  // 8 consecutive activations, loaded as 16 or 32 bytes

template <>
struct Vec8<__nv_bfloat16> {
  uint4 raw;
  __device__ __forceinline__ void load(const __nv_bfloat16* p) {
    raw = __ldg(reinterpret_cast<const uint4*>(p));
  }
  __device__ __forceinline__ float get(int i) const {
    const uint32_t w = i < 2 ? raw.x : i < 4 ? raw.y : i < 6 ? raw.z : raw.w;
    return (i & 1) ? bf16_hi(w) : bf16_lo(w);
  }
};

template <>
struct Vec8<float> {
  float4 a, b;
  __device__ __forceinline__ void load(const float* p) {
    a = __ldg(reinterpret_cast<const float4*>(p));
    b = __ldg(reinterpret_cast<const float4*>(p) + 1);
  }
  __device__ __forceinline__ float get(int i) const {
    switch (i) {
      case 0: return a.x; case 1: return a.y; case 2: return a.z; case 3: return a.w;
      case 4: return b.x; case 5: return b.y; case 6: return b.z; default: return b.w;
    }
  }
};

// Block b handles tokens [b*TOKB, b*TOKB + TOKB).  Each thread accumulates the logits of all
// TOKB tokens over its 8-element chunks of the hidden dimension (so a W_g row is loaded once
// per TOKB tokens); lanes and then warps are summed in a fixed order.
template <typename Tin, int NPAD, int TOKB>
__global__ void __launch_bounds__(ROUTE_THREADS)
    router_topk_kernel(const Tin* __restrict__ x, const float* __restrict__ Wg, int64_t T,
                       int d, int n, int K, int32_t* __restrict__ idx,
                       float* __restrict__ gate, int32_t* __restrict__ blk_counts) {
  static_assert(NPAD * TOKB == 64, "64 partial sums per lane");
  __shared__ float red[ROUTE_THREADS / 32][64];
  __shared__ float logits[TOKB][NPAD];
  __shared__ int hist[64];

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t t0 = (int64_t)blockIdx.x * TOKB;
  const int ntok = (int)(T - t0 < TOKB ? T - t0 : TOKB);
  if (threadIdx.x < 64) hist[threadIdx.x] = 0;

  float acc[TOKB][NPAD];
#pragma unroll
  for (int a = 0; a < TOKB; ++a)
#pragma unroll
    for (int e = 0; e < NPAD; ++e) acc[a][e] = 0.f;

  // 8-element chunks of the hidden dimension, thread-interleaved (coalesced 16-byte loads)
  for (int ci = threadIdx.x; ci < d / 8; ci += ROUTE_THREADS) {
    const int j0 = ci * 8;
    Vec8<Tin> xv[TOKB];
#pragma unroll
    for (int a = 0; a < TOKB; ++a)
      if (a < ntok) xv[a].load(x + (t0 + a) * (int64_t)d + j0);
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      float w[NPAD];
      const float* wr = Wg + (int64_t)(j0 + i) * n;
      if (NPAD == 8 && n == 8) {  // one 32-byte row: two aligned float4 loads
        const float4 w0 = __ldg(reinterpret_cast<const float4*>(wr));
        const float4 w1 = __ldg(reinterpret_cast<const float4*>(wr) + 1);
        w[0] = w0.x; w[1] = w0.y; w[2] = w0.z; w[3] = w0.w;
        w[4] = w1.x; w[5] = w1.y; w[6] = w1.z; w[7] = w1.w;
      } else {
#pragma unroll
        for (int e = 0; e < NPAD; ++e) w[e] = e < n ? __ldg(wr + e) : 0.f;
      }
#pragma unroll
      for (int a = 0; a < TOKB; ++a) {
        if (a < ntok) {
          const float xa = xv[a].get(i);
#pragma unroll
          for (int e = 0; e < NPAD; ++e) acc[a][e] = fmaf(xa, w[e], acc[a][e]);
        }
      }
    }
  }

  // Butterfly reduce-scatter of the 64 partial sums over the 32 lanes: after five steps
  // each lane owns two complete warp sums.
  float v[64];
#pragma unroll
  for (int a = 0; a < TOKB; ++a)
#pragma unroll
    for (int e = 0; e < NPAD; ++e) v[a * NPAD + e] = acc[a][e];
  int base = 0;
#pragma unroll
  for (int half = 32, off = 16; off >= 1; half >>= 1, off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < half; ++i) {
      const float send = upper ? v[i] : v[half + i];
      const float keep = upper ? v[half + i] : v[i];
      v[i] = keep + __shfl_xor_sync(0xffffffffu, send, off);
    }
    if (upper) base += half;
  }
  red[warp][base] = v[0];
  red[warp][base + 1] = v[1];
  __syncthreads();
  if (threadIdx.x < 64) {
    float s = 0.f;
#pragma unroll
    for (int w = 0; w < ROUTE_THREADS / 32; ++w) s += red[w][threadIdx.x];
    logits[threadIdx.x / NPAD][threadIdx.x % NPAD] = s;
  }
  __syncthreads();

  // TopK by repeated arg-max (strict '>' keeps the lower index on ties), then Softmax over
  // the kept logits shifted by the largest.
  if (threadIdx.x < ntok) {
    const int a = threadIdx.x;
    const int64_t t = t0 + a;
    uint64_t used = 0;
    float top = 0.f, z = 0.f;
    int sel[64];
    float val[64];
    for (int k = 0; k < K; ++k) {
      int best = -1;
      float bv = 0.f;
      for (int e = 0; e < n; ++e) {
        if ((used >> e) & 1ull) continue;
        const float le = logits[a][e];
        if (best < 0 || le > bv) { best = e; bv = le; }
      }
      used |= 1ull << best;
      sel[k] = best;
      val[k] = bv;
      if (k == 0) top = bv;
      z += expf(bv - top);
      atomicAdd(&hist[best], 1);
    }
    for (int k = 0; k < K; ++k) {
      idx[t * K + k] = sel[k];
      gate[t * K + k] = expf(val[k] - top) / z;
    }
  }
  __syncthreads();
  if (threadIdx.x < n) blk_counts[(int64_t)blockIdx.x * n + threadIdx.x] = hist[threadIdx.x];
}

// One CTA: for every expert, exclusive prefix of the block histograms over blocks, the
// expert's total, and the start row of its group (groups padded to row_align rows).
__global__ void __launch_bounds__(1024)
    route_scan_kernel(const int32_t* __restrict__ blk_counts, int64_t nblk, int n,
                      int row_align, int64_t rows_max, int32_t* __restrict__ blk_base,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      uint32_t* status) {
  __shared__ int wsum[32];
  __shared__ int total[64];
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t chunk = (nblk + blockDim.x - 1) / blockDim.x;
  const int64_t b0 = tid * chunk, b1 = b0 + chunk < nblk ? b0 + chunk : nblk;
  for (int e = 0; e < n; ++e) {
    int local = 0;
    for (int64_t b = b0; b < b1; ++b) local += blk_counts[b * n + e];
    // inclusive warp scan, then across warps
    int incl = local;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int s = lane < (int)(blockDim.x >> 5) ? wsum[lane] : 0;
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xffffffffu, s, off);
        if (lane >= off) s += y;
      }
      wsum[lane] = s;  // inclusive over warps
    }
    __syncthreads();
    int run = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
    for (int64_t b = b0; b < b1; ++b) {
      blk_base[b * n + e] = run;
      run += blk_counts[b * n + e];
    }
    if (tid == 0) total[e] = wsum[(blockDim.x >> 5) - 1];
    __syncthreads();
  }
  if (tid == 0) {
    int64_t off = 0;
    for (int e = 0; e < n; ++e) {
      counts[e] = total[e];
      offsets[e] = (int32_t)off;
      off += (int64_t)(total[e] + row_align - 1) / row_align * row_align;
    }
    offsets[n] = (int32_t)off;
    if (off > rows_max) set_status(status, DEV_ERR_ROW);
  }
}

// Block b takes the same tokens as router block b.  Entry i = (token, slot) in token-major
// order gets rank = number of earlier entries of this block routed to the same expert, so
// the placement is stable (rows of an expert ordered by token, then slot).
template <typename Tact>
__global__ void __launch_bounds__(256)
    permute_gather_kernel(const Tact* __restrict__ x, int64_t T, int d, int n, int K,
                          int tokb, const int32_t* __restrict__ idx,
                          const int32_t* __restrict__ blk_base,
                          const int32_t* __restrict__ offsets, int64_t rows_max,
                          int32_t* __restrict__ inv, Tact* __restrict__ xperm,
                          uint32_t* status) {
  __shared__ int ent_e[64];
  __shared__ int ent_row[64];
  const int64_t t0 = (int64_t)blockIdx.x * tokb;
  const int ntok = (int)(T - t0 < tokb ? T - t0 : tokb);
  const int E = ntok * K;  // <= 64 by construction (tokb * K <= tokb * NPAD = 64)
  const int i = threadIdx.x;
  if (i < E) ent_e[i] = idx[t0 * K + i];
  __syncthreads();
  if (i < E) {
    const int e = ent_e[i];
    int row = -1;
    if (e < 0 || e >= n) {
      set_status(status, DEV_ERR_EXPERT);
    } else {
      int rank = 0;
      for (int j = 0; j < i; ++j) rank += ent_e[j] == e;
      row = offsets[e] + blk_base[(int64_t)blockIdx.x * n + e] + rank;
      if (row < 0 || row >= rows_max) {
        set_status(status, DEV_ERR_ROW);
        row = -1;
      }
    }
    ent_row[i] = row;
    inv[t0 * K + i] = row;
  }
  __syncthreads();
  // gather: 16-byte vectors of each selected x row into its permuted row
  const int vpr = d * (int)sizeof(Tact) / 16;
  for (int v = threadIdx.x; v < E * vpr; v += blockDim.x) {
    const int ei = v / vpr, c = v % vpr;
    const int row = ent_row[ei];
    if (row < 0) continue;
    const int64_t t = t0 + ei / K;
    const uint4 val = __ldg(reinterpret_cast<const uint4*>(x + t * d) + c);
    reinterpret_cast<uint4*>(xperm + (int64_t)row * d)[c] = val;
  }
}

// ---------------------------------------------------------------- host launchers

int route_tokens_per_block(int n) { return n <= 8 ? 8 : n <= 16 ? 4 : n <= 32 ? 2 : 1; }

template <typename Tin>
static cudaError_t launch_router_t(const Tin* x, const float* Wg, int64_t T, int d, int n,
                                   int K, int32_t* idx, float* gate, int32_t* blk_counts,
                                   cudaStream_t s) {
  const int tokb = route_tokens_per_block(n);
  const unsigned grid = (unsigned)((T + tokb - 1) / tokb);
  if (n <= 8)
    router_topk_kernel<Tin, 8, 8><<<grid, ROUTE_THREADS, 0, s>>>(x, Wg, T, d, n, K, idx, gate,
                                                                 blk_counts);
  else if (n <= 16)
    router_topk_kernel<Tin, 16, 4><<<grid, ROUTE_THREADS, 0, s>>>(x, Wg, T, d, n, K, idx,
                                                                  gate, blk_counts);
  else if (n <= 32)
    router_topk_kernel<Tin, 32, 2><<<grid, ROUTE_THREADS, 0, s>>>(x, Wg, T, d, n, K, idx,
                                                                  gate, blk_counts);
  else
    router_topk_kernel<Tin, 64, 1><<<grid, ROUTE_THREADS, 0, s>>>(x, Wg, T, d, n, K, idx,
                                                                  gate, blk_counts);
  return cudaGetLastError();
}

cudaError_t launch_route(const Plan& p, const void* x, const float* Wg, const Workspace& w,
                         cudaStream_t s) {
  cudaError_t err;
  if (p.dt == 1)
    err = launch_router_t(static_cast<const __nv_bfloat16*>(x), Wg, p.T, (int)p.d, p.n, p.K,
                          w.idx, w.gate, w.blk_counts, s);
  else
    err = launch_router_t(static_cast<const float*>(x), Wg, p.T, (int)p.d, p.n, p.K, w.idx,
                          w.gate, w.blk_counts, s);
  if (err != cudaSuccess) return err;
  route_scan_kernel<<<1, 1024, 0, s>>>(w.blk_counts, p.nblk, p.n, p.row_align, p.rows_max,
                                       w.blk_base, w.counts, w.offsets, w.status);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int tokb = route_tokens_per_block(p.n);
  if (p.dt == 1)
    permute_gather_kernel<__nv_bfloat16><<<(unsigned)p.nblk, 256, 0, s>>>(
        static_cast<const __nv_bfloat16*>(x), p.T, (int)p.d, p.n, p.K, tokb, w.idx,
        w.blk_base, w.offsets, p.rows_max, w.inv, static_cast<__nv_bfloat16*>(w.xperm),
        w.status);
  else
    permute_gather_kernel<float><<<(unsigned)p.nblk, 256, 0, s>>>(
        static_cast<const float*>(x), p.T, (int)p.d, p.n, p.K, tokb, w.idx, w.blk_base,
        w.offsets, p.rows_max, w.inv, static_cast<float*>(w.xperm), w.status);
  return cudaGetLastError();
}

}  // namespace moe
