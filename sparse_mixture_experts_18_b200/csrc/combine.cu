// combine.cu -- gate-weighted combine back to token order and the RMSNorm of the stacked
// blocks.
//
//  combine:  out[t] = sum_k G(x_t)_k * y_{e_k}(x_t)  ("Mixtral of Experts", method section,
//            equation y; expert outputs return to their token's original position, as the
//            Indonesian news summary's expert-parallelism notes put it).  fp32 sum over the
//            K slots in slot order (and over split slabs in split order), rounded once;
//            16-byte vectorised loads and stores.  With a residual input, out = resid + sum,
//            also in fp32 before the single rounding (the stacked-block workload).  With the
//            gather-from-x option of the CTA-pair path (MOE_GATHER_X=1) the down-projection
//            epilogue has already multiplied each row by its gate, and the combine only sums
//            the K rows; with FP8 expert weights it applies the h and W2 row scales.
//  rmsnorm:  xn = x / sqrt(mean(x^2) + eps) with unit gain, fp32 math, bf16 result.
#include "internal.h"

namespace moe {

template <typename Tout>
struct Out8;

template <>
struct Out8<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[8]) {
    const uint4 r = *reinterpret_cast<const uint4*>(p);
    const uint32_t w[4] = {r.x, r.y, r.z, r.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      v[2 * i] = bf16_lo(w[i]);
      v[2 * i + 1] = bf16_hi(w[i]);
    }
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[8]) {
    *reinterpret_cast<uint4*>(p) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                              pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
  }
};

template <>
struct Out8<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[8]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    const float4 b = *reinterpret_cast<const float4*>(p + 4);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
    v[4] = b.x; v[5] = b.y; v[6] = b.z; v[7] = b.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[8]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
    *reinterpret_cast<float4*>(p + 4) = make_float4(v[4], v[5], v[6], v[7]);
  }
};

// One thread per 4 output columns of a token.  All K x S loads of a thread are issued
// before they are summed (splits unrolled up to MAX_S), then the fp32 sum over slots is
// taken in slot order and rounded once.
constexpr int COMBINE_MAX_S = 8;

template <typename Tout>
struct Out4;
template <>
struct Out4<__nv_bfloat16> {
  static __device__ __forceinline__ void load(const __nv_bfloat16* p, float (&v)[4]) {
    const uint2 r = *reinterpret_cast<const uint2*>(p);
    v[0] = bf16_lo(r.x); v[1] = bf16_hi(r.x); v[2] = bf16_lo(r.y); v[3] = bf16_hi(r.y);
  }
  static __device__ __forceinline__ void store(__nv_bfloat16* p, const float (&v)[4]) {
    *reinterpret_cast<uint2*>(p) = make_uint2(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]));
  }
};
template <>
struct Out4<float> {
  static __device__ __forceinline__ void load(const float* p, float (&v)[4]) {
    const float4 a = *reinterpret_cast<const float4*>(p);
    v[0] = a.x; v[1] = a.y; v[2] = a.z; v[3] = a.w;
  }
  static __device__ __forceinline__ void store(float* p, const float (&v)[4]) {
    *reinterpret_cast<float4*>(p) = make_float4(v[0], v[1], v[2], v[3]);
  }
};

template <typename Tout, bool RESID>
__global__ void __launch_bounds__(256)
    combine_kernel(const float* __restrict__ Y, int S, int64_t split_stride, int64_t T, int d,
                   int K, const int32_t* __restrict__ inv, const float* __restrict__ gate,
                   Tout* out, const Tout* resid) {
  pdl_wait();
  pdl_trigger();
  const int vpr = d / 4;
  const int64_t total = T * vpr;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t t = v / vpr;
    const int c = (int)(v % vpr) * 4;
    float acc[4] = {0.f, 0.f, 0.f, 0.f};
    for (int k = 0; k < K; ++k) {
      const int row = inv[t * K + k];
      if (row < 0) continue;
      const float g = gate ? gate[t * K + k] : 1.f;  // null: rows already gated
      const float* src = Y + (int64_t)row * d + c;
      float4 part[COMBINE_MAX_S];
#pragma unroll
      for (int s = 0; s < COMBINE_MAX_S; ++s)
        if (s < S) part[s] = __ldg(reinterpret_cast<const float4*>(src + s * split_stride));
      float4 yk = make_float4(0.f, 0.f, 0.f, 0.f);
#pragma unroll
      for (int s = 0; s < COMBINE_MAX_S; ++s)
        if (s < S) {
          yk.x += part[s].x; yk.y += part[s].y; yk.z += part[s].z; yk.w += part[s].w;
        }
      acc[0] = fmaf(g, yk.x, acc[0]);
      acc[1] = fmaf(g, yk.y, acc[1]);
      acc[2] = fmaf(g, yk.z, acc[2]);
      acc[3] = fmaf(g, yk.w, acc[3]);
    }
    if (RESID) {
      float r[4];
      Out4<Tout>::load(resid + t * d + c, r);
#pragma unroll
      for (int i = 0; i < 4; ++i) acc[i] = r[i] + acc[i];
    }
    Out4<Tout>::store(out + t * d + c, acc);
  }
}

// Large batches: one warp per token, each lane 8 groups of 4 columns (128 columns apart)
// per pass, with all of a slot's loads in flight before they are summed.  Same arithmetic
// (split order, then slot order, one rounding) as combine_kernel.
constexpr int COMBINE_U = 8;

template <typename Tout, bool RESID>
__global__ void __launch_bounds__(256)
    combine_rows_kernel(const float* __restrict__ Y, int S, int64_t split_stride, int64_t T,
                        int d, int K, const int32_t* __restrict__ inv,
                        const float* __restrict__ gate, Tout* out, const Tout* resid) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
       t += nwarps) {
    for (int c0 = lane * 4; c0 < d; c0 += 128 * COMBINE_U) {
      float4 acc[COMBINE_U];
#pragma unroll
      for (int u = 0; u < COMBINE_U; ++u) acc[u] = make_float4(0.f, 0.f, 0.f, 0.f);
      for (int k = 0; k < K; ++k) {
        const int row = inv[t * K + k];
        if (row < 0) continue;
        const float g = gate ? gate[t * K + k] : 1.f;  // null: rows already gated
        float4 yk[COMBINE_U];
#pragma unroll
        for (int u = 0; u < COMBINE_U; ++u) yk[u] = make_float4(0.f, 0.f, 0.f, 0.f);
        for (int s = 0; s < S; ++s) {
          const float* src = Y + s * split_stride + (int64_t)row * d + c0;
          float4 v[COMBINE_U];
#pragma unroll
          for (int u = 0; u < COMBINE_U; ++u)
            if (c0 + 128 * u < d) v[u] = __ldg(reinterpret_cast<const float4*>(src + 128 * u));
#pragma unroll
          for (int u = 0; u < COMBINE_U; ++u)
            if (c0 + 128 * u < d) {
              yk[u].x += v[u].x; yk[u].y += v[u].y; yk[u].z += v[u].z; yk[u].w += v[u].w;
            }
        }
#pragma unroll
        for (int u = 0; u < COMBINE_U; ++u) {
          acc[u].x = fmaf(g, yk[u].x, acc[u].x);
          acc[u].y = fmaf(g, yk[u].y, acc[u].y);
          acc[u].z = fmaf(g, yk[u].z, acc[u].z);
          acc[u].w = fmaf(g, yk[u].w, acc[u].w);
        }
      }
#pragma unroll
      for (int u = 0; u < COMBINE_U; ++u) {
        const int c = c0 + 128 * u;
        if (c >= d) continue;
        float o[4] = {acc[u].x, acc[u].y, acc[u].z, acc[u].w};
        if (RESID) {
          float r[4];
          Out4<Tout>::load(resid + t * d + c, r);
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = r[i] + o[i];
        }
        Out4<Tout>::store(out + t * d + c, o);
      }
    }
  }
}

// RMSNorm of one row by one warp, in the column order of the large-batch combine (lane l takes
// columns l*4 + 128 u + 1024 p, four at a time): the sum of squares is accumulated in that
// order with fmaf and reduced by a fixed xor tree, so that the combine that fuses the next
// block's RMSNorm (combine_rows_k2_kernel with NORM) produces bit for bit the same result.
__device__ __forceinline__ float rms_inv_from_sumsq(float ss, int d, float eps) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) ss += __shfl_xor_sync(0xffffffffu, ss, off);
  return 1.0f / sqrtf(ss / (float)d + eps);
}

__device__ __forceinline__ void rms_scale_row(const __nv_bfloat16* xr, __nv_bfloat16* xnr, int d,
                                              int lane, float inv) {
  for (int c0 = lane * 4; c0 < d; c0 += 128 * COMBINE_U) {
#pragma unroll
    for (int u = 0; u < COMBINE_U; ++u) {
      const int c = c0 + 128 * u;
      if (c >= d) continue;
      float v[4];
      Out4<__nv_bfloat16>::load(xr + c, v);
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] *= inv;
      Out4<__nv_bfloat16>::store(xnr + c, v);
    }
  }
}

// combine_rows_kernel for K = 2 without split slabs (the large-batch tilings): both slots'
// loads and the residual's are issued together before any is used, so a lane has 2 x 8
// float4 plus 8 residual vectors in flight; same arithmetic and result as combine_rows_kernel
// (acc = fma(g1, y1, fma(g0, y0, 0)), then resid + acc, rounded once).
// NORM (bf16 only, with the residual): the kernel also writes the RMSNorm of each result row
// (the next stacked block's input) to xn, exactly as rmsnorm_kernel would from the stored row.
template <typename Tout, bool RESID, bool NORM = false>
__global__ void __launch_bounds__(256)
    combine_rows_k2_kernel(const float* __restrict__ Y, int64_t T, int d,
                           const int32_t* __restrict__ inv, const float* __restrict__ gate,
                           Tout* out, const Tout* resid, __nv_bfloat16* xn, float eps) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t nwarps = (int64_t)gridDim.x * (blockDim.x >> 5);
  for (int64_t t = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5); t < T;
       t += nwarps) {
    const int2 rows = *reinterpret_cast<const int2*>(inv + 2 * t);
    float g0 = 1.f, g1 = 1.f;  // null gate: rows already gated
    if (gate) {
      const float2 g = *reinterpret_cast<const float2*>(gate + 2 * t);
      g0 = g.x;
      g1 = g.y;
    }
    const float* y0 = Y + (int64_t)(rows.x < 0 ? 0 : rows.x) * d;
    const float* y1 = Y + (int64_t)(rows.y < 0 ? 0 : rows.y) * d;
    float ss = 0.f;  // NORM: sum of squares of the stored (rounded) row
    for (int c0 = lane * 4; c0 < d; c0 += 128 * COMBINE_U) {
      float4 a[COMBINE_U], b[COMBINE_U];
      float r[COMBINE_U][4];
#pragma unroll
      for (int u = 0; u < COMBINE_U; ++u) {
        const int c = c0 + 128 * u;
        if (c < d) {
          a[u] = __ldg(reinterpret_cast<const float4*>(y0 + c));
          b[u] = __ldg(reinterpret_cast<const float4*>(y1 + c));
          if (RESID) Out4<Tout>::load(resid + t * d + c, r[u]);
        }
      }
#pragma unroll
      for (int u = 0; u < COMBINE_U; ++u) {
        const int c = c0 + 128 * u;
        if (c >= d) continue;
        float o[4] = {0.f, 0.f, 0.f, 0.f};
        if (rows.x >= 0) {
          o[0] = fmaf(g0, a[u].x, o[0]); o[1] = fmaf(g0, a[u].y, o[1]);
          o[2] = fmaf(g0, a[u].z, o[2]); o[3] = fmaf(g0, a[u].w, o[3]);
        }
        if (rows.y >= 0) {
          o[0] = fmaf(g1, b[u].x, o[0]); o[1] = fmaf(g1, b[u].y, o[1]);
          o[2] = fmaf(g1, b[u].z, o[2]); o[3] = fmaf(g1, b[u].w, o[3]);
        }
        if (RESID) {
#pragma unroll
          for (int i = 0; i < 4; ++i) o[i] = r[u][i] + o[i];
        }
        Out4<Tout>::store(out + t * d + c, o);
        if constexpr (NORM) {
          const uint32_t lo = pack_bf16x2(o[0], o[1]), hi = pack_bf16x2(o[2], o[3]);
          const float q[4] = {bf16_lo(lo), bf16_hi(lo), bf16_lo(hi), bf16_hi(hi)};
#pragma unroll
          for (int i = 0; i < 4; ++i) ss = fmaf(q[i], q[i], ss);
        }
      }
    }
    if constexpr (NORM) {
      // this lane re-reads only the columns it stored itself (plain loads, program order)
      rms_scale_row(reinterpret_cast<const __nv_bfloat16*>(out) + t * d, xn + t * d, d, lane,
                    rms_inv_from_sumsq(ss, d, eps));
    }
  }
}

static bool combine_k2_fits(int64_t T, int K, int S, const int32_t* inv, const float* gate) {
  return T >= 1024 && K == 2 && S == 1 && (reinterpret_cast<uintptr_t>(inv) & 7u) == 0 &&
         (!gate || (reinterpret_cast<uintptr_t>(gate) & 7u) == 0);
}

// out[t] = (resid[t] +) sum_k gate[t][k] * sum_s Y[s][inv[t][k]] for T tokens, Tout = bf16
// or fp32 (gate null: 1), picking the one-warp-per-token kernel for T >= 1024.
template <typename Tout>
static cudaError_t combine_rows_t(const float* Y, int S, int64_t split_stride, int64_t T, int d,
                                  int K, const int32_t* inv, const float* gate, Tout* out,
                                  const Tout* resid, cudaStream_t s) {
  if (T >= 1024) {  // enough tokens for one warp each
    const int64_t blocks = (T + 7) / 8;
    const unsigned g = (unsigned)(blocks < ((int64_t)1 << 30) ? blocks : ((int64_t)1 << 30));
    if (combine_k2_fits(T, K, S, inv, gate)) {
      if (resid)
        pdl(combine_rows_k2_kernel<Tout, true>, g, 256, 0, s)(Y, T, d, inv, gate, out, resid,
                                                              nullptr, 0.f);
      else
        pdl(combine_rows_k2_kernel<Tout, false>, g, 256, 0, s)(Y, T, d, inv, gate, out,
                                                               nullptr, nullptr, 0.f);
      return cudaGetLastError();
    }
    if (resid)
      pdl(combine_rows_kernel<Tout, true>, g, 256, 0, s)(Y, S, split_stride, T, d, K, inv, gate,
                                                         out, resid);
    else
      pdl(combine_rows_kernel<Tout, false>, g, 256, 0, s)(Y, S, split_stride, T, d, K, inv,
                                                          gate, out, nullptr);
    return cudaGetLastError();
  }
  const int64_t total = T * (d / 4);
  int64_t blocks = (total + 255) / 256;  // one 4-column item per thread: all loads in flight
  if (blocks > ((int64_t)1 << 30)) blocks = (int64_t)1 << 30;
  if (blocks < 1) blocks = 1;
  if (resid)
    pdl(combine_kernel<Tout, true>, (unsigned)blocks, 256, 0, s)(
        Y, S, split_stride, T, d, K, inv, gate, out, resid);
  else
    pdl(combine_kernel<Tout, false>, (unsigned)blocks, 256, 0, s)(
        Y, S, split_stride, T, d, K, inv, gate, out, nullptr);
  return cudaGetLastError();
}

cudaError_t launch_combine_rows(const float* Y, int S, int64_t split_stride, int64_t T, int d,
                                int K, const int32_t* inv, const float* gate, void* out,
                                const void* resid, bool out_f32, cudaStream_t s) {
  if (out_f32)
    return combine_rows_t(Y, S, split_stride, T, d, K, inv, gate, static_cast<float*>(out),
                          static_cast<const float*>(resid), s);
  return combine_rows_t(Y, S, split_stride, T, d, K, inv, gate,
                        static_cast<__nv_bfloat16*>(out),
                        static_cast<const __nv_bfloat16*>(resid), s);
}

cudaError_t launch_combine(const Plan& p, const Workspace& w, void* out, const void* resid,
                           cudaStream_t s, void* norm_out, float eps, bool* normed) {
  if (normed) *normed = false;
  const float* g2 = p.gather_x ? nullptr : w.gate;
  if (norm_out && resid && p.dt == 1 && !p.fp8 && !p.swap &&
      combine_k2_fits(p.T, p.K, 1, w.inv, g2)) {
    const int64_t blocks = (p.T + 7) / 8;
    const unsigned g = (unsigned)(blocks < ((int64_t)1 << 30) ? blocks : ((int64_t)1 << 30));
    pdl(combine_rows_k2_kernel<__nv_bfloat16, true, true>, g, 256, 0, s)(
        w.y, p.T, (int)p.d, w.inv, g2, static_cast<__nv_bfloat16*>(out),
        static_cast<const __nv_bfloat16*>(resid), static_cast<__nv_bfloat16*>(norm_out), eps);
    if (normed) *normed = true;
    return cudaGetLastError();
  }
  const int S = p.swap ? p.s2 : 1;
  const int64_t split_stride = p.rows_max * p.d;
  const float* gates = p.gather_x ? nullptr : w.gate;  // gather_x: G2 applied the gates
  return launch_combine_rows(w.y, S, split_stride, p.T, (int)p.d, p.K, w.inv, gates, out, resid,
                             p.dt == 0, s);
}

__global__ void __launch_bounds__(256)
    rmsnorm_kernel(const __nv_bfloat16* __restrict__ x, __nv_bfloat16* __restrict__ xn,
                   int64_t T, int d, float eps) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int64_t row = (int64_t)blockIdx.x * (blockDim.x >> 5) + (threadIdx.x >> 5);
  if (row >= T) return;
  const __nv_bfloat16* xr = x + row * d;
  float ss = 0.f;
  for (int c0 = lane * 4; c0 < d; c0 += 128 * COMBINE_U) {
    float v[COMBINE_U][4];
#pragma unroll
    for (int u = 0; u < COMBINE_U; ++u)
      if (c0 + 128 * u < d) Out4<__nv_bfloat16>::load(xr + c0 + 128 * u, v[u]);
#pragma unroll
    for (int u = 0; u < COMBINE_U; ++u)
      if (c0 + 128 * u < d)
#pragma unroll
        for (int i = 0; i < 4; ++i) ss = fmaf(v[u][i], v[u][i], ss);
  }
  rms_scale_row(xr, xn + row * d, d, lane, rms_inv_from_sumsq(ss, d, eps));
}

cudaError_t launch_rmsnorm(const void* x, void* xn, int64_t T, int64_t d, float eps,
                           cudaStream_t s) {
  const unsigned blocks = (unsigned)((T + 7) / 8);
  pdl(rmsnorm_kernel, blocks, 256, 0, s)(static_cast<const __nv_bfloat16*>(x),
                                        static_cast<__nv_bfloat16*>(xn), T, (int)d, eps);
  return cudaGetLastError();
}

}  // namespace moe
