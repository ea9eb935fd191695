// gemm_simt.cu -- fp32 grouped expert GEMMs on the CUDA cores (IEEE fp32 FMA, no TF32), the
// path taken when x and the expert weights are fp32.  Same SwiGLU expert as the tensor-core
// path ("Mixtral of Experts", method section and glossary):
//   G13:  h = silu(X_e . W1_e^T) * (X_e . W3_e^T)          (fp32)
//   G2:   Y = h_e . W2_e^T                                 (fp32)
// 64x64 output tiles, 256 threads each computing 4x4 outputs, K staged through shared
// memory in chunks of 16.  Each expert's rows are padded to a multiple of 64 by the permute
// kernel, so a tile never mixes experts.
#include "internal.h"

namespace moe {

constexpr int SK = 16;

template <bool G13>
__global__ void __launch_bounds__(256)
    simt_grouped_gemm_kernel(const float* __restrict__ A, int64_t a_ld, int kdim,
                             const float* __restrict__ W0, const float* __restrict__ W1,
                             int nw, const int32_t* __restrict__ offsets, int n,
                             float* __restrict__ out, int64_t out_ld) {
  pdl_wait();
  pdl_trigger();
  __shared__ float As[SK][SIMT_TILE + 4];
  __shared__ float B0s[SK][SIMT_TILE + 4];
  __shared__ float B1s[SK][SIMT_TILE + 4];
  __shared__ int s_e, s_end;
  const int nt = blockIdx.x, mt = blockIdx.y;
  const int row0 = mt * SIMT_TILE;
  if (threadIdx.x == 0) {
    int e = -1;
    for (int i = 0; i < n; ++i)
      if (row0 >= offsets[i] && row0 < offsets[i + 1]) e = i;
    s_e = e;
    s_end = e >= 0 ? offsets[e + 1] : 0;
  }
  __syncthreads();
  const int e = s_e;
  if (e < 0) return;  // beyond the last expert's group
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  const int col0 = nt * SIMT_TILE;
  const float* w0 = W0 + (int64_t)e * nw * kdim;
  const float* w1 = G13 ? W1 + (int64_t)e * nw * kdim : nullptr;
  float acc0[4][4] = {}, acc1[4][4] = {};
  for (int k0 = 0; k0 < kdim; k0 += SK) {
    for (int i = threadIdx.x; i < SIMT_TILE * SK; i += 256) {
      const int rr = i / SK, kk = i % SK;
      const int k = k0 + kk;
      const int ar = row0 + rr, wc = col0 + rr;
      As[kk][rr] = (k < kdim && ar < s_end) ? A[(int64_t)ar * a_ld + k] : 0.f;
      B0s[kk][rr] = (k < kdim && wc < nw) ? w0[(int64_t)wc * kdim + k] : 0.f;
      if (G13) B1s[kk][rr] = (k < kdim && wc < nw) ? w1[(int64_t)wc * kdim + k] : 0.f;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float a[4], b0[4], b1[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        a[i] = As[kk][ty * 4 + i];
        b0[i] = B0s[kk][tx * 4 + i];
        if (G13) b1[i] = B1s[kk][tx * 4 + i];
      }
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          acc0[i][j] = fmaf(a[i], b0[j], acc0[i][j]);
          if (G13) acc1[i][j] = fmaf(a[i], b1[j], acc1[i][j]);
        }
    }
    __syncthreads();
  }
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int r = row0 + ty * 4 + i;
    if (r >= s_end) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col = col0 + tx * 4 + j;
      if (col >= nw) continue;
      out[(int64_t)r * out_ld + col] = G13 ? silu(acc0[i][j]) * acc1[i][j] : acc0[i][j];
    }
  }
}

cudaError_t launch_expert_gemms_simt(const Plan& p, const float* W1, const float* W3,
                                     const float* W2, const Workspace& w, cudaStream_t s,
                                     cudaEvent_t const* ev) {
  const int d = (int)p.d, F = (int)p.F;
  const unsigned mtiles = (unsigned)(p.rows_max / SIMT_TILE);
  dim3 g13((F + SIMT_TILE - 1) / SIMT_TILE, mtiles);
  pdl(simt_grouped_gemm_kernel<true>, g13, 256, 0, s)(static_cast<const float*>(w.xperm), d, d,
                                                      W1, W3, F, w.offsets, p.n,
                                                      static_cast<float*>(w.h), F);
  cudaError_t err = cudaGetLastError();
  if (err != cudaSuccess) return err;
  if (ev && ((err = cudaEventRecord(ev[0], s)) != cudaSuccess ||
             (err = cudaEventRecord(ev[1], s)) != cudaSuccess))
    return err;
  dim3 g2((d + SIMT_TILE - 1) / SIMT_TILE, mtiles);
  pdl(simt_grouped_gemm_kernel<false>, g2, 256, 0, s)(static_cast<const float*>(w.h), F, F, W2,
                                                      nullptr, d, w.offsets, p.n, w.y, d);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  return ev ? cudaEventRecord(ev[2], s) : cudaSuccess;
}

}  // namespace moe
