// quantize.cu -- MXFP8 quantisation of expert weights (done once per model, outside the
// forward): E4M3 codes in blocks of 32 consecutive elements of a row sharing an E8M0 scale X
// (mx_scale_code: the smallest power of two with max |v| <= 448 X), the scales written in the
// tile order the small-batch GEMMs' scale copies read.
#include "internal.h"

namespace moe {

// Weights: [rows][cols] bf16 -> codes q [rows][cols] and scales in the tile order the GEMMs
// read: the word of row r, K block kb at byte ((r / 128) * (cols / 128) + kb) * 512
// + 16 (r % 32) + 4 ((r % 128) / 32).  rows and cols multiples of 128.  One warp per 256
// columns of a row: lane c holds columns 8c .. 8c + 7 (one 16-byte load), so a 32-element
// block is 4 lanes and each half-warp one K block.
__global__ void __launch_bounds__(256)
    quantize_mx_e4m3_kernel(const __nv_bfloat16* __restrict__ v, int64_t rows, int64_t cols,
                            uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  const int lane = threadIdx.x & 31;
  const int64_t kbs = cols / 128, upr = (cols + 255) / 256;  // K blocks, warp units per row
  for (int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); gw < rows * upr;
       gw += (int64_t)gridDim.x * 8) {  // warp-uniform
    const int64_t r = gw / upr;
    const int64_t c = (gw % upr) * 256 + lane * 8;
    const bool in = c < cols;  // a whole half-warp (one K block) is in or out
    const uint4 raw = in ? __ldg(reinterpret_cast<const uint4*>(v + r * cols + c))
                         : make_uint4(0u, 0u, 0u, 0u);
    const float f[8] = {bf16_lo(raw.x), bf16_hi(raw.x), bf16_lo(raw.y), bf16_hi(raw.y),
                        bf16_lo(raw.z), bf16_hi(raw.z), bf16_lo(raw.w), bf16_hi(raw.w)};
    float amax = 0.f;
#pragma unroll
    for (int i = 0; i < 8; ++i) amax = fmaxf(amax, fabsf(f[i]));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
    amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
    const uint32_t code = mx_scale_code(amax);
    const float inv = mx_inv_scale(code);
    const int h = lane & 16;
    const uint32_t word = __shfl_sync(0xffffffffu, code, h) |
                          (__shfl_sync(0xffffffffu, code, h + 4) << 8) |
                          (__shfl_sync(0xffffffffu, code, h + 8) << 16) |
                          (__shfl_sync(0xffffffffu, code, h + 12) << 24);
    if (in) {
      *reinterpret_cast<uint2*>(q + r * cols + c) =
          make_uint2(e4m3x4_mul(f[0], f[1], f[2], f[3], inv),
                     e4m3x4_mul(f[4], f[5], f[6], f[7], inv));
      if ((lane & 15) == 0)
        *reinterpret_cast<uint32_t*>(sf + ((r / 128) * kbs + c / 128) * 512 + 16 * (r % 32) +
                                     4 * ((r % 128) / 32)) = word;
    }
  }
}

cudaError_t launch_quantize_mx_e4m3(const void* v, int64_t rows, int64_t cols, uint8_t* q,
                                    uint8_t* sf, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  const int64_t warps = rows * ((cols + 255) / 256);
  int64_t blocks = (warps + 7) / 8;
  if (blocks > 64 * (int64_t)num_sms()) blocks = 64 * (int64_t)num_sms();
  quantize_mx_e4m3_kernel<<<(unsigned)blocks, 256, 0, s>>>(
      static_cast<const __nv_bfloat16*>(v), rows, cols, q, sf);
  return cudaGetLastError();
}

}  // namespace moe
