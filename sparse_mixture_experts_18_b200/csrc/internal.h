// internal.h -- host-side plan, workspace carving and kernel launchers shared by the
// library's translation units.  Not part of the public ABI (see include/moe.h).
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include <utility>

#include "common.cuh"

namespace moe {

constexpr int TILE_M = 128;       // rows of one tensor-core accumulator tile
constexpr int SIMT_TILE = 64;     // rows of one fp32 SIMT tile
constexpr int MID_TOK_MAX = 256;  // mid-size tiling: most rows of an expert per pass (MMA N)
constexpr int MID_BOX = 64;       // mid-size tiling: rows of one TMA box of B rows
constexpr int MAX_EXPERTS = 64;
constexpr int SMALL_ROUTE_MAX_ROWS = 1024;  // T*K limit of the one-launch routing

// Everything about a forward call that depends only on its shape.
struct Plan {
  int64_t T = 0, d = 0, F = 0;
  int n = 0, K = 0;
  int dt = 1;              // 0 = fp32 (SIMT path), 1 = bf16 (tensor-core path)
  bool swap = false;       // small-batch path: weights are the MMA's 128-row operand
  bool pair = false;       // large batches: 256-row tiles on 2-CTA clusters (cta_group::2)
  bool mid = false;        // mid-size groups: weight-stationary tiles, an expert's rows (up to
                           // 256 per pass) as the MMA's N, SwiGLU fused into G13
  bool gather_x = false;   // pair path: G13 gathers its A rows from x by token (no X_perm),
                           // G2 applies the gates in its epilogue
  int row_align = 1;       // each expert's group is padded to a multiple of this
  int64_t rows_max = 0;    // upper bound of permuted rows (T*K plus padding)
  int64_t nblk = 0;        // router / permute blocks
  bool fused_route = false;  // small batch: routing in one launch (route_split_kernel)
  bool gather_small = false; // small batch (bf16, fused routing): G13 gathers its token rows
                             // from x (TMA gather4); routing writes no X_perm
  int tok_tile = 0;        // swap: MMA N (tokens per expert tile), multiple of 16; mid: rows
                           // of an expert per pass, multiple of MID_BOX
  int s13 = 1, s2 = 1;     // swap: split-K factors of the two expert GEMMs
  bool stack = false;      // workspace also holds the normalised activations
  bool fp8 = false;        // MXFP8 expert weights (small batch only)
  // failure-path test hook (moe_debug_forward_withheld only): the one-CTA G13 kernel issues
  // no loads and its pipeline waits give up after g13_wait_limit cycles
  bool g13_withhold = false;
  long long g13_wait_limit = 0;
  // workspace byte offsets
  size_t o_rpart;          // small batch: partial router logits [ceil(d/64)][T][n]
  size_t o_rowtok;         // token of each permuted row [rows_max] (small batch, gather_x)
  size_t o_rowgate;        // gather_x: gate of each permuted row [rows_max]
  size_t o_sx, o_sfx, o_sh;  // fp8 block scales: per token [T][d/128] words; per expert
                             // row slot for G13's B [n][d/128][512 B] and G2's B [n][F/128][512 B]
  size_t o_wparts;         // tensor-core router: W_g as three bf16 parts [3n padded][d]
  size_t o_status, o_idx, o_gate, o_blk_counts, o_blk_base, o_counts, o_offsets, o_inv,
      o_xperm, o_h, o_y, o_p13, o_xn, total;
};

// Device pointers into the workspace.
struct Workspace {
  uint32_t* status;
  unsigned int* ticket;  // small-batch routing: CTAs finished (in the status header, starts 0)
  unsigned int* scan_ticket;  // routing scan: expert CTAs finished (status header, starts 0)
  float* rpart;          // small-batch routing: partial logits
  int32_t* row_tok;      // token of each permuted row (small batch, gather_x)
  float* row_gate;       // gather_x: gate of each permuted row
  uint32_t* sxw;         // fp8: each token's block-scale words [T][d / 128]
  uint32_t* sfx;         // fp8: the token rows' scales by expert row slot (G13 B operand)
  uint32_t* sfh;         // fp8: the h rows' scales by expert row slot (G2 B operand)
  __nv_bfloat16* wparts; // tensor-core router: the W_g parts
  int32_t *idx, *blk_counts, *blk_base, *counts, *offsets, *inv;
  float* gate;
  void* xperm;  // [rows_max][d] activations in permuted order
  void* h;      // [rows_max][F] silu(a) * b (bf16 on the tensor-core path, fp32 on SIMT)
  float* y;     // [s2][rows_max][d] expert outputs (per split on the swap path)
  float* p13;   // swap: [s13][rows_max][2F] split-K partial sums of x.W1 | x.W3
  void* xn;     // stack: normalised activations [T][d]
};

// Launch with programmatic stream serialization (the kernel may begin while its predecessor
// in the stream finishes; see pdl_wait / pdl_trigger):  pdl(kernel, grid, block, smem, s)(args)
template <typename... KArgs>
struct PdlLaunch {
  void (*kern)(KArgs...);
  dim3 grid, block;
  size_t smem;
  cudaStream_t stream;
  template <typename... Args>
  cudaError_t operator()(Args&&... args) const {
    cudaLaunchConfig_t cfg = {};
    cfg.gridDim = grid;
    cfg.blockDim = block;
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[1];
    attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[0].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 1;
    return cudaLaunchKernelEx(&cfg, kern, std::forward<Args>(args)...);
  }
};
template <typename... KArgs>
PdlLaunch<KArgs...> pdl(void (*kern)(KArgs...), dim3 grid, dim3 block, size_t smem,
                        cudaStream_t s) {
  return PdlLaunch<KArgs...>{kern, grid, block, smem, s};
}

// route_only: the plan of moe_route (routing and unpadded grouping into a caller buffer; no
// expert stages, F unused).
bool make_plan(int64_t T, int64_t d, int64_t F, int n, int K, int dt, bool stack, Plan* p,
               bool fp8 = false, bool route_only = false);
Workspace carve(const Plan& p, void* base);

int route_tokens_per_block(int K);
// The router of large batches on the tensor cores (route_tc.cu): taken for bf16, T >= 1024,
// n <= 64, K <= 8; writes idx, gate and the 8-token block histograms like the CUDA-core
// router.
bool router_tc_applies(const Plan& p);
size_t router_tc_parts_bytes(int64_t d, int n);
cudaError_t launch_router_tc(const Plan& p, const void* x, const float* Wg, const Workspace& w,
                             cudaStream_t s);
// 2-D bf16 tensor map [outer][inner], box box_rows x 64 elements, 128-byte swizzle.
bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                   uint32_t box_rows);
cudaError_t launch_route(const Plan& p, const void* x, const float* Wg, const Workspace& w,
                         cudaStream_t s);
// ev (may be null): events recorded after G13, after the split-K reduction, after G2.
cudaError_t launch_expert_gemms_tc(const Plan& p, const void* x, const void* W1,
                                   const void* W3, const void* W2, const Workspace& w,
                                   cudaStream_t s, cudaEvent_t const* ev = nullptr);
// fp8: the small-batch GEMMs on MXFP8 codes; W1q/W3q [n][F][d], W2q [n][d][F] E4M3 codes;
// sf1/sf3/sf2 their E8M0 block scales in the tile order of launch_quantize_mx_e4m3.  ev as
// for launch_expert_gemms_tc.
cudaError_t launch_expert_gemms_e4m3(const Plan& p, const uint8_t* W1q, const uint8_t* W3q,
                                     const uint8_t* W2q, const uint8_t* sf1,
                                     const uint8_t* sf3, const uint8_t* sf2, const Workspace& w,
                                     cudaStream_t s, cudaEvent_t const* ev);
// MXFP8 quantisation of [rows][cols] bf16 (multiples of 128): codes and block scales in the
// GEMMs' tile order.
cudaError_t launch_quantize_mx_e4m3(const void* v, int64_t rows, int64_t cols, uint8_t* q,
                                    uint8_t* sf, cudaStream_t s);
cudaError_t launch_expert_gemms_simt(const Plan& p, const float* W1, const float* W3,
                                     const float* W2, const Workspace& w, cudaStream_t s,
                                     cudaEvent_t const* ev = nullptr);
// fp8 (p.fp8): s2 [n][d] are the W2 row scales; expert outputs are scaled by s_h[row] s2[e][i]
// norm_out (may be null; bf16 with a residual): when the large-batch K = 2 combine applies,
// it also writes the RMSNorm (unit gain, eps) of every result row there -- the next stacked
// block's input -- and sets *normed; otherwise the caller runs launch_rmsnorm.
cudaError_t launch_combine(const Plan& p, const Workspace& w, void* out, const void* resid,
                           cudaStream_t s, void* norm_out = nullptr, float eps = 0.f,
                           bool* normed = nullptr);
// out[t] = (resid[t] +) sum_k gate[t][k] * sum_{s < S} Y[s * split_stride + inv[t][k] row]
// (gate null: weight 1), fp32 sums in split then slot order, rounded once to bf16, or kept
// fp32 (out_f32).
cudaError_t launch_combine_rows(const float* Y, int S, int64_t split_stride, int64_t T, int d,
                                int K, const int32_t* inv, const float* gate, void* out,
                                const void* resid, bool out_f32, cudaStream_t s);
// Expert-parallel local stage: rows received from S sources, each source's rows grouped by
// the nl local experts (seg_counts [S][nl] on the device), are placed in the padded
// per-expert layout of the plan (X_perm, counts, offsets, inv = padded row of each row).
cudaError_t launch_ep_regroup(const Plan& p, const void* x_rows, const int32_t* seg_counts,
                              int S, const Workspace& w, cudaStream_t s);
// out[i] = in[index[i]], rows of row_bytes (a multiple of 16) bytes; indices outside
// [0, in_rows) leave their row unwritten.
cudaError_t launch_gather_rows(const void* in, int64_t in_rows, const int32_t* index,
                               int64_t rows, int64_t row_bytes, void* out, cudaStream_t s);
cudaError_t launch_rmsnorm(const void* x, void* xn, int64_t T, int64_t d, float eps,
                           cudaStream_t s);
int num_sms();

// Raise kernel `kern`'s dynamic shared-memory limit to at least `smem` bytes on the current
// device; `configured` is the caller's per-device record for that kernel instance (a repeated
// or concurrent first call only sets the attribute again).
constexpr int MAX_DEVICES = 64;
template <typename Kern>
cudaError_t ensure_dynamic_smem(Kern kern, size_t smem, int (&configured)[MAX_DEVICES]) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const bool tracked = dev >= 0 && dev < MAX_DEVICES;
  if (tracked && configured[dev] >= (int)smem) return cudaSuccess;
  e = cudaFuncSetAttribute(kern, cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
  if (e == cudaSuccess && tracked) configured[dev] = (int)smem;
  return e;
}

}  // namespace moe
