// moe_api.cu -- the C ABI of libmoe.so (declared in include/moe.h): argument validation,
// the per-shape plan, workspace carving, and the kernel sequence of one MoE block forward:
//   router + TopK + softmax  ->  histogram scan  ->  permute / gather
//   ->  expert GEMMs (tensor cores for bf16, CUDA cores for fp32)  ->  gated combine.
#include <stdlib.h>
#include <string.h>

#include "../../include/moe.h"
#include "internal.h"

namespace moe {

int num_sms() {
  static int cached[64] = {0};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 148;
  if (!cached[dev]) {
    int v = 0;
    if (cudaDeviceGetAttribute(&v, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess || v <= 0)
      v = 148;
    cached[dev] = v;
  }
  return cached[dev];
}

static size_t align256(size_t v) { return (v + 255) & ~(size_t)255; }

// Smallest split of `num_kb` K-blocks (a divisor, at least 4 blocks per split, at most 16
// splits) for which `units_per_split` * splits work units fill whole waves of the SMs to
// within 5%; otherwise the best fill found.
static int choose_split(int num_kb, int units_per_split, int sms) {
  int best = 1;
  double best_eff = 0.0;
  for (int s = 1; s <= 16; ++s) {
    if (num_kb % s || num_kb / s < 4 || s > 8) continue;  // the combine unrolls <= 8 splits
    const double u = (double)units_per_split * s;
    const double waves = u / sms;
    const double eff = waves / (double)((int64_t)((u + sms - 1) / sms));
    if (eff >= 0.95) return s;
    if (eff > best_eff + 1e-9) { best_eff = eff; best = s; }
  }
  return best;
}

// The CTA-pair path's alternative data path (MOE_GATHER_X=1 in the environment, read at
// every call): G13 gathers its A rows from x by token with TMA tile::gather4 instead of
// reading X_perm, and G2 applies the gates in its epilogue.  Off by default: on B200 the
// 512-byte gathers starve the tensor cores (G13 2.3x slower at T = 4096), which costs far
// more than the X_perm pass it saves.
static bool gather_x_requested() {
  const char* v = getenv("MOE_GATHER_X");
  return v != nullptr && v[0] == '1';
}

// Mid-size tiling: rows per pass.  A pass's stage holds its rows' K block beside the weight
// tiles, so the pass is sized to what most experts have rather than to the largest possible
// group: the mean M_e = T*K/n plus 2.5 standard deviations of a uniform routing (sqrt(M_e)),
// in whole 64-row TMA boxes (32-row boxes measured up to 10% slower on the down projection).
// A larger expert takes a second pass over the same weight block.
static int mid_pass_rows(int64_t P, int n) {
  const int64_t mean = (P + n - 1) / n;
  int64_t r = mean;
  int64_t s = 0;
  while ((s + 1) * (s + 1) <= mean) ++s;  // floor(sqrt(mean))
  r += (5 * s + 1) / 2;
  r = (r + MID_BOX - 1) / MID_BOX * MID_BOX;
  return (int)(r > MID_TOK_MAX ? MID_TOK_MAX : r);
}

bool make_plan(int64_t T, int64_t d, int64_t F, int n, int K, int dt, bool stack, Plan* p,
               bool fp8, bool route_only) {
  if (T < 0 || d <= 0 || F <= 0 || n < 1 || n > MAX_EXPERTS || K < 1 || K > n) return false;
  if (fp8 && (dt != 1 || stack || d % 128 || F % 128)) return false;
  if (dt == 1) {
    if (d % 64 || F % 64) return false;
  } else if (dt == 0) {
    if (d % 8 || F % 8) return false;
  } else {
    return false;
  }
  if (d > (1 << 20) || F > (1 << 20) || T > (int64_t)1 << 26) return false;
  Plan q;
  q.T = T; q.d = d; q.F = F; q.n = n; q.K = K; q.dt = dt; q.stack = stack;
  q.swap = dt == 1 && T <= 256 && T * K < 64 * (int64_t)n;
  // CTA pairs (256-row tiles, 128-row tails) from about 80 rows per expert on.
  q.pair = dt == 1 && !q.swap && T * K >= 640 * (int64_t)n;
  // Mid-size groups (at most 160 rows per expert on average): each CTA keeps a 128-row block
  // of the expert's weights as the MMA's M and takes the expert's rows (up to 192 per pass at
  // this mean) as N, so the weights stream once per pass instead of once per 128-row tile.
  // Above it passes grow to 256 rows, whose W1 and W3 accumulators fill TMEM (no overlap of
  // a pass's epilogue with the next) in three stages: the 128-row tiles were faster from a
  // mean of 192 rows on (n = 16, K = 1: 1489 against 1559 us per block), the mid-size tiles
  // at 160 (1271 against 1385 us).
  q.mid = dt == 1 && !q.swap && !q.pair && T * K <= 160 * (int64_t)n;
  q.row_align = dt == 0 ? SIMT_TILE : (q.swap || q.mid ? 1 : TILE_M);
  q.gather_x = q.pair && gather_x_requested();
  if (route_only) {  // experts' rows contiguous and unpadded, in the caller's buffer
    q.swap = q.pair = q.mid = q.gather_x = false;
    q.row_align = 1;
  }
  const int64_t P = T * K;
  q.rows_max = (P + (int64_t)n * (q.row_align - 1) + q.row_align - 1) / q.row_align * q.row_align;
  if (q.swap) q.rows_max = (P + 31) / 32 * 32;  // >= tok_tile rows for the token TMA box
  if (q.mid) {
    q.tok_tile = mid_pass_rows(P, n);
    q.rows_max = (P + MID_BOX - 1) / MID_BOX * MID_BOX;  // whole boxes of B rows
  }
  if (q.rows_max >= ((int64_t)1 << 31) / 2) return false;
  const int tokb = route_tokens_per_block(K);
  q.nblk = (T + tokb - 1) / tokb;
  q.fused_route = T <= 64 && T * K <= 1024;  // limits of route_split_kernel
  // FP8 expert weights: the small-batch path with its one-launch routing only
  q.fp8 = fp8;
  if (fp8 && !(q.swap && q.fused_route)) return false;
  q.gather_small = q.swap && q.fused_route && dt == 1;  // (FP8: from the quantised rows)
  if (route_only) q.rows_max = P;
  const int kbw = fp8 ? 128 : 64;  // elements per 128-byte K block
  if (q.swap) {
    // (fp8: a multiple of 32, the granularity of the B operand's block scales in TMEM)
    q.tok_tile = fp8 ? (int)((T + 31) / 32 * 32) : (int)((T + 15) / 16 * 16);
    const int sms = num_sms();
    q.s13 = choose_split((int)(d / kbw), n * (int)((F + 127) / 128), sms);
    q.s2 = choose_split((int)(F / kbw), n * (int)((d + 127) / 128), sms);
  }
  const size_t es = dt == 1 ? 2 : 4;
  size_t o = 0;
  auto take = [&](size_t bytes) { const size_t at = o; o = align256(o + bytes); return at; };
  q.o_status = take(256);
  q.o_idx = take((size_t)P * 4);
  q.o_gate = take((size_t)P * 4);
  q.o_blk_counts = take((size_t)q.nblk * n * 4);
  q.o_blk_base = take((size_t)q.nblk * n * 4);
  q.o_counts = take((size_t)n * 4);
  q.o_offsets = take((size_t)(n + 1) * 4);
  q.o_inv = take((size_t)P * 4);
  q.o_xperm = take(route_only ? 0 : (size_t)q.rows_max * d * es);
  q.o_h = take(route_only ? 0 : (size_t)q.rows_max * F * es);
  q.o_y = take(route_only ? 0 : (size_t)(q.swap ? q.s2 : 1) * q.rows_max * d * 4);
  q.o_p13 = take(q.swap ? (size_t)q.s13 * q.rows_max * 2 * F * 4 : 0);
  q.o_xn = take(stack ? (size_t)T * d * es : 0);
  q.o_rpart = take(q.fused_route ? (size_t)((d + 63) / 64) * T * n * 4 : 0);
  // (the layout does not depend on gather_x, so a workspace sized earlier stays valid)
  q.o_rowtok = take(q.fused_route || q.pair ? (size_t)q.rows_max * 4 : 0);
  q.o_rowgate = take(q.pair ? (size_t)q.rows_max * 4 : 0);
  // fp8: X_perm holds each token's E4M3 row (by token) and h the E4M3 rows; block scales
  q.o_sx = take(fp8 ? (size_t)T * (d / 128) * 4 : 0);
  q.o_sfx = take(fp8 ? (size_t)n * (d / 128) * 512 : 0);
  q.o_sh = take(fp8 ? (size_t)n * (F / 128) * 512 : 0);
  q.o_wparts = take(router_tc_applies(q) ? router_tc_parts_bytes(d, n) : 0);
  q.total = o;
  *p = q;
  return true;
}

Workspace carve(const Plan& p, void* base) {
  uint8_t* b = static_cast<uint8_t*>(base);
  Workspace w;
  w.status = reinterpret_cast<uint32_t*>(b + p.o_status);
  w.ticket = reinterpret_cast<unsigned int*>(b + p.o_status + 64);
  w.scan_ticket = reinterpret_cast<unsigned int*>(b + p.o_status + 128);
  w.rpart = reinterpret_cast<float*>(b + p.o_rpart);
  w.row_tok = reinterpret_cast<int32_t*>(b + p.o_rowtok);
  w.row_gate = reinterpret_cast<float*>(b + p.o_rowgate);
  w.sxw = reinterpret_cast<uint32_t*>(b + p.o_sx);
  w.sfx = reinterpret_cast<uint32_t*>(b + p.o_sfx);
  w.sfh = reinterpret_cast<uint32_t*>(b + p.o_sh);
  w.wparts = reinterpret_cast<__nv_bfloat16*>(b + p.o_wparts);
  w.idx = reinterpret_cast<int32_t*>(b + p.o_idx);
  w.gate = reinterpret_cast<float*>(b + p.o_gate);
  w.blk_counts = reinterpret_cast<int32_t*>(b + p.o_blk_counts);
  w.blk_base = reinterpret_cast<int32_t*>(b + p.o_blk_base);
  w.counts = reinterpret_cast<int32_t*>(b + p.o_counts);
  w.offsets = reinterpret_cast<int32_t*>(b + p.o_offsets);
  w.inv = reinterpret_cast<int32_t*>(b + p.o_inv);
  w.xperm = b + p.o_xperm;
  w.h = b + p.o_h;
  w.y = reinterpret_cast<float*>(b + p.o_y);
  w.p13 = reinterpret_cast<float*>(b + p.o_p13);
  w.xn = b + p.o_xn;
  return w;
}

static bool aligned(const void* ptr, size_t a) {
  return (reinterpret_cast<uintptr_t>(ptr) & (a - 1)) == 0;
}

static moe_status check_common(const void* x, const float* W_g, const void* W1, const void* W3,
                               const void* W2, const void* out, const void* ws) {
  if (!x || !W_g || !W1 || !W3 || !W2 || !out || !ws) return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(W_g, 16) || !aligned(W1, 16) || !aligned(W3, 16) ||
      !aligned(W2, 16) || !aligned(out, 16) || !aligned(ws, 256))
    return MOE_ERR_INVALID_ARG;
  return MOE_OK;
}

static moe_status shape_status(int64_t T, int64_t d, int64_t F, int n, int K, int dt) {
  if (T < 0 || d <= 0 || F <= 0 || n < 1 || K < 1 || K > n) return MOE_ERR_INVALID_ARG;
  if (dt != 0 && dt != 1) return MOE_ERR_INVALID_ARG;
  return MOE_ERR_UNSUPPORTED;
}

// The kernel sequence of one block on already-validated arguments.
// ev (may be null): six events recorded at the stage boundaries (see moe_forward_profiled).
// norm_out (stacked blocks): where the combine may also write the next block's RMSNorm input
// (*normed tells whether it did; see launch_combine).
static moe_status forward_impl(const Plan& p, const void* x, const float* W_g, const void* W1,
                               const void* W3, const void* W2, void* out, const void* resid,
                               const Workspace& w, cudaStream_t s,
                               cudaEvent_t const* ev = nullptr, void* norm_out = nullptr,
                               float eps = 0.f, bool* normed = nullptr) {
  if (ev && cudaEventRecord(ev[0], s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_route(p, x, W_g, w, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (ev && cudaEventRecord(ev[1], s) != cudaSuccess) return MOE_ERR_CUDA;
  cudaError_t err =
      p.dt == 1 ? launch_expert_gemms_tc(p, x, W1, W3, W2, w, s, ev ? ev + 2 : nullptr)
                : launch_expert_gemms_simt(p, static_cast<const float*>(W1),
                                           static_cast<const float*>(W3),
                                           static_cast<const float*>(W2), w, s,
                                           ev ? ev + 2 : nullptr);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_combine(p, w, out, resid, s, norm_out, eps, normed) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (ev && cudaEventRecord(ev[5], s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

}  // namespace moe

using namespace moe;

extern "C" {

int moe_abi_version(void) { return 3; }

const char* moe_status_string(moe_status s) {
  switch (s) {
    case MOE_OK: return "ok";
    case MOE_ERR_INVALID_ARG: return "invalid argument (null, misaligned or bad size)";
    case MOE_ERR_UNSUPPORTED: return "unsupported shape";
    case MOE_ERR_WORKSPACE: return "workspace too small";
    case MOE_ERR_CUDA: return "CUDA error";
    case MOE_ERR_TIMEOUT: return "a kernel's bounded wait ran out";
    case MOE_ERR_DEVICE: return "a kernel detected an out-of-range index";
  }
  return "unknown status";
}

size_t moe_workspace_bytes(int64_t T, int64_t d, int64_t F, int n, int K, moe_dtype dt) {
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, false, &p)) return 0;
  return p.total;
}

size_t moe_stack_workspace_bytes(int64_t T, int64_t d, int64_t F, int n, int K, moe_dtype dt) {
  Plan p;
  if (dt != MOE_BF16 || !make_plan(T, d, F, n, K, (int)dt, true, &p)) return 0;
  return p.total;
}

moe_status moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream) {
  if (!workspace || workspace_bytes < 256 || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  if (cudaMemsetAsync(workspace, 0, 256, static_cast<cudaStream_t>(stream)) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_workspace_status(void* workspace, void* stream, uint32_t* raw) {
  if (!workspace || !aligned(workspace, 256)) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  uint32_t bits = 0;
  if (cudaStreamSynchronize(s) != cudaSuccess) return MOE_ERR_CUDA;
  if (cudaMemcpyAsync(&bits, workspace, sizeof bits, cudaMemcpyDeviceToHost, s) != cudaSuccess ||
      cudaStreamSynchronize(s) != cudaSuccess)
    return MOE_ERR_CUDA;
  // cleared on the same stream, so the next call enqueued there sees zero
  if (bits && cudaMemsetAsync(workspace, 0, sizeof bits, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (raw) *raw = bits;
  if (bits & DEV_ERR_TIMEOUT) return MOE_ERR_TIMEOUT;
  if (bits) return MOE_ERR_DEVICE;
  return MOE_OK;
}

moe_status moe_forward(const void* x, const float* W_g, const void* W1, const void* W3,
                       const void* W2, int64_t T, int64_t d, int64_t F, int n, int K,
                       moe_dtype dt, void* out, void* workspace, size_t workspace_bytes,
                       void* stream) {
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, false, &p)) return shape_status(T, d, F, n, K, dt);
  if (T == 0) return MOE_OK;
  moe_status st = check_common(x, W_g, W1, W3, W2, out, workspace);
  if (st != MOE_OK) return st;
  if (out == x) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  const Workspace w = carve(p, workspace);
  return forward_impl(p, x, W_g, W1, W3, W2, out, nullptr, w, static_cast<cudaStream_t>(stream));
}

size_t moe_workspace_bytes_fp8(int64_t T, int64_t d, int64_t F, int n, int K) {
  Plan p;
  if (!make_plan(T, d, F, n, K, 1, false, &p, true)) return 0;
  return p.total;
}

moe_status moe_quantize_mx_e4m3(const void* v, int64_t rows, int64_t cols, uint8_t* q,
                                uint8_t* sf, void* stream) {
  if (rows < 0 || cols <= 0 || rows % 128 || cols % 128) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!v || !q || !sf || !aligned(v, 8) || !aligned(q, 4) || !aligned(sf, 16))
    return MOE_ERR_INVALID_ARG;
  if (rows > ((int64_t)1 << 31) - 1 || cols > ((int64_t)1 << 20)) return MOE_ERR_UNSUPPORTED;
  return launch_quantize_mx_e4m3(v, rows, cols, q, sf, static_cast<cudaStream_t>(stream)) ==
                 cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_forward_fp8(const void* x, const float* W_g, const uint8_t* W1q,
                           const uint8_t* W3q, const uint8_t* W2q, const uint8_t* sf1,
                           const uint8_t* sf3, const uint8_t* sf2, int64_t T, int64_t d, int64_t F,
                           int n, int K, void* out, void* workspace, size_t workspace_bytes,
                           void* stream, void* const* events, int n_events) {
  Plan p;
  if (!make_plan(T, d, F, n, K, 1, false, &p, true)) {
    const moe_status st = shape_status(T, d, F, n, K, MOE_BF16);
    return st == MOE_ERR_INVALID_ARG ? st : MOE_ERR_UNSUPPORTED;
  }
  if (n_events != 0 && (n_events != 6 || !events)) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  moe_status st = check_common(x, W_g, W1q, W3q, W2q, out, workspace);
  if (st != MOE_OK) return st;
  if (!sf1 || !sf3 || !sf2 || !aligned(sf1, 16) || !aligned(sf3, 16) || !aligned(sf2, 16))
    return MOE_ERR_INVALID_ARG;
  if (out == x) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  const Workspace w = carve(p, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  cudaEvent_t ev[6];
  for (int i = 0; i < n_events; ++i) ev[i] = static_cast<cudaEvent_t>(events[i]);
  cudaEvent_t const* evp = n_events ? ev : nullptr;
  if (evp && cudaEventRecord(ev[0], s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_route(p, x, W_g, w, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (evp && cudaEventRecord(ev[1], s) != cudaSuccess) return MOE_ERR_CUDA;
  if (launch_expert_gemms_e4m3(p, W1q, W3q, W2q, sf1, sf3, sf2, w, s,
                               evp ? ev + 2 : nullptr) != cudaSuccess)
    return MOE_ERR_CUDA;
  if (launch_combine(p, w, out, nullptr, s) != cudaSuccess) return MOE_ERR_CUDA;
  if (evp && cudaEventRecord(ev[5], s) != cudaSuccess) return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_forward_profiled(const void* x, const float* W_g, const void* W1,
                                const void* W3, const void* W2, int64_t T, int64_t d, int64_t F,
                                int n, int K, moe_dtype dt, void* out, void* workspace,
                                size_t workspace_bytes, void* stream, void* const* events,
                                int n_events) {
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, false, &p)) return shape_status(T, d, F, n, K, dt);
  if (!events || n_events != 6) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < 6; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  if (T == 0) return MOE_OK;
  moe_status st = check_common(x, W_g, W1, W3, W2, out, workspace);
  if (st != MOE_OK) return st;
  if (out == x) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  const Workspace w = carve(p, workspace);
  cudaEvent_t ev[6];
  for (int i = 0; i < 6; ++i) ev[i] = static_cast<cudaEvent_t>(events[i]);
  return forward_impl(p, x, W_g, W1, W3, W2, out, nullptr, w, static_cast<cudaStream_t>(stream),
                      ev);
}

moe_status moe_plan_info(int64_t T, int64_t d, int64_t F, int n, int K, moe_dtype dt,
                         int* small_batch, int* split13, int* split2, int* launches,
                         int* tiling) {
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, false, &p)) return shape_status(T, d, F, n, K, dt);
  if (small_batch) *small_batch = p.swap ? 1 : 0;
  if (split13) *split13 = p.swap ? p.s13 : 1;
  if (split2) *split2 = p.swap ? p.s2 : 1;
  if (launches)
    *launches = T == 0 ? 0
                       : (p.fused_route ? 1 : 3) + (router_tc_applies(p) ? 1 : 0) +
                             (p.swap ? 3 : 2) + 1;
  if (tiling) *tiling = p.pair ? 1 : p.mid ? 2 : 0;
  return MOE_OK;
}

moe_status moe_forward_debug(const void* x, const float* W_g, const void* W1, const void* W3,
                             const void* W2, int64_t T, int64_t d, int64_t F, int n, int K,
                             moe_dtype dt, void* out, void* workspace, size_t workspace_bytes,
                             void* stream, int32_t* topk_idx, float* topk_gate,
                             int32_t* expert_counts, int32_t* expert_offsets,
                             int32_t* token_rows) {
  moe_status st = moe_forward(x, W_g, W1, W3, W2, T, d, F, n, K, dt, out, workspace,
                              workspace_bytes, stream);
  if (st != MOE_OK || T == 0) return st;
  Plan p;
  make_plan(T, d, F, n, K, (int)dt, false, &p);
  const Workspace w = carve(p, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t tk = (size_t)T * K * 4;
  struct { void* dst; const void* src; size_t bytes; } cp[5] = {
      {topk_idx, w.idx, tk}, {topk_gate, w.gate, tk}, {expert_counts, w.counts, (size_t)n * 4},
      {expert_offsets, w.offsets, (size_t)(n + 1) * 4}, {token_rows, w.inv, tk}};
  for (auto& c : cp)
    if (c.dst && cudaMemcpyAsync(c.dst, c.src, c.bytes, cudaMemcpyDeviceToDevice, s) != cudaSuccess)
      return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_forward_host_io(const void* x_host, void* x_dev, const float* W_g,
                               const void* W1, const void* W3, const void* W2, int64_t T,
                               int64_t d, int64_t F, int n, int K, moe_dtype dt,
                               void* out_dev, void* out_host, void* workspace,
                               size_t workspace_bytes, void* stream) {
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, false, &p)) return shape_status(T, d, F, n, K, dt);
  if (T == 0) return MOE_OK;
  if (!x_host || !out_host) return MOE_ERR_INVALID_ARG;
  moe_status st = check_common(x_dev, W_g, W1, W3, W2, out_dev, workspace);
  if (st != MOE_OK) return st;
  if (out_dev == x_dev) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)T * d * (dt == MOE_BF16 ? 2 : 4);
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  const Workspace w = carve(p, workspace);
  st = forward_impl(p, x_dev, W_g, W1, W3, W2, out_dev, nullptr, w, s);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(out_host, out_dev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// Validation shared by the stack entry points (bf16 only; x is updated in place).
static moe_status stack_check(const Plan& p, const void* x, const float* const* W_g,
                              const void* const* W1, const void* const* W3,
                              const void* const* W2, int L, float eps, size_t workspace_bytes,
                              const void* workspace) {
  if (L < 0 || !W_g || !W1 || !W3 || !W2 || !(eps >= 0.f)) return MOE_ERR_INVALID_ARG;
  if (p.T == 0 || L == 0) return MOE_OK;
  for (int l = 0; l < L; ++l) {
    moe_status st = check_common(x, W_g[l], W1[l], W3[l], W2[l], x, workspace);
    if (st != MOE_OK) return st;
  }
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  return MOE_OK;
}

// L blocks in place on x; ev (may be null): 6 events per block, as moe_forward_profiled.
static moe_status stack_impl(const Plan& p, void* x, const float* const* W_g,
                             const void* const* W1, const void* const* W3,
                             const void* const* W2, int L, float eps, void* workspace,
                             cudaStream_t s, cudaEvent_t const* ev) {
  const Workspace w = carve(p, workspace);
  bool have_xn = false;  // the previous block's combine already wrote this block's input
  for (int l = 0; l < L; ++l) {
    if (!have_xn && launch_rmsnorm(x, w.xn, p.T, p.d, eps, s) != cudaSuccess)
      return MOE_ERR_CUDA;
    moe_status st = forward_impl(p, w.xn, W_g[l], W1[l], W3[l], W2[l], x, x, w, s,
                                 ev ? ev + 6 * (size_t)l : nullptr,
                                 l + 1 < L ? w.xn : nullptr, eps, &have_xn);
    if (st != MOE_OK) return st;
  }
  return MOE_OK;
}

moe_status moe_stack_forward(void* x, const float* const* W_g, const void* const* W1,
                             const void* const* W3, const void* const* W2, int L, int64_t T,
                             int64_t d, int64_t F, int n, int K, moe_dtype dt, float eps,
                             void* workspace, size_t workspace_bytes, void* stream) {
  if (dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, true, &p)) return shape_status(T, d, F, n, K, dt);
  moe_status st = stack_check(p, x, W_g, W1, W3, W2, L, eps, workspace_bytes, workspace);
  if (st != MOE_OK || T == 0 || L == 0) return st;
  return stack_impl(p, x, W_g, W1, W3, W2, L, eps, workspace,
                    static_cast<cudaStream_t>(stream), nullptr);
}

moe_status moe_stack_forward_profiled(void* x, const float* const* W_g, const void* const* W1,
                                      const void* const* W3, const void* const* W2, int L,
                                      int64_t T, int64_t d, int64_t F, int n, int K,
                                      moe_dtype dt, float eps, void* workspace,
                                      size_t workspace_bytes, void* stream,
                                      void* const* events, int n_events) {
  if (dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, true, &p)) return shape_status(T, d, F, n, K, dt);
  if (L < 0 || n_events != 6 * L || (L > 0 && !events)) return MOE_ERR_INVALID_ARG;
  for (int i = 0; i < n_events; ++i)
    if (!events[i]) return MOE_ERR_INVALID_ARG;
  moe_status st = stack_check(p, x, W_g, W1, W3, W2, L, eps, workspace_bytes, workspace);
  if (st != MOE_OK || T == 0 || L == 0) return st;
  return stack_impl(p, x, W_g, W1, W3, W2, L, eps, workspace,
                    static_cast<cudaStream_t>(stream),
                    reinterpret_cast<cudaEvent_t const*>(events));
}

moe_status moe_stack_forward_host_io(const void* x_host, void* x_dev, const float* const* W_g,
                                     const void* const* W1, const void* const* W3,
                                     const void* const* W2, int L, int64_t T, int64_t d,
                                     int64_t F, int n, int K, moe_dtype dt, float eps,
                                     void* out_host, void* workspace, size_t workspace_bytes,
                                     void* stream) {
  if (dt != MOE_BF16) return MOE_ERR_UNSUPPORTED;
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, true, &p)) return shape_status(T, d, F, n, K, dt);
  if (T > 0 && (!x_host || !out_host)) return MOE_ERR_INVALID_ARG;
  moe_status st = stack_check(p, x_dev, W_g, W1, W3, W2, L, eps, workspace_bytes, workspace);
  if (st != MOE_OK || T == 0) return st;
  if (!x_dev) return MOE_ERR_INVALID_ARG;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  const size_t bytes = (size_t)T * d * 2;
  if (cudaMemcpyAsync(x_dev, x_host, bytes, cudaMemcpyHostToDevice, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  st = stack_impl(p, x_dev, W_g, W1, W3, W2, L, eps, workspace, s, nullptr);
  if (st != MOE_OK) return st;
  if (cudaMemcpyAsync(out_host, x_dev, bytes, cudaMemcpyDeviceToHost, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

// ---------------------------------------------------------------- expert parallelism
size_t moe_route_workspace_bytes(int64_t T, int64_t d, int n, int K, moe_dtype dt) {
  Plan p;
  if (!make_plan(T, d, 64, n, K, (int)dt, false, &p, false, true)) return 0;
  return p.total;
}

moe_status moe_route(const void* x, const float* W_g, int64_t T, int64_t d, int n, int K,
                     moe_dtype dt, void* x_grouped, int32_t* topk_idx, float* topk_gate,
                     int32_t* expert_counts, int32_t* token_rows, void* workspace,
                     size_t workspace_bytes, void* stream) {
  Plan p;
  if (!make_plan(T, d, 64, n, K, (int)dt, false, &p, false, true))
    return shape_status(T, d, 64, n, K, dt);
  if (T == 0) return MOE_OK;
  if (!x || !W_g || !x_grouped || !topk_idx || !topk_gate || !expert_counts || !token_rows ||
      !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x, 16) || !aligned(W_g, 16) || !aligned(x_grouped, 16) || !aligned(workspace, 256) ||
      !aligned(topk_idx, 4) || !aligned(topk_gate, 4) || !aligned(expert_counts, 4) ||
      !aligned(token_rows, 4))
    return MOE_ERR_INVALID_ARG;
  if (x_grouped == x) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  Workspace w = carve(p, workspace);
  w.idx = topk_idx;
  w.gate = topk_gate;
  w.counts = expert_counts;
  w.inv = token_rows;
  w.xperm = x_grouped;
  return launch_route(p, x, W_g, w, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

size_t moe_experts_workspace_bytes(int64_t rows, int64_t d, int64_t F, int n_local,
                                   moe_dtype dt) {
  Plan p;
  if (!make_plan(rows, d, F, n_local, 1, (int)dt, false, &p)) return 0;
  return p.total;
}

moe_status moe_experts_forward(const void* x_rows, int64_t rows, const int32_t* seg_counts,
                               int S, const void* W1, const void* W3, const void* W2, int64_t d,
                               int64_t F, int n_local, moe_dtype dt, float* y_rows,
                               void* workspace, size_t workspace_bytes, void* stream) {
  Plan p;
  if (!make_plan(rows, d, F, n_local, 1, (int)dt, false, &p))
    return shape_status(rows, d, F, n_local, 1, dt);
  if (S < 1 || (int64_t)S * n_local > 2048) return MOE_ERR_INVALID_ARG;
  if (rows == 0) return MOE_OK;
  if (!x_rows || !seg_counts || !W1 || !W3 || !W2 || !y_rows || !workspace)
    return MOE_ERR_INVALID_ARG;
  if (!aligned(x_rows, 16) || !aligned(W1, 16) || !aligned(W3, 16) || !aligned(W2, 16) ||
      !aligned(y_rows, 16) || !aligned(workspace, 256) || !aligned(seg_counts, 4))
    return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  p.gather_small = false;  // the rows are regrouped into X_perm below
  p.gather_x = false;
  const Workspace w = carve(p, workspace);
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (launch_ep_regroup(p, x_rows, seg_counts, S, w, s) != cudaSuccess) return MOE_ERR_CUDA;
  const cudaError_t err =
      p.dt == 1 ? launch_expert_gemms_tc(p, x_rows, W1, W3, W2, w, s)
                : launch_expert_gemms_simt(p, static_cast<const float*>(W1),
                                           static_cast<const float*>(W3),
                                           static_cast<const float*>(W2), w, s);
  if (err != cudaSuccess) return MOE_ERR_CUDA;
  // back to the received order, splits summed, kept in fp32 (no gate: the sender applies it)
  if (launch_combine_rows(w.y, p.swap ? p.s2 : 1, p.rows_max * d, rows, (int)d, 1, w.inv,
                          nullptr, y_rows, nullptr, true, s) != cudaSuccess)
    return MOE_ERR_CUDA;
  return MOE_OK;
}

moe_status moe_combine(const float* y_rows, const int32_t* token_rows, const float* topk_gate,
                       int64_t T, int64_t d, int K, moe_dtype dt, void* out, void* stream) {
  if (T < 0 || d <= 0 || K < 1 || K > MAX_EXPERTS || (dt != MOE_F32 && dt != MOE_BF16))
    return MOE_ERR_INVALID_ARG;
  if (d % 4 || d > (1 << 20)) return MOE_ERR_UNSUPPORTED;
  if (T == 0) return MOE_OK;
  if (!y_rows || !token_rows || !topk_gate || !out || !aligned(y_rows, 16) || !aligned(out, 16) ||
      !aligned(token_rows, 4) || !aligned(topk_gate, 4))
    return MOE_ERR_INVALID_ARG;
  return launch_combine_rows(y_rows, 1, 0, T, (int)d, K, token_rows, topk_gate, out, nullptr,
                             dt == MOE_F32, static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_gather_rows(const void* in, int64_t in_rows, const int32_t* index, int64_t rows,
                           int64_t row_bytes, void* out, void* stream) {
  if (in_rows < 0 || rows < 0 || row_bytes <= 0 || row_bytes % 16) return MOE_ERR_INVALID_ARG;
  if (row_bytes > ((int64_t)1 << 24) || rows > ((int64_t)1 << 40)) return MOE_ERR_UNSUPPORTED;
  if (rows == 0) return MOE_OK;
  if (!in || !index || !out || !aligned(in, 16) || !aligned(out, 16) || !aligned(index, 4) ||
      in == out)
    return MOE_ERR_INVALID_ARG;
  return launch_gather_rows(in, in_rows, index, rows, row_bytes, out,
                            static_cast<cudaStream_t>(stream)) == cudaSuccess
             ? MOE_OK
             : MOE_ERR_CUDA;
}

moe_status moe_debug_forward_withheld(const void* x, const float* W_g, const void* W1,
                                      const void* W3, const void* W2, int64_t T, int64_t d,
                                      int64_t F, int n, int K, moe_dtype dt, void* out,
                                      void* workspace, size_t workspace_bytes, void* stream,
                                      int64_t wait_limit_cycles) {
  Plan p;
  if (!make_plan(T, d, F, n, K, (int)dt, false, &p)) return shape_status(T, d, F, n, K, dt);
  if (wait_limit_cycles < 1 || wait_limit_cycles > WAIT_LIMIT_CYCLES) return MOE_ERR_INVALID_ARG;
  if (p.dt != 1 || p.pair) return MOE_ERR_UNSUPPORTED;  // the one-CTA tensor-core kernel only
  if (T == 0) return MOE_OK;
  moe_status st = check_common(x, W_g, W1, W3, W2, out, workspace);
  if (st != MOE_OK) return st;
  if (out == x) return MOE_ERR_INVALID_ARG;
  if (workspace_bytes < p.total) return MOE_ERR_WORKSPACE;
  p.g13_withhold = true;
  p.g13_wait_limit = wait_limit_cycles;
  const Workspace w = carve(p, workspace);
  return forward_impl(p, x, W_g, W1, W3, W2, out, nullptr, w, static_cast<cudaStream_t>(stream));
}

}  // extern "C"
