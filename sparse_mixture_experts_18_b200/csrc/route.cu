// route.cu -- routing kernels of the MoE block forward.
//
//  router_topk:   l = x . W_g (fp32 accumulation), TopK (ties -> lower expert index) and
//                 Softmax over the K kept logits ("Mixtral of Experts", method section,
//                 equation G(x)); also a per-block expert histogram.  Large bf16 batches
//                 with n <= 64 take the tensor-core router of route_tc.cu instead.
//  route_scan:    per-expert exclusive prefix over router blocks and the row offsets of each
//                 expert's group (each group padded to `row_align` rows).
//  permute:       stable placement of every (token, slot) in its expert's group, the
//                 inverse map token -> row, and the gather of x rows into that order.  This
//                 is how experts with zero gate are skipped ("Mixtral 8x7B: Model Bahasa
//                 Sparse Mixture of Experts", hada.io, section "Cara Komputasi Layer MoE")
//                 while each expert sees a variable number of tokens (same page, section
//                 "Implementasi dan Efisiensi Inferensi").
#include <type_traits>

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

// Router, TopK and softmax of tokens [t0, t0 + ntok), ntok <= RT_TOK, by ROUTE_THREADS
// threads (tid = 0..255).  Experts are taken eight at a time: each thread accumulates the
// logits of the block's tokens for eight experts over its 8-element chunks of the hidden
// dimension (so each W_g row segment is loaded once per RT_TOK tokens); lanes and then warps
// are summed in a fixed order.  hist (shared, may be null) counts selections.
constexpr int RT_TOK = 8;

// w_vec: W_g rows are 16-byte aligned and n % 8 == 0 (eight experts per two float4 loads).
template <typename Tin>
__device__ __forceinline__ void route_token_block(
    const Tin* __restrict__ x, const float* __restrict__ Wg, bool w_vec, int64_t t0, int ntok,
    int d, int n, int K, int tid, float (*red)[64], float (*logits)[MAX_EXPERTS], int* hist,
    int32_t* __restrict__ idx, float* __restrict__ gate) {
  const int warp = tid >> 5, lane = tid & 31;
  for (int eg = 0; eg < n; eg += 8) {
    float acc[RT_TOK][8];
#pragma unroll
    for (int a = 0; a < RT_TOK; ++a)
#pragma unroll
      for (int e = 0; e < 8; ++e) acc[a][e] = 0.f;

    // 8-element chunks of the hidden dimension, thread-interleaved (coalesced 16-byte loads)
    for (int ci = tid; ci < d / 8; ci += ROUTE_THREADS) {
      const int j0 = ci * 8;
      Vec8<Tin> xv[RT_TOK];
#pragma unroll
      for (int a = 0; a < RT_TOK; ++a)
        if (a < ntok) xv[a].load(x + (t0 + a) * (int64_t)d + j0);
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        float w[8];
        if (w_vec) {  // eight experts of one row: two aligned float4 loads
          const float* wr = Wg + (int64_t)(j0 + i) * n + eg;
          const float4 w0 = __ldg(reinterpret_cast<const float4*>(wr));
          const float4 w1 = __ldg(reinterpret_cast<const float4*>(wr) + 1);
          w[0] = w0.x; w[1] = w0.y; w[2] = w0.z; w[3] = w0.w;
          w[4] = w1.x; w[5] = w1.y; w[6] = w1.z; w[7] = w1.w;
        } else {
          const float* wr = Wg + (int64_t)(j0 + i) * n + eg;
#pragma unroll
          for (int e = 0; e < 8; ++e) w[e] = eg + e < n ? __ldg(wr + e) : 0.f;
        }
#pragma unroll
        for (int a = 0; a < RT_TOK; ++a) {
          if (a < ntok) {
            const float xa = xv[a].get(i);
#pragma unroll
            for (int e = 0; e < 8; ++e) acc[a][e] = fmaf(xa, w[e], acc[a][e]);
          }
        }
      }
    }

    // Butterfly reduce-scatter of the 64 partial sums over the 32 lanes: after five steps
    // each lane owns two complete warp sums.
    float v[64];
#pragma unroll
    for (int a = 0; a < RT_TOK; ++a)
#pragma unroll
      for (int e = 0; e < 8; ++e) v[a * 8 + e] = acc[a][e];
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
    if (tid < 64 && eg + (tid & 7) < n) {
      float sum = 0.f;
#pragma unroll
      for (int w = 0; w < ROUTE_THREADS / 32; ++w) sum += red[w][tid];
      logits[tid >> 3][eg + (tid & 7)] = sum;
    }
    __syncthreads();
  }

  // TopK by repeated arg-max (strict '>' keeps the lower index on ties), then Softmax over
  // the kept logits shifted by the largest; the selection runs twice (normaliser, then
  // output) so that nothing is kept in per-thread arrays.
  if (tid < ntok) {
    const int a = tid;
    const int64_t t = t0 + a;
    float top = 0.f, z = 0.f;
    for (int pass = 0; pass < 2; ++pass) {
      uint64_t used = 0;
      for (int k = 0; k < K; ++k) {
        int best = -1;
        float bv = 0.f;
        for (int e = 0; e < n; ++e) {
          if ((used >> e) & 1ull) continue;
          const float le = logits[a][e];
          if (best < 0 || le > bv) { best = e; bv = le; }
        }
        used |= 1ull << best;
        if (pass == 0) {
          if (k == 0) top = bv;
          z += expf(bv - top);
        } else {
          idx[t * K + k] = best;
          gate[t * K + k] = expf(bv - top) / z;
          if (hist) atomicAdd(&hist[best], 1);
        }
      }
    }
  }
  __syncthreads();
}

// Block b routes tokens [b*tokb, b*tokb + tokb) (tokb <= RT_TOK) and writes its expert
// histogram.
template <typename Tin>
__global__ void __launch_bounds__(ROUTE_THREADS)
    router_topk_kernel(const Tin* __restrict__ x, const float* __restrict__ Wg, bool w_vec,
                       int64_t T, int d, int n, int K, int tokb, int32_t* __restrict__ idx,
                       float* __restrict__ gate, int32_t* __restrict__ blk_counts) {
  pdl_wait();
  pdl_trigger();
  __shared__ float red[ROUTE_THREADS / 32][64];
  __shared__ float logits[RT_TOK][MAX_EXPERTS];
  __shared__ int hist[MAX_EXPERTS];
  const int64_t t0 = (int64_t)blockIdx.x * tokb;
  const int ntok = (int)(T - t0 < tokb ? T - t0 : tokb);
  if (threadIdx.x < MAX_EXPERTS) hist[threadIdx.x] = 0;
  __syncthreads();
  route_token_block<Tin>(x, Wg, w_vec, t0, ntok, d, n, K, threadIdx.x, red, logits, hist, idx,
                         gate);
  if (threadIdx.x < n) blk_counts[(int64_t)blockIdx.x * n + threadIdx.x] = hist[threadIdx.x];
}

// Copy the x rows of `E` entries (entry i = (token t0 + i / K, slot i % K)) to their
// permuted rows (row[i] < 0: skip).  One warp per row, 16-byte vectors, U loads in flight per
// lane before the stores; no per-vector index arithmetic beyond the lane stride.
template <typename Tact>
__device__ __forceinline__ void gather_rows(const Tact* __restrict__ x, int64_t t0, int d, int K,
                                            int E, const int* row, Tact* __restrict__ xperm,
                                            int tid, int nthreads) {
  constexpr int U = 8;
  const int lane = tid & 31, nwarps = nthreads >> 5;
  const int vpr = d * (int)sizeof(Tact) / 16;
  for (int i = tid >> 5; i < E; i += nwarps) {
    const int r = row[i];
    if (r < 0) continue;
    const uint4* src = reinterpret_cast<const uint4*>(x + (t0 + i / K) * d);
    uint4* dst = reinterpret_cast<uint4*>(xperm + (int64_t)r * d);
    for (int c0 = lane; c0 < vpr; c0 += 32 * U) {
      uint4 buf[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < vpr) buf[u] = __ldg(src + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < vpr) dst[c0 + 32 * u] = buf[u];
    }
  }
}

// Small batches (T <= 64, T*K <= 1024) in ONE launch of G = ceil(d / 64) CTAs of 1024 threads.
// CTA c owns hidden elements [64c, 64c + 64): 8 lanes per token each take one 8-element chunk, sum
// their products with W_g and reduce over the 8 lanes in a fixed butterfly order; the CTA
// writes partial logits [c][t][e].  The last CTA to finish (ticket counter, wrapped by
// atomicInc so it is back at 0 for the next call) sums the partials in CTA order, then does
// TopK and softmax, the expert counts, group offsets (padded to row_align), the stable rank
// of every (token, slot) (per-warp match + per-expert prefix over 32-entry chunks), the
// inverse map token -> row and the map row -> token.  Then, if xq is given (FP8 weights), the
// token rows' block scales by expert row slot for G13 (sfx: slot j of expert e, K block kb at
// word (e * d/128 + kb) * 128 + 4 (j % 32) + j / 32) -- every CTA has already written its 64
// columns of each token row as MXFP8 codes (xq) and their block scale codes (sxw: per token,
// one byte per 32 columns); else, if xperm is given, the bf16 rows in permuted order.  The
// G13 kernel gathers token rows from x (bf16) or xq (FP8) otherwise.
constexpr int RS_THREADS = 1024;
constexpr int RS_MAX_T = 64;
constexpr int RS_MAX_ENTRIES = SMALL_ROUTE_MAX_ROWS;

template <typename Tact>
__global__ void __launch_bounds__(RS_THREADS)
    route_split_kernel(const Tact* __restrict__ x, const float* __restrict__ Wg, int T, int d,
                       int n, int K, int row_align, int64_t rows_max,
                       float* __restrict__ part, unsigned int* ticket,
                       int32_t* __restrict__ idx, float* __restrict__ gate,
                       int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                       int32_t* __restrict__ inv, int32_t* __restrict__ row_tok,
                       Tact* __restrict__ xperm, uint32_t* status,
                       uint8_t* __restrict__ xq, uint32_t* __restrict__ sxw,
                       uint32_t* __restrict__ sfx) {
  pdl_wait();
  pdl_trigger();
  constexpr int PER = RS_MAX_ENTRIES / RS_THREADS;  // entries per thread in the rank phase
  constexpr int CPL = 1;                            // 8-element chunks per lane
  __shared__ float logit[RS_MAX_T * MAX_EXPERTS];
  __shared__ int ccnt[RS_MAX_ENTRIES / 32][MAX_EXPERTS];  // per (32-entry chunk, expert)
  __shared__ int s_off[MAX_EXPERTS + 1];
  __shared__ int s_row[RS_MAX_ENTRIES];
  __shared__ int s_idx[RS_MAX_ENTRIES];
  __shared__ float s_sel[RS_THREADS / 32][MAX_EXPERTS];  // per warp: the kept logits
  __shared__ int s_last;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int G = gridDim.x, c = blockIdx.x;

  // ---- partial logits of this CTA's 64 hidden elements: a warp takes four tokens and eight
  // experts at a time (work items (token quad, expert octet) spread over the warps)
  const int sub = lane & 7;
  const int neg = (n + 7) / 8;
  for (int wi = warp; wi < ((T + 3) / 4) * neg; wi += RS_THREADS / 32) {
    const int tb = (wi / neg) * 4, eg = (wi % neg) * 8;
    const int t = tb + (lane >> 3);
    Vec8<Tact> xv[CPL];
    int j0[CPL];
#pragma unroll
    for (int q = 0; q < CPL; ++q) {
      j0[q] = (c * 8 * CPL + q * 8 + sub) * 8;
      if (t < T && j0[q] < d) xv[q].load(x + (int64_t)t * d + j0[q]);
    }
    if constexpr (std::is_same<Tact, __nv_bfloat16>::value) {
      static_assert(CPL == 1, "the MXFP8 blocks below assume 8 columns per lane");
      if (xq != nullptr && eg == 0) {  // FP8-weight block: this CTA's 64 columns as MXFP8
        // lanes sub 0-3 and 4-7 of the token hold one 32-element block each
        const bool have = t < T && j0[0] < d;
        float f[8], amax = 0.f;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          f[i] = have ? xv[0].get(i) : 0.f;
          amax = fmaxf(amax, fabsf(f[i]));
        }
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 1));
        amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, 2));
        const uint32_t code = mx_scale_code(amax);
        const float inv = mx_inv_scale(code);
        if (have) {
          *reinterpret_cast<uint2*>(xq + (int64_t)t * d + j0[0]) = make_uint2(
              (uint32_t)cvt_e4m3x2(f[0] * inv, f[1] * inv) |
                  ((uint32_t)cvt_e4m3x2(f[2] * inv, f[3] * inv) << 16),
              (uint32_t)cvt_e4m3x2(f[4] * inv, f[5] * inv) |
                  ((uint32_t)cvt_e4m3x2(f[6] * inv, f[7] * inv) << 16));
          // the block's code is byte j0 / 32 of the token's scale words (kb = j0 / 128)
          if ((sub & 3) == 0)
            reinterpret_cast<uint8_t*>(sxw)[(int64_t)t * (d / 32) + j0[0] / 32] = (uint8_t)code;
        }
      }
    }
    {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
#pragma unroll
      for (int q = 0; q < CPL; ++q) {
        if (t >= T || j0[q] >= d) continue;
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          const float xi = xv[q].get(i);
          const float* wr = Wg + (int64_t)(j0[q] + i) * n + eg;
          if (n % 4 == 0 && eg + 8 <= n) {  // 16-byte aligned: two float4 loads
            const float4 w0 = __ldg(reinterpret_cast<const float4*>(wr));
            const float4 w1 = __ldg(reinterpret_cast<const float4*>(wr) + 1);
            acc[0] = fmaf(xi, w0.x, acc[0]); acc[1] = fmaf(xi, w0.y, acc[1]);
            acc[2] = fmaf(xi, w0.z, acc[2]); acc[3] = fmaf(xi, w0.w, acc[3]);
            acc[4] = fmaf(xi, w1.x, acc[4]); acc[5] = fmaf(xi, w1.y, acc[5]);
            acc[6] = fmaf(xi, w1.z, acc[6]); acc[7] = fmaf(xi, w1.w, acc[7]);
          } else {
#pragma unroll
            for (int e = 0; e < 8; ++e)
              if (eg + e < n) acc[e] = fmaf(xi, __ldg(wr + e), acc[e]);
          }
        }
      }
#pragma unroll
      for (int off = 1; off < 8; off <<= 1)
#pragma unroll
        for (int e = 0; e < 8; ++e) acc[e] += __shfl_xor_sync(0xffffffffu, acc[e], off);
      if (sub == 0 && t < T) {
#pragma unroll
        for (int e = 0; e < 8; ++e)
          if (eg + e < n) part[((int64_t)c * T + t) * n + eg + e] = acc[e];
      }
    }
  }

  // ---- the last CTA to finish does the rest
  __threadfence();
  __syncthreads();
  if (tid == 0) s_last = atomicInc(ticket, (unsigned)G - 1u) == (unsigned)G - 1u;
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  for (int i = tid; i < RS_MAX_ENTRIES / 32 * MAX_EXPERTS; i += RS_THREADS) (&ccnt[0][0])[i] = 0;
  // logit (t, e) = sum over CTAs of the partials: 8 threads per logit each sum every 8th CTA
  // in order, then a fixed xor-butterfly over the 8 (one round of loads, deterministic)
  for (int v0 = 0; v0 < T * n; v0 += RS_THREADS / 8) {
    const int v = v0 + (tid >> 3), sub8 = tid & 7;
    float sum = 0.f;
    if (v < T * n) {
      float pv[8];
#pragma unroll
      for (int u = 0; u < 8; ++u) {
        const int cc = sub8 + 8 * u;
        pv[u] = cc < G ? __ldcg(part + (int64_t)cc * T * n + v) : 0.f;
      }
      for (int cc0 = 64; cc0 < G; cc0 += 8)  // G > 64 (d > 4096): remaining CTAs
        if (cc0 + sub8 < G) pv[7] += __ldcg(part + (int64_t)(cc0 + sub8) * T * n + v);
#pragma unroll
      for (int u = 0; u < 8; ++u) sum += pv[u];
    }
#pragma unroll
    for (int off = 1; off < 8; off <<= 1) sum += __shfl_xor_sync(0xffffffffu, sum, off);
    if (v < T * n && sub8 == 0) logit[v] = sum;
  }
  __syncthreads();
  // TopK by repeated arg-max (ties -> lower index), one warp per token with the n <= 64
  // logits spread over the lanes (lane e holds experts e and e + 32); then the softmax over
  // the kept logits shifted by the largest, summed in slot order
  for (int t = warp; t < T; t += RS_THREADS / 32) {
    const float* l = logit + t * n;
    const float v0 = lane < n ? l[lane] : -INFINITY;
    const float v1 = lane + 32 < n ? l[lane + 32] : -INFINITY;
    bool u0 = lane >= n, u1 = lane + 32 >= n;
    float top = 0.f, z = 0.f;
    for (int k = 0; k < K; ++k) {
      float bv;
      int bi;
      if (!u0 && (u1 || !(v1 > v0))) { bv = v0; bi = lane; }
      else if (!u1) { bv = v1; bi = lane + 32; }
      else { bv = -INFINITY; bi = 64 + lane; }
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) {
        const float ov = __shfl_xor_sync(0xffffffffu, bv, off);
        const int oi = __shfl_xor_sync(0xffffffffu, bi, off);
        if (ov > bv || (ov == bv && oi < bi)) { bv = ov; bi = oi; }
      }
      if (bi == lane) u0 = true;
      if (bi == lane + 32) u1 = true;
      if (k == 0) top = bv;
      z += expf(bv - top);
      if (lane == 0) {
        idx[t * K + k] = bi;
        s_idx[t * K + k] = bi;
        s_sel[warp][k] = bv;
      }
    }
    __syncwarp();
    for (int k = lane; k < K; k += 32) gate[t * K + k] = expf(s_sel[warp][k] - top) / z;
    __syncwarp();
  }
  __syncthreads();
  const int E = T * K;
  int e_i[PER], rank_c[PER];
#pragma unroll
  for (int j = 0; j < PER; ++j) {  // entry i = j*256 + tid lies in chunk i/32 = j*8 + warp
    const int i = j * RS_THREADS + tid;
    e_i[j] = i < E ? s_idx[i] : -1;
    const unsigned vmask = __ballot_sync(0xffffffffu, e_i[j] >= 0);
    const unsigned peers = __match_any_sync(0xffffffffu, e_i[j]) & vmask;
    rank_c[j] = __popc(peers & ((1u << lane) - 1u));
    if (e_i[j] >= 0 && rank_c[j] == 0)
      ccnt[j * (RS_THREADS / 32) + warp][e_i[j]] = __popc(peers);
  }
  __syncthreads();
  for (int e = warp; e < n; e += RS_THREADS / 32) {  // expert e: prefix over the 32 chunks
    const int v = ccnt[lane][e];
    int incl = v;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, incl, off);
      if (lane >= off) incl += y;
    }
    ccnt[lane][e] = incl - v;
    if (lane == 31) s_off[e] = incl;  // total for now
  }
  __syncthreads();
  if (tid == 0) {
    int64_t off = 0;
    for (int e = 0; e < n; ++e) {
      const int cnt = s_off[e];
      counts[e] = cnt;
      s_off[e] = (int)off;
      offsets[e] = (int)off;
      off += (int64_t)(cnt + row_align - 1) / row_align * row_align;
    }
    s_off[n] = (int)off;
    offsets[n] = (int)off;
    if (off > rows_max) set_status(status, DEV_ERR_ROW);
  }
  __syncthreads();
#pragma unroll
  for (int j = 0; j < PER; ++j) {
    const int i = j * RS_THREADS + tid;
    if (i >= E) continue;
    int row = s_off[e_i[j]] + ccnt[j * (RS_THREADS / 32) + warp][e_i[j]] + rank_c[j];
    if (row >= rows_max) {
      set_status(status, DEV_ERR_ROW);
      row = -1;
    }
    s_row[i] = row;
    inv[i] = row;
    if (row >= 0) row_tok[row] = i / K;
  }
  if (xq != nullptr) {  // FP8-weight block: quantised token rows and their block scales
    if constexpr (std::is_same<Tact, __nv_bfloat16>::value) {
      __syncthreads();  // s_row is complete (sxw: written by every CTA before its ticket)
      const int kbs = d / 128;
      for (int q = tid; q < E * kbs; q += RS_THREADS) {
        const int i = q / kbs, kb = q % kbs;
        const int row = s_row[i];
        if (row < 0) continue;
        const int e = s_idx[i];
        const int j = row - s_off[e];  // < 64: an expert gets at most T rows
        sfx[((int64_t)e * kbs + kb) * 128 + 4 * (j & 31) + (j >> 5)] =
            sxw[(int64_t)(i / K) * kbs + kb];
      }
    }
    return;
  }
  if (xperm == nullptr) return;  // the G13 kernel gathers the token rows from x
  __syncthreads();
  gather_rows(x, 0, d, K, E, s_row, xperm, tid, RS_THREADS);
}

// One CTA per expert e: exclusive prefix over router blocks of the block histograms
// (blk_base[b][e]) and the expert's total (counts[e]).  Each thread takes a contiguous run of
// blocks; the runs' sums are scanned across the CTA (warp shuffles, then the 32 warp sums).
// The last CTA to finish (a ticket that wraps back to 0) lays out the groups: offsets[e] =
// sum over e' < e of counts[e'] rounded up to row_align (the counts are read in one round of
// loads: reading them one after the other took the scan from 12.5 to 20.5 us at n = 64).
constexpr int SCAN_THREADS = 1024;
constexpr int SCAN_RUN = 8;  // blocks per thread held in registers per pass

__global__ void __launch_bounds__(SCAN_THREADS)
    route_scan_kernel(const int32_t* __restrict__ blk_counts, int64_t nblk, int n,
                      int row_align, int64_t rows_max, int32_t* __restrict__ blk_base,
                      int32_t* __restrict__ counts, int32_t* __restrict__ offsets,
                      unsigned int* ticket, uint32_t* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int wsum[SCAN_THREADS / 32];
  __shared__ int s_last;
  __shared__ int s_cnt[MAX_EXPERTS];
  const int e = blockIdx.x, tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int64_t run = (nblk + SCAN_THREADS - 1) / SCAN_THREADS;
  const int64_t b0 = tid * run, b1 = b0 + run < nblk ? b0 + run : nblk;
  int local = 0;
  for (int64_t b = b0; b < b1; b += SCAN_RUN) {
    int v[SCAN_RUN];
#pragma unroll
    for (int j = 0; j < SCAN_RUN; ++j) v[j] = b + j < b1 ? blk_counts[(b + j) * n + e] : 0;
#pragma unroll
    for (int j = 0; j < SCAN_RUN; ++j) local += v[j];
  }
  // inclusive scan of the per-thread sums: within each warp, then over the warps
  int incl = local;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int y = __shfl_up_sync(0xffffffffu, incl, off);
    if (lane >= off) incl += y;
  }
  if (lane == 31) wsum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int ws = wsum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xffffffffu, ws, off);
      if (lane >= off) ws += y;
    }
    wsum[lane] = ws;  // inclusive over warps
  }
  __syncthreads();
  int prefix = incl - local + (warp > 0 ? wsum[warp - 1] : 0);
  for (int64_t b = b0; b < b1; b += SCAN_RUN) {
    int v[SCAN_RUN];
#pragma unroll
    for (int j = 0; j < SCAN_RUN; ++j) v[j] = b + j < b1 ? blk_counts[(b + j) * n + e] : 0;
#pragma unroll
    for (int j = 0; j < SCAN_RUN; ++j)
      if (b + j < b1) {
        blk_base[(b + j) * n + e] = prefix;
        prefix += v[j];
      }
  }
  if (tid == SCAN_THREADS - 1) {
    counts[e] = wsum[31];
    __threadfence();
    s_last = atomicInc(ticket, (unsigned)gridDim.x - 1u) == (unsigned)gridDim.x - 1u;
  }
  __syncthreads();
  if (!s_last) return;
  // the last CTA: every expert's count in one round of L2 loads, then the offsets
  __threadfence();
  if (tid < n) s_cnt[tid] = __ldcg(&counts[tid]);
  __syncthreads();
  if (tid == 0) {
    int64_t off = 0;
    for (int x = 0; x < n; ++x) {
      offsets[x] = (int32_t)off;
      off += (int64_t)(s_cnt[x] + row_align - 1) / row_align * row_align;
    }
    offsets[n] = (int32_t)off;
    if (off > rows_max) set_status(status, DEV_ERR_ROW);
  }
}

// Block b takes the same tokens as router block b.  Entry i = (token, slot) in token-major
// order gets rank = number of earlier entries of this block routed to the same expert, so
// the placement is stable (rows of an expert ordered by token, then slot).  Writes the
// inverse map and either gathers the x rows into X_perm or (xperm == null) records the token
// and the gate of each row for the GEMMs that read x directly.
template <typename Tact>
__global__ void __launch_bounds__(256)
    permute_gather_kernel(const Tact* __restrict__ x, int64_t T, int d, int n, int K,
                          int tokb, const int32_t* __restrict__ idx,
                          const float* __restrict__ gate,
                          const int32_t* __restrict__ blk_base,
                          const int32_t* __restrict__ offsets, int64_t rows_max,
                          int32_t* __restrict__ inv, Tact* __restrict__ xperm,
                          int32_t* __restrict__ row_tok, float* __restrict__ row_gate,
                          uint32_t* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int ent_e[64];
  __shared__ int ent_row[64];
  const int64_t t0 = (int64_t)blockIdx.x * tokb;
  const int ntok = (int)(T - t0 < tokb ? T - t0 : tokb);
  const int E = ntok * K;  // <= 64: tokb = route_tokens_per_block(K)
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
    if (xperm == nullptr && row >= 0) {
      row_tok[row] = (int32_t)(t0 + i / K);
      row_gate[row] = gate[t0 * K + i];
    }
  }
  if (xperm == nullptr) return;
  __syncthreads();
  gather_rows(x, t0, d, K, E, ent_row, xperm, threadIdx.x, blockDim.x);
}

// ---------------------------------------------------------------- expert-parallel regroup
// The rows a rank receives for its nl local experts arrive from S sources (ranks), each
// source's rows grouped by local expert in expert order, with seg_counts[s][e] rows in
// segment (s, e).  This kernel places them in the per-expert layout the grouped GEMMs take:
// expert e's group is padded to row_align rows and holds the segments (0, e), (1, e), ...
// in source order.  Every CTA recomputes the segment starts in shared memory (S * nl <= 2048
// entries); CTA 0 also writes counts and offsets.  Then one warp per received row r finds its
// segment (binary search over the segment starts), writes inv[r] = its padded row and copies
// the row into X_perm.  The counts must add up to `rows` (else DEV_ERR_ROW, nothing copied).
constexpr int EP_MAX_SEGS = 2048;

template <typename Tact>
__global__ void __launch_bounds__(256)
    ep_regroup_kernel(const Tact* __restrict__ xr, int64_t rows, int d,
                      const int32_t* __restrict__ seg_counts, int S, int nl, int row_align,
                      int64_t rows_max, int32_t* __restrict__ counts,
                      int32_t* __restrict__ offsets, int32_t* __restrict__ inv,
                      Tact* __restrict__ xperm, uint32_t* status) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_cnt[EP_MAX_SEGS];    // segment (s, e) at s * nl + e: its count
  __shared__ int s_start[EP_MAX_SEGS];  // its first received row
  __shared__ int s_base[EP_MAX_SEGS];   // its first row in the padded layout
  __shared__ int s_off[MAX_EXPERTS + 1];
  __shared__ int s_ok;
  const int nseg = S * nl;
  for (int i = threadIdx.x; i < nseg; i += blockDim.x) s_cnt[i] = seg_counts[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int64_t off = 0, start = 0;
    bool ok = true;
    for (int e = 0; e < nl; ++e) {  // expert groups: segments of expert e in source order
      s_off[e] = (int)off;
      int64_t c = 0;
      for (int q = 0; q < S; ++q) {
        const int v = s_cnt[q * nl + e];
        ok = ok && v >= 0;
        s_base[q * nl + e] = (int)(off + c);
        c += v;
      }
      if (blockIdx.x == 0) counts[e] = (int32_t)c;
      off += (c + row_align - 1) / row_align * row_align;
    }
    s_off[nl] = (int)off;
    for (int i = 0; i < nseg; ++i) {  // received order: source-major, then expert
      s_start[i] = (int)start;
      start += s_cnt[i];
    }
    ok = ok && start == rows && off <= rows_max;
    if (blockIdx.x == 0) {
      for (int e = 0; e <= nl; ++e) offsets[e] = s_off[e];
      if (!ok) set_status(status, DEV_ERR_ROW);
    }
    s_ok = ok;
  }
  __syncthreads();
  if (!s_ok) return;
  const int lane = threadIdx.x & 31;
  const int vpr = d * (int)sizeof(Tact) / 16;
  for (int64_t r = ((int64_t)blockIdx.x * blockDim.x + threadIdx.x) >> 5; r < rows;
       r += ((int64_t)gridDim.x * blockDim.x) >> 5) {
    int lo = 0, hi = nseg - 1;  // last segment starting at or before r (it is not empty)
    while (lo < hi) {
      const int mid = (lo + hi + 1) >> 1;
      if (s_start[mid] <= r) lo = mid; else hi = mid - 1;
    }
    const int64_t dst = s_base[lo] + (r - s_start[lo]);
    if (lane == 0) inv[r] = (int32_t)dst;
    const uint4* src = reinterpret_cast<const uint4*>(xr + r * d);
    uint4* out = reinterpret_cast<uint4*>(xperm + dst * d);
    for (int c = lane; c < vpr; c += 32) out[c] = __ldg(src + c);
  }
}

cudaError_t launch_ep_regroup(const Plan& p, const void* x_rows, const int32_t* seg_counts,
                              int S, const Workspace& w, cudaStream_t s) {
  const int64_t rows = p.T;  // the received rows are the plan's tokens (K = 1)
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = 4 * (int64_t)num_sms();
  if (blocks > cap) blocks = cap;
  if (blocks < 1) blocks = 1;
  if (p.dt == 1)
    pdl(ep_regroup_kernel<__nv_bfloat16>, (unsigned)blocks, 256, 0, s)(
        static_cast<const __nv_bfloat16*>(x_rows), rows, (int)p.d, seg_counts, S, p.n,
        p.row_align, p.rows_max, w.counts, w.offsets, w.inv,
        static_cast<__nv_bfloat16*>(w.xperm), w.status);
  else
    pdl(ep_regroup_kernel<float>, (unsigned)blocks, 256, 0, s)(
        static_cast<const float*>(x_rows), rows, (int)p.d, seg_counts, S, p.n, p.row_align,
        p.rows_max, w.counts, w.offsets, w.inv, static_cast<float*>(w.xperm), w.status);
  return cudaGetLastError();
}

// ---------------------------------------------------------------- row gather
// out[i] = in[index[i]] for rows of vpr 16-byte vectors (the expert-parallel exchange with
// replicated experts puts a rank's grouped rows in destination order and its returned rows
// back in grouped order with it).  One warp per output row, U loads in flight per lane; an
// index outside [0, in_rows) leaves its output row unwritten.
__global__ void __launch_bounds__(256)
    gather_rows_kernel(const uint4* __restrict__ in, int64_t in_rows,
                       const int32_t* __restrict__ index, int64_t rows, int vpr,
                       uint4* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  constexpr int U = 8;
  const int lane = threadIdx.x & 31;
  for (int64_t r = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5); r < rows;
       r += (int64_t)gridDim.x * 8) {  // warp-uniform
    const int64_t src = index[r];
    if (src < 0 || src >= in_rows) continue;
    const uint4* sp = in + src * vpr;
    uint4* dp = out + r * vpr;
    for (int c0 = lane; c0 < vpr; c0 += 32 * U) {
      uint4 buf[U];
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < vpr) buf[u] = __ldg(sp + c0 + 32 * u);
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (c0 + 32 * u < vpr) dp[c0 + 32 * u] = buf[u];
    }
  }
}

cudaError_t launch_gather_rows(const void* in, int64_t in_rows, const int32_t* index,
                               int64_t rows, int64_t row_bytes, void* out, cudaStream_t s) {
  if (rows <= 0) return cudaSuccess;
  int64_t blocks = (rows + 7) / 8;
  const int64_t cap = 8 * (int64_t)num_sms();
  if (blocks > cap) blocks = cap;
  pdl(gather_rows_kernel, (unsigned)blocks, 256, 0, s)(
      static_cast<const uint4*>(in), in_rows, index, rows, (int)(row_bytes / 16),
      static_cast<uint4*>(out));
  return cudaGetLastError();
}

// ---------------------------------------------------------------- host launchers

// Tokens per router / permute block: eight, or fewer when K > 8 so that a block's
// (token, slot) entries stay within 64.
int route_tokens_per_block(int K) { return K <= 8 ? RT_TOK : (64 / K > 0 ? 64 / K : 1); }

template <typename Tin>
static cudaError_t launch_router_t(const Tin* x, const float* Wg, int64_t T, int d, int n,
                                   int K, int32_t* idx, float* gate, int32_t* blk_counts,
                                   cudaStream_t s) {
  const int tokb = route_tokens_per_block(K);
  const int64_t nblk = (T + tokb - 1) / tokb;
  const bool w_vec = n % 8 == 0 && (reinterpret_cast<uintptr_t>(Wg) & 15u) == 0;
  pdl(router_topk_kernel<Tin>, (unsigned)nblk, ROUTE_THREADS, 0, s)(x, Wg, w_vec, T, d, n, K,
                                                                    tokb, idx, gate,
                                                                    blk_counts);
  return cudaGetLastError();
}

template <typename Tact>
static cudaError_t launch_route_small_t(const Plan& p, const Tact* x, const float* Wg,
                                        const Workspace& w, cudaStream_t s) {
  const int G = (int)((p.d + 63) / 64);
  pdl(route_split_kernel<Tact>, G, RS_THREADS, 0, s)(
      x, Wg, (int)p.T, (int)p.d, p.n, p.K, p.row_align, p.rows_max, w.rpart, w.ticket, w.idx,
      w.gate, w.counts, w.offsets, w.inv, w.row_tok,
      p.gather_small ? nullptr : static_cast<Tact*>(w.xperm), w.status,
      p.fp8 ? static_cast<uint8_t*>(w.xperm) : nullptr, p.fp8 ? w.sxw : nullptr,
      p.fp8 ? w.sfx : nullptr);
  return cudaGetLastError();
}

cudaError_t launch_route(const Plan& p, const void* x, const float* Wg, const Workspace& w,
                         cudaStream_t s) {
  if (p.fused_route)
    return p.dt == 1 ? launch_route_small_t(p, static_cast<const __nv_bfloat16*>(x), Wg, w, s)
                     : launch_route_small_t(p, static_cast<const float*>(x), Wg, w, s);
  cudaError_t err;
  if (router_tc_applies(p))
    err = launch_router_tc(p, x, Wg, w, s);
  else if (p.dt == 1)
    err = launch_router_t(static_cast<const __nv_bfloat16*>(x), Wg, p.T, (int)p.d, p.n, p.K,
                          w.idx, w.gate, w.blk_counts, s);
  else
    err = launch_router_t(static_cast<const float*>(x), Wg, p.T, (int)p.d, p.n, p.K, w.idx,
                          w.gate, w.blk_counts, s);
  if (err != cudaSuccess) return err;
  pdl(route_scan_kernel, (unsigned)p.n, SCAN_THREADS, 0, s)(
      w.blk_counts, p.nblk, p.n, p.row_align, p.rows_max, w.blk_base, w.counts, w.offsets,
      w.scan_ticket, w.status);
  if ((err = cudaGetLastError()) != cudaSuccess) return err;
  const int tokb = route_tokens_per_block(p.K);
  if (p.dt == 1)
    pdl(permute_gather_kernel<__nv_bfloat16>, (unsigned)p.nblk, 256, 0, s)(
        static_cast<const __nv_bfloat16*>(x), p.T, (int)p.d, p.n, p.K, tokb, w.idx, w.gate,
        w.blk_base, w.offsets, p.rows_max, w.inv,
        p.gather_x ? nullptr : static_cast<__nv_bfloat16*>(w.xperm), w.row_tok, w.row_gate,
        w.status);
  else
    pdl(permute_gather_kernel<float>, (unsigned)p.nblk, 256, 0, s)(
        static_cast<const float*>(x), p.T, (int)p.d, p.n, p.K, tokb, w.idx, w.gate, w.blk_base,
        w.offsets, p.rows_max, w.inv, static_cast<float*>(w.xperm), w.row_tok, w.row_gate,
        w.status);
  return cudaGetLastError();
}

}  // namespace moe
