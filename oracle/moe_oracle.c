/*
 * moe_oracle.c -- plain, slow, obviously-correct CPU oracle for the forward pass of
 * Mixtral's sparse Mixture-of-Experts block.
 *
 * TEST INFRASTRUCTURE ONLY.  Nothing on the product path may link, load or call this file:
 * only the test-suite, the smoke check and the benchmark's CPU-baseline leg use it.  It
 * shares no code, header, table or helper with the CUDA library.
 *
 * Everything is computed in IEEE double from the exact values of the given (bf16 or fp32)
 * inputs, one token at a time, in the order the method states it:
 *
 *   "Mixtral of Experts" (arXiv 2401.04088), method section with equations G(x) and y:
 *     l        = x . W_g                       router logits over n experts (no bias)
 *     TopK(l)_i = l_i if l_i is among the K largest coordinates of l, -inf otherwise
 *     G(x)     = Softmax(TopK(l))              K = 2 in Mixtral
 *     y        = sum_{i=0}^{n-1} G(x)_i * SwiGLU_i(x)
 *   The same page fixes n = 8 experts, each a SwiGLU FFN of intermediate width 14336 on a
 *   hidden size of 4096, and its glossary describes SwiGLU as Swish combined with an
 *   element-wise product; the plainest reading (no biases, Swish beta = 1) is
 *     SwiGLU_e(x) = W2_e . ( silu(W1_e . x) * (W3_e . x) ),  silu(z) = z / (1 + e^-z).
 *   The Indonesian news summary (section on how the MoE layer is computed) adds that experts
 *   whose gate is 0 need not be computed; oracle_moe_dense() runs all n experts anyway so
 *   that this equivalence can be checked.
 *
 * Readings where the pages are silent (each is listed with the reasoning in the design notes):
 *   - ties in TopK go to the lower expert index; slot 0 holds the larger logit;
 *   - the softmax is taken over the K kept logits, shifted by the largest one;
 *   - h = silu(a) * b is rounded to the expert dtype (bf16 round-to-nearest-even for bf16
 *     weights, no rounding for fp32) before the down-projection, and y is rounded once to
 *     the output dtype (rounding is left to the caller, which gets y in double);
 *   - RMSNorm for the 32-block stack: gamma = 1, eps given by the caller, output rounded to
 *     the activation dtype; the residual add is x + y in double, rounded once.
 *
 * Layouts (row-major): x [T][d]; W_g [d][n] fp32; W1, W3 [n][F][d]; W2 [n][d][F].
 *
 * Parity status: every function here is pinned by tests against closed forms, brute force
 * or library routines (see tests/test_oracle.py); none is "parity unpinned".  The FP8
 * functions at the end (E4M3 codes, E8M0 block scales, block quantisation, the FP8-weight
 * block) are pinned against the formats' defining values, an independent numpy/torch
 * restatement of the block-scale rule and torch's float8_e4m3fn conversion.
 */
#include <math.h>
#include <stdint.h>
#include <stdlib.h>
#include <string.h>

#define ORACLE_F32 0
#define ORACLE_BF16 1

/* ---------------------------------------------------------------- element access */

/* Exact value of one stored element.  A bf16 is the top 16 bits of an IEEE binary32. */
static double elem(const void* base, int dtype, int64_t i) {
  if (dtype == ORACLE_F32) return (double)((const float*)base)[i];
  uint32_t bits = (uint32_t)((const uint16_t*)base)[i] << 16;
  float f;
  memcpy(&f, &bits, sizeof f);
  return (double)f;
}

/* Round a double to the nearest bfloat16 value (ties to even), returned as a double.
 * bfloat16: 1 sign bit, 8 exponent bits (same range as binary32), 7 stored mantissa bits,
 * i.e. 8 significant bits for normal numbers, quantum 2^-133 below 2^-126. */
double oracle_round_bf16(double v) {
  if (v == 0.0 || isnan(v) || isinf(v)) return v;
  int e;
  double m = frexp(v, &e);          /* v = m * 2^e, 0.5 <= |m| < 1 */
  int q = e - 8;                    /* quantum exponent for 8 significant bits */
  if (q < -133) q = -133;           /* subnormal range has a fixed quantum */
  double scaled = ldexp(v, -q);
  double r = nearbyint(scaled);     /* default rounding mode: nearest, ties to even */
  double out = ldexp(r, q);
  if (fabs(out) > 3.3895313892515355e38) return v > 0 ? INFINITY : -INFINITY;
  return out;
}

double oracle_round_f32(double v) { return (double)(float)v; }

/* In-place rounding of an array to dtype (the contract's single output rounding). */
void oracle_round_array(double* v, int64_t count, int dtype) {
  for (int64_t i = 0; i < count; ++i)
    v[i] = dtype == ORACLE_BF16 ? oracle_round_bf16(v[i]) : oracle_round_f32(v[i]);
}

static double round_to(double v, int dtype) {
  return dtype == ORACLE_BF16 ? oracle_round_bf16(v) : oracle_round_f32(v);
}

double oracle_silu(double z) { return z / (1.0 + exp(-z)); }

/* ---------------------------------------------------------------- router: l, TopK, G */

/* Logits l = x . W_g of one token, in double. */
static void router_logits(int64_t d, int n, int x_dtype, const void* x, int64_t t,
                          const float* Wg, double* l) {
  for (int i = 0; i < n; ++i) l[i] = 0.0;
  for (int64_t j = 0; j < d; ++j) {
    double xj = elem(x, x_dtype, t * d + j);
    for (int i = 0; i < n; ++i) l[i] += xj * (double)Wg[j * n + i];
  }
}

/* Expert order: larger logit first, equal logits by lower index. */
static int before(const double* l, int a, int b) {
  return l[a] > l[b] || (l[a] == l[b] && a < b);
}

/* TopK then Softmax over the kept K logits.  Full insertion sort of the n experts. */
static void topk_softmax(int n, int K, const double* l, int32_t* idx, double* gate) {
  int order[256];
  for (int i = 0; i < n; ++i) order[i] = i;
  for (int i = 1; i < n; ++i) {
    int v = order[i], j = i - 1;
    while (j >= 0 && before(l, v, order[j])) { order[j + 1] = order[j]; --j; }
    order[j + 1] = v;
  }
  double top = l[order[0]], z = 0.0;
  for (int k = 0; k < K; ++k) z += exp(l[order[k]] - top);
  for (int k = 0; k < K; ++k) {
    idx[k] = order[k];
    gate[k] = exp(l[order[k]] - top) / z;
  }
}

/* Router for T tokens: logits [T][n] (may be NULL), idx [T][K], gate [T][K]. */
int oracle_route(int64_t T, int64_t d, int n, int K, int x_dtype, const void* x,
                 const float* Wg, double* logits, int32_t* idx, double* gate) {
  if (n < 1 || n > 256 || K < 1 || K > n) return 1;
#pragma omp parallel for schedule(static)
  for (int64_t t = 0; t < T; ++t) {
    double l[256];
    router_logits(d, n, x_dtype, x, t, Wg, l);
    if (logits) for (int i = 0; i < n; ++i) logits[t * n + i] = l[i];
    topk_softmax(n, K, l, idx + t * K, gate + t * K);
  }
  return 0;
}

/* ---------------------------------------------------------------- one SwiGLU expert */

/* y = W2_e . round(silu(W1_e . x_t) * (W3_e . x_t)), accumulated into acc with weight g.
 * h_dtype: dtype h is rounded to (-1 = no rounding). */
static void expert_accumulate(int64_t d, int64_t F, int w_dtype, int h_dtype,
                              const double* xt, const void* W1, const void* W3,
                              const void* W2, int e, double g, double* acc, double* h) {
  const int64_t w13 = (int64_t)e * F * d, w2 = (int64_t)e * d * F;
  for (int64_t f = 0; f < F; ++f) {
    double a = 0.0, b = 0.0;
    for (int64_t j = 0; j < d; ++j) {
      a += xt[j] * elem(W1, w_dtype, w13 + f * d + j);
      b += xt[j] * elem(W3, w_dtype, w13 + f * d + j);
    }
    double hf = oracle_silu(a) * b;
    h[f] = h_dtype < 0 ? hf : round_to(hf, h_dtype);
  }
  for (int64_t i = 0; i < d; ++i) {
    double yi = 0.0;
    for (int64_t f = 0; f < F; ++f) yi += h[f] * elem(W2, w_dtype, w2 + i * F + f);
    acc[i] += g * yi;
  }
}

/* ---------------------------------------------------------------- the MoE block */

/* Sparse MoE forward for the tokens in tok[0..n_tok): y[r][0..d) (double, unrounded) for
 * token tok[r]; idx/gate of those tokens are written too (may be NULL).
 * round_h: 1 = round h to the weight dtype (bf16 contract), 0 = keep h in double. */
int oracle_moe_forward(int64_t T, int64_t d, int64_t F, int n, int K, int dtype,
                       const void* x, const float* Wg, const void* W1, const void* W3,
                       const void* W2, int round_h, int64_t n_tok, const int64_t* tok,
                       double* y, int32_t* idx_out, double* gate_out) {
  if (n < 1 || n > 256 || K < 1 || K > n) return 1;
  for (int64_t r = 0; r < n_tok; ++r) if (tok[r] < 0 || tok[r] >= T) return 2;
  int fail = 0;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * d);
    double* h = (double*)malloc(sizeof(double) * F);
    if (!xt || !h) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_tok; ++r) {
      if (!xt || !h) continue;
      int64_t t = tok[r];
      double l[256], gate[256];
      int32_t idx[256];
      router_logits(d, n, dtype, x, t, Wg, l);
      topk_softmax(n, K, l, idx, gate);
      for (int64_t j = 0; j < d; ++j) xt[j] = elem(x, dtype, t * d + j);
      double* yr = y + r * d;
      for (int64_t i = 0; i < d; ++i) yr[i] = 0.0;
      for (int k = 0; k < K; ++k)
        expert_accumulate(d, F, dtype, round_h ? dtype : -1, xt, W1, W3, W2, idx[k],
                          gate[k], yr, h);
      for (int k = 0; k < K; ++k) {
        if (idx_out) idx_out[r * K + k] = idx[k];
        if (gate_out) gate_out[r * K + k] = gate[k];
      }
    }
    free(xt);
    free(h);
  }
  return fail ? 3 : 0;
}

/* Same block for one token, but with the K experts given explicitly (experts[0..K)); the
 * gates are the softmax of the token's own logits over that set, shifted by its largest.
 * Used where logits tie within rounding, so that every admissible expert set can be
 * evaluated by the oracle itself. */
int oracle_moe_token_with_experts(int64_t T, int64_t d, int64_t F, int n, int K, int dtype,
                                  const void* x, const float* Wg, const void* W1,
                                  const void* W3, const void* W2, int round_h, int64_t t,
                                  const int32_t* experts, double* y) {
  if (t < 0 || t >= T || K < 1 || K > n || n > 256) return 1;
  double l[256], top = -INFINITY, z = 0.0;
  router_logits(d, n, dtype, x, t, Wg, l);
  for (int k = 0; k < K; ++k) {
    if (experts[k] < 0 || experts[k] >= n) return 2;
    if (l[experts[k]] > top) top = l[experts[k]];
  }
  for (int k = 0; k < K; ++k) z += exp(l[experts[k]] - top);
  double* xt = (double*)malloc(sizeof(double) * d);
  double* h = (double*)malloc(sizeof(double) * F);
  if (!xt || !h) { free(xt); free(h); return 3; }
  for (int64_t j = 0; j < d; ++j) xt[j] = elem(x, dtype, t * d + j);
  for (int64_t i = 0; i < d; ++i) y[i] = 0.0;
  for (int k = 0; k < K; ++k)
    expert_accumulate(d, F, dtype, round_h ? dtype : -1, xt, W1, W3, W2, experts[k],
                      exp(l[experts[k]] - top) / z, y, h);
  free(xt);
  free(h);
  return 0;
}

/* Dense-masked form: every one of the n experts is evaluated and weighted by G(x)_i, which
 * is 0 off the top-K.  Equal to oracle_moe_forward in exact arithmetic. */
int oracle_moe_dense(int64_t T, int64_t d, int64_t F, int n, int K, int dtype, const void* x,
                     const float* Wg, const void* W1, const void* W3, const void* W2,
                     int round_h, int64_t n_tok, const int64_t* tok, double* y) {
  if (n < 1 || n > 256 || K < 1 || K > n) return 1;
  for (int64_t r = 0; r < n_tok; ++r) if (tok[r] < 0 || tok[r] >= T) return 2;
  int fail = 0;
#pragma omp parallel
  {
    double* xt = (double*)malloc(sizeof(double) * d);
    double* h = (double*)malloc(sizeof(double) * F);
    if (!xt || !h) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_tok; ++r) {
      if (!xt || !h) continue;
      int64_t t = tok[r];
      double l[256], gate[256], G[256];
      int32_t idx[256];
      router_logits(d, n, dtype, x, t, Wg, l);
      topk_softmax(n, K, l, idx, gate);
      for (int i = 0; i < n; ++i) G[i] = 0.0;
      for (int k = 0; k < K; ++k) G[idx[k]] = gate[k];
      for (int64_t j = 0; j < d; ++j) xt[j] = elem(x, dtype, t * d + j);
      double* yr = y + r * d;
      for (int64_t i = 0; i < d; ++i) yr[i] = 0.0;
      for (int i = 0; i < n; ++i)
        expert_accumulate(d, F, dtype, round_h ? dtype : -1, xt, W1, W3, W2, i, G[i], yr, h);
    }
    free(xt);
    free(h);
  }
  return fail ? 3 : 0;
}

/* ---------------------------------------------------------------- 32-block stack pieces */

/* RMSNorm with gamma = 1: xn = x / sqrt(mean(x^2) + eps), rounded to dtype.
 * x and xn are [rows][d] doubles holding values exactly representable in dtype. */
void oracle_rmsnorm(int64_t rows, int64_t d, int dtype, double eps, const double* x,
                    double* xn) {
  for (int64_t r = 0; r < rows; ++r) {
    double ss = 0.0;
    for (int64_t j = 0; j < d; ++j) ss += x[r * d + j] * x[r * d + j];
    double inv = 1.0 / sqrt(ss / (double)d + eps);
    for (int64_t j = 0; j < d; ++j) xn[r * d + j] = round_to(x[r * d + j] * inv, dtype);
  }
}

/* One stacked block for a set of independent token rows:
 *   x <- round(x + MoE(RMSNorm(x)))
 * x: [rows][d] doubles (values of the activation dtype), updated in place.
 * Weights of this layer in their stored dtype.  idx_out/gate_out: routing of each row. */
int oracle_block_forward(int64_t rows, int64_t d, int64_t F, int n, int K, int dtype,
                         double eps, double* x, const float* Wg, const void* W1,
                         const void* W3, const void* W2, int32_t* idx_out,
                         double* gate_out) {
  if (n < 1 || n > 256 || K < 1 || K > n) return 1;
  double* xn = (double*)malloc(sizeof(double) * rows * d);
  if (!xn) return 3;
  oracle_rmsnorm(rows, d, dtype, eps, x, xn);
  int fail = 0;
#pragma omp parallel
  {
    double* h = (double*)malloc(sizeof(double) * F);
    double* yr = (double*)malloc(sizeof(double) * d);
    if (!h || !yr) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < rows; ++r) {
      if (!h || !yr) continue;
      const double* xt = xn + r * d;
      double l[256], gate[256];
      int32_t idx[256];
      for (int i = 0; i < n; ++i) l[i] = 0.0;
      for (int64_t j = 0; j < d; ++j)
        for (int i = 0; i < n; ++i) l[i] += xt[j] * (double)Wg[j * n + i];
      topk_softmax(n, K, l, idx, gate);
      for (int64_t i = 0; i < d; ++i) yr[i] = 0.0;
      for (int k = 0; k < K; ++k)
        expert_accumulate(d, F, dtype, dtype, xt, W1, W3, W2, idx[k], gate[k], yr, h);
      for (int64_t i = 0; i < d; ++i) x[r * d + i] = round_to(x[r * d + i] + yr[i], dtype);
      for (int k = 0; k < K; ++k) {
        if (idx_out) idx_out[r * K + k] = idx[k];
        if (gate_out) gate_out[r * K + k] = gate[k];
      }
    }
    free(h);
    free(yr);
  }
  free(xn);
  return fail ? 3 : 0;
}

/* ---------------------------------------------------------------- FP8 expert weights
 *
 * The low-precision-weights variant (the pages mention only quantised community builds of
 * the model, so the format below is this library's own reading: the OCP Microscaling (MX)
 * format MXFP8 with E4M3 elements, which the sm_100a tensor cores scale in hardware):
 *   - OCP FP8 E4M3 ("fn" flavour): 1 sign bit, 4 exponent bits with bias 7, 3 mantissa bits,
 *     no infinities, S.1111.111 is NaN, largest finite value 448 = 1.75 * 2^8, smallest
 *     subnormal 2^-9;
 *   - every row of every matrix (W1, W3 rows f of [F][d]; W2 rows i of [d][F]; each token's
 *     row of x; each row of h) is cut along its length into blocks of 32 consecutive
 *     elements, and each block shares one scale X = 2^E, stored as an E8M0 code E + 127:
 *     E is the smallest integer with max_j |v_j| <= 448 * 2^E, so that no element of the
 *     block overflows E4M3's largest finite value (with max |v| = m 2^e, 1 <= m < 2:
 *     E = e - 8 if m <= 1.75, else e - 7), clamped to [-127, 127]; an all-zero block takes
 *     E = 0.  (The OCP text's E = floor(log2 max |v|) - 8 would clip block maxima in
 *     [448, 512) X to 448.)
 *     element codes P_j = E4M3(v_j / X): the nearest code, ties to the even mantissa (values
 *     past 448, only possible when E was clamped, saturate) -- v_j / X is exact (X a power
 *     of two);
 *   - a_f = sum over blocks b of X_x,b X_1,f,b sum_{j in b} P_x,j P_1,f,j (exact in double),
 *     b_f likewise with W3; h_f = silu(a_f) b_f rounded to binary32 and block-quantised the
 *     same way; y_i = sum_b X_h,b X_2,i,b sum_{f in b} P_h,f P_2,i,f;
 *     out = sum_k G_k y_{e_k}, rounded once.
 *   Routing is the bf16 block's (the router reads the bf16 activations and fp32 W_g).
 *   Scale codes are stored plainly here, [rows][cols / 32].
 */

#define MX_BLOCK 32

/* Value of an E4M3 code. */
double oracle_e4m3_value(uint8_t c) {
  const int s = c >> 7, e = (c >> 3) & 15, m = c & 7;
  if (e == 15 && m == 7) return NAN;
  double v = e == 0 ? ldexp((double)m, -9) : ldexp(1.0 + m / 8.0, e - 7);
  return s ? -v : v;
}

/* Nearest E4M3 code to v (ties to the even code, i.e. the even mantissa), saturating.  The
 * non-negative finite codes 0..126 are in increasing order of value, so the nearest one is
 * found by a plain search. */
uint8_t oracle_e4m3_code(float v) {
  const uint8_t sign = signbit(v) ? 0x80 : 0x00;
  const double a = fabs((double)v);
  if (a >= 448.0) return sign | 126;
  int best = 0;
  double bd = a;
  for (int c = 1; c <= 126; ++c) {
    const double dist = fabs(oracle_e4m3_value((uint8_t)c) - a);
    if (dist < bd || (dist == bd && (c & 1) == 0)) { best = c; bd = dist; }
  }
  return sign | (uint8_t)best;
}

/* Value of an E8M0 scale code: 2^(c - 127); 255 is NaN. */
double oracle_e8m0_value(uint8_t c) { return c == 255 ? NAN : ldexp(1.0, (int)c - 127); }

/* E8M0 code of the shared scale of the block v[0..len). */
uint8_t oracle_mx_scale_code(const float* v, int len) {
  float amax = 0.0f;
  for (int j = 0; j < len; ++j) {
    const float a = fabsf(v[j]);
    if (a > amax) amax = a;
  }
  if (amax == 0.0f) return 127;
  int ex;
  const double f = frexp((double)amax, &ex);  /* amax = f 2^ex, f in [0.5, 1) */
  /* amax <= 448 2^E = 0.875 2^(E + 9): the smallest such E */
  int E = f <= 0.875 ? ex - 9 : ex - 8;
  if (E < -127) E = -127;
  if (E > 127) E = 127;
  return (uint8_t)(E + 127);
}

/* One row of cols values (cols a multiple of 32): codes q[cols], scale codes sf[cols / 32]. */
static void mx_quantize_row(const float* v, int64_t cols, uint8_t* q, uint8_t* sf) {
  for (int64_t b = 0; b < cols / MX_BLOCK; ++b) {
    const float* vb = v + b * MX_BLOCK;
    const uint8_t c = oracle_mx_scale_code(vb, MX_BLOCK);
    const double X = oracle_e8m0_value(c);
    sf[b] = c;
    for (int j = 0; j < MX_BLOCK; ++j) q[b * MX_BLOCK + j] = oracle_e4m3_code((float)(vb[j] / X));
  }
}

/* Block quantisation of a [rows][cols] matrix of dtype (bf16 or fp32) values; cols % 32 == 0.
 * q [rows][cols] E4M3 codes, sf [rows][cols / 32] E8M0 codes. */
void oracle_quantize_mx_e4m3(int64_t rows, int64_t cols, int dtype, const void* v, uint8_t* q,
                             uint8_t* sf) {
#pragma omp parallel
  {
    float* row = (float*)malloc(sizeof(float) * cols);
#pragma omp for schedule(static)
    for (int64_t r = 0; r < rows; ++r) {
      if (!row) continue;
      for (int64_t j = 0; j < cols; ++j) row[j] = (float)elem(v, dtype, r * cols + j);
      mx_quantize_row(row, cols, q + r * cols, sf + r * (cols / MX_BLOCK));
    }
    free(row);
  }
}

/* sum over the blocks of (X_a,b X_w,b sum_{j in b} P_a,j P_w,j) for rows of len elements. */
static double mx_dot(const uint8_t* qa, const uint8_t* sa, const uint8_t* qw, const uint8_t* sw,
                     int64_t len, const double* lut) {
  double total = 0.0;
  for (int64_t b = 0; b < len / MX_BLOCK; ++b) {
    double s = 0.0;
    for (int j = 0; j < MX_BLOCK; ++j) s += lut[qa[b * MX_BLOCK + j]] * lut[qw[b * MX_BLOCK + j]];
    total += oracle_e8m0_value(sa[b]) * oracle_e8m0_value(sw[b]) * s;
  }
  return total;
}

/* The block with FP8 expert weights for the tokens tok[0..n_tok): y[r][0..d) in double
 * (unrounded).  x bf16 [T][d]; W1q, W3q [n][F][d] and W2q [n][d][F] E4M3 codes; sf1, sf3
 * [n][F][d / 32] and sf2 [n][d][F / 32] E8M0 block-scale codes.  d and F multiples of 32. */
int oracle_moe_forward_fp8(int64_t T, int64_t d, int64_t F, int n, int K, const void* x,
                           const float* Wg, const uint8_t* W1q, const uint8_t* W3q,
                           const uint8_t* W2q, const uint8_t* sf1, const uint8_t* sf3,
                           const uint8_t* sf2, int64_t n_tok, const int64_t* tok, double* y,
                           int32_t* idx_out, double* gate_out) {
  if (n < 1 || n > 256 || K < 1 || K > n || d % MX_BLOCK || F % MX_BLOCK) return 1;
  for (int64_t r = 0; r < n_tok; ++r) if (tok[r] < 0 || tok[r] >= T) return 2;
  double lut[256];
  for (int c = 0; c < 256; ++c) lut[c] = oracle_e4m3_value((uint8_t)c);
  const int64_t bd = d / MX_BLOCK, bf = F / MX_BLOCK;
  int fail = 0;
#pragma omp parallel
  {
    float* xf = (float*)malloc(sizeof(float) * d);
    uint8_t* qx = (uint8_t*)malloc(d);
    uint8_t* sx = (uint8_t*)malloc(bd);
    float* hf = (float*)malloc(sizeof(float) * F);
    uint8_t* qh = (uint8_t*)malloc(F);
    uint8_t* sh = (uint8_t*)malloc(bf);
    const int ok = xf && qx && sx && hf && qh && sh;
    if (!ok) {
#pragma omp atomic write
      fail = 1;
    }
#pragma omp for schedule(dynamic, 1)
    for (int64_t r = 0; r < n_tok; ++r) {
      if (!ok) continue;
      const int64_t t = tok[r];
      double l[256], gate[256];
      int32_t idx[256];
      router_logits(d, n, ORACLE_BF16, x, t, Wg, l);
      topk_softmax(n, K, l, idx, gate);
      for (int64_t j = 0; j < d; ++j) xf[j] = (float)elem(x, ORACLE_BF16, t * d + j);
      mx_quantize_row(xf, d, qx, sx);
      double* yr = y + r * d;
      for (int64_t i = 0; i < d; ++i) yr[i] = 0.0;
      for (int k = 0; k < K; ++k) {
        const int e = idx[k];
        for (int64_t f = 0; f < F; ++f) {
          const int64_t wr = (int64_t)e * F + f;
          const double a = mx_dot(qx, sx, W1q + wr * d, sf1 + wr * bd, d, lut);
          const double b = mx_dot(qx, sx, W3q + wr * d, sf3 + wr * bd, d, lut);
          hf[f] = (float)(oracle_silu(a) * b);
        }
        mx_quantize_row(hf, F, qh, sh);
        for (int64_t i = 0; i < d; ++i) {
          const int64_t wr = (int64_t)e * d + i;
          yr[i] += gate[k] * mx_dot(qh, sh, W2q + wr * F, sf2 + wr * bf, F, lut);
        }
      }
      for (int k = 0; k < K; ++k) {
        if (idx_out) idx_out[r * K + k] = idx[k];
        if (gate_out) gate_out[r * K + k] = gate[k];
      }
    }
    free(xf);
    free(qx);
    free(sx);
    free(hf);
    free(qh);
    free(sh);
  }
  return fail ? 3 : 0;
}
