/*
 * moe.h -- C ABI of the B200 (sm_100a) sparse Mixture-of-Experts block library (libmoe.so).
 *
 * What is computed, per token x (a row of the activation matrix), as defined in
 * "Mixtral of Experts" (arXiv 2401.04088; the xyznot.com summary page of that title, method
 * section, equations G(x) and y):
 *
 *   l    = x . W_g                         router logits over n experts, fp32, no bias
 *   G(x) = Softmax(TopK(l))                TopK keeps the K largest logits (others -inf);
 *                                          Mixtral uses K = 2 of n = 8
 *   y    = sum_i G(x)_i * SwiGLU_i(x),     SwiGLU_i(x) = W2_i . (silu(W1_i . x) * (W3_i . x))
 *
 * Experts whose gate is zero are not evaluated ("Mixtral 8x7B: Model Bahasa Sparse Mixture of
 * Experts", id.news.hada.io, section "Cara Komputasi Layer MoE": outputs of zero-gate experts
 * need not be computed); tokens are grouped per expert instead (same page, section
 * "Implementasi dan Efisiensi Inferensi": the number of tokens per expert varies).
 * Below, "the method section" is the xyznot.com page's and "the hada.io page" is the
 * Indonesian summary.
 *
 * Conventions shared by every entry point
 * ---------------------------------------
 *  - Every pointer argument not marked "host" is a DEVICE pointer on the current CUDA device.
 *  - Layouts are row-major:  x, out [T][d];  W_g [d][n] (always fp32);
 *    W1, W3 [n][F][d];  W2 [n][d][F].  x, W1, W3, W2 and out share the dtype `dt`.
 *  - Ties in TopK go to the lower expert index; slot 0 holds the larger logit.
 *  - bf16 path: fp32 accumulation on the tensor cores; h = silu(a) * b is rounded to bf16
 *    before the down-projection; each token's gated sum is accumulated in fp32 and rounded
 *    once to bf16.  fp32 path: fp32 everywhere (no TF32).
 *  - The caller owns all memory, including a workspace of at least moe_workspace_bytes()
 *    bytes (256-byte aligned) that must be initialised once with moe_workspace_init().
 *    The library never allocates or frees memory and never synchronises the stream on the
 *    forward path; all work is enqueued on `stream` (a cudaStream_t; NULL = legacy stream).
 *  - Argument errors are detected on the host before anything is enqueued and returned
 *    synchronously.  Launch errors return MOE_ERR_CUDA.  Faults detected inside kernels
 *    (a bounded wait that ran out, an index out of range) set bits in a status word in the
 *    workspace; moe_workspace_status() synchronises the stream, reads and clears it.
 *  - T = 0 is a valid no-op.  Requirements: 1 <= n <= 64, 1 <= K <= n, d and F multiples
 *    of 64 on the bf16 path and of 8 on the fp32 path; otherwise MOE_ERR_UNSUPPORTED.
 *  - out must not alias x.  Calls sharing one workspace must not overlap on the GPU.
 *  - Thread safety: no mutable global state; concurrent calls need separate workspaces.
 *  - Environment: MOE_GATHER_X=1 (read at every call) switches large batches (T*K >= 640 n,
 *    bf16) to an alternative data path: the up-projection gathers its activation rows from x
 *    by token (TMA tile::gather4) instead of reading a permuted copy, and the
 *    down-projection applies the gates.  Same results within rounding, same workspace size;
 *    slower on B200 (the default is the permuted copy).  The pages describe grouping the
 *    tokens per expert but fix no data path between the grouping and the expert GEMMs.
 */
#ifndef MOE_B200_H
#define MOE_B200_H

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define MOE_API __attribute__((visibility("default")))
#else
#define MOE_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  MOE_OK = 0,
  MOE_ERR_INVALID_ARG = 1, /* null pointer, bad size, misaligned pointer */
  MOE_ERR_UNSUPPORTED = 2, /* shape outside the supported set (see above) */
  MOE_ERR_WORKSPACE = 3,   /* workspace smaller than moe_workspace_bytes() */
  MOE_ERR_CUDA = 4,        /* a CUDA runtime call or kernel launch failed */
  MOE_ERR_TIMEOUT = 5,     /* a kernel's bounded wait ran out (reported by status calls) */
  MOE_ERR_DEVICE = 6       /* a kernel detected an out-of-range index (status calls) */
} moe_status;

typedef enum { MOE_F32 = 0, MOE_BF16 = 1 } moe_dtype;

/* Workspace plumbing (the pages have no counterpart: the caller-owned scratch memory of the
 * grouping and expert stages below).
 * Bytes of device workspace moe_forward / moe_forward_debug need for this shape
 * (0 if the shape is unsupported).  moe_stack_forward needs moe_stack_workspace_bytes(). */
MOE_API size_t moe_workspace_bytes(int64_t T, int64_t d, int64_t F, int n, int K, moe_dtype dt);

/* Zero the workspace's status word and counters (enqueued on `stream`); call once after
 * allocating it, and again after any error that moe_workspace_status() reports. */
MOE_API moe_status moe_workspace_init(void* workspace, size_t workspace_bytes, void* stream);

/* Synchronise `stream`, then read the workspace status word written by kernels and, if it is
 * not zero, clear it (the clear is enqueued on `stream`).  Returns MOE_OK, MOE_ERR_TIMEOUT (a
 * bounded wait ran out), MOE_ERR_DEVICE (an index out of range) or MOE_ERR_CUDA (the stream
 * reported an error).  *raw (may be NULL) receives the raw bit mask (bit 0: a wait ran out;
 * bit 1: an expert index outside [0, n); bit 2: a permuted row outside the workspace).
 * After any error, call moe_workspace_init() again before reusing the workspace (an
 * interrupted call can leave its counters mid-count). */
MOE_API moe_status moe_workspace_status(void* workspace, void* stream, uint32_t* raw);

/* One MoE block forward:  out[t] = sum_k G(x_t)_k * SwiGLU_{e_k}(x_t)
 * (the method section, equations G(x) = Softmax(TopK(x . W_g)) and y; the hada.io page,
 * "Cara Komputasi Layer MoE": softmax over the top-K logits of a linear layer, K = 2).
 *   x    [T][d]   dt           token activations
 *   W_g  [d][n]   fp32         router weight
 *   W1   [n][F][d] dt          gate projection of each expert
 *   W3   [n][F][d] dt          up projection of each expert
 *   W2   [n][d][F] dt          down projection of each expert
 *   out  [T][d]   dt           result (written, never read)
 * Device pointers; x/W1/W3/W2/out 16-byte aligned, workspace 256-byte aligned. */
MOE_API moe_status moe_forward(const void* x, const float* W_g, const void* W1, const void* W3,
                       const void* W2, int64_t T, int64_t d, int64_t F, int n, int K,
                       moe_dtype dt, void* out, void* workspace, size_t workspace_bytes,
                       void* stream);

/* moe_forward, then copies of the routing state into caller buffers (each may be NULL) --
 * the router's choice G(x) (method section, equation G(x)) and the per-expert grouping of
 * the tokens (hada.io page, "Implementasi dan Efisiensi Inferensi"):
 *   topk_idx [T][K] int32      selected experts, slot 0 = larger logit
 *   topk_gate [T][K] fp32      G(x) over the kept experts (rows sum to 1)
 *   expert_counts [n] int32    tokens routed to each expert
 *   expert_offsets [n+1] int32 first row of each expert's group in the permuted layout
 *   token_rows [T][K] int32    permuted row of each (token, slot)
 * Enqueued on `stream` like moe_forward (no synchronisation). */
MOE_API moe_status moe_forward_debug(const void* x, const float* W_g, const void* W1,
                             const void* W3, const void* W2, int64_t T, int64_t d, int64_t F,
                             int n, int K, moe_dtype dt, void* out, void* workspace,
                             size_t workspace_bytes,
                             void* stream, int32_t* topk_idx, float* topk_gate,
                             int32_t* expert_counts, int32_t* expert_offsets,
                             int32_t* token_rows);

/* ---- FP8 expert weights (a variant for decode bandwidth; the pages only mention quantised
 * community builds -- the reader comments on the hada.io page -- and fix no format, so the
 * format is this library's plain reading): MXFP8, the OCP Microscaling format with FP8 E4M3
 * elements (1 sign, 4 exponent bits with bias 7, 3 mantissa bits, no infinities, largest
 * finite 448) in blocks of 32 consecutive elements of a row sharing one E8M0 scale X = 2^E
 * (code E + 127):
 *   E = the smallest integer with max_j |w_j| <= 448 2^E (no element overflows), clamped to
 *   [-127, 127] (E = 0 for an all-zero block);
 *   code_j = E4M3(w_j / X), nearest, ties to even, saturating;  w_j ~ X value(code_j).
 * The block quantises each token's x row and each h row the same way on the device, and the
 * tensor cores apply both operands' block scales in the MMA (tcgen05 kind::mxf8f6f4,
 * block_scale), accumulating in fp32:
 *   a_f = sum_blocks X_x X_1,f sum_j x_q,j W1q_f,j,  b_f likewise,  h_f = silu(a_f) b_f,
 *   y_i = sum_blocks X_h X_2,i sum_f h_q,f W2q_i,f,  out = sum_k G_k y_{e_k} rounded once.
 * Routing is the bf16 block's (bf16 x, fp32 W_g).
 *
 * Scale layout ("tile order", what the tensor cores' scale copies read): for a [rows][cols]
 * matrix (both multiples of 128) the scale code of row r, elements [32c, 32c + 32) is the byte
 *   ((r / 128) * (cols / 128) + c / 4) * 512 + 16 * (r % 32) + 4 * ((r % 128) / 32) + c % 4,
 * i.e. one 512-byte chunk per 128 rows x 128 columns. */

/* MXFP8 codes and block scales of a [rows][cols] bf16 matrix v (device pointers; rows and
 * cols multiples of 128; v 8-byte, q 4-byte and sf 16-byte aligned): q [rows][cols] uint8,
 * sf rows * cols / 32 bytes in tile order.  Enqueued on `stream`.  Use it once on W1 and W3
 * (as [n*F][d]) and W2 (as [n*d][F]). */
MOE_API moe_status moe_quantize_mx_e4m3(const void* v, int64_t rows, int64_t cols, uint8_t* q,
                                        uint8_t* sf, void* stream);

/* Workspace bytes for moe_forward_fp8 (0 if unsupported).  Supported: the small-batch
 * decode shapes (T <= 64, T*K <= 1024 and T*K < 64 n), d and F multiples of 128. */
MOE_API size_t moe_workspace_bytes_fp8(int64_t T, int64_t d, int64_t F, int n, int K);

/* The block with MXFP8 expert weights:
 *   x [T][d] bf16, W_g [d][n] fp32, W1q, W3q [n][F][d] and W2q [n][d][F] E4M3 codes,
 *   sf1, sf3 (of [n*F][d]) and sf2 (of [n*d][F]) their block scales in tile order as
 *   moe_quantize_mx_e4m3 writes them (16-byte aligned), out [T][d] bf16.
 * events: NULL / 0, or six cudaEvent_t recorded at the stage boundaries (routing, G13,
 * SwiGLU + h quantisation, G2, combine), as moe_forward_profiled.  Other conventions as
 * moe_forward; shapes outside the supported set return MOE_ERR_UNSUPPORTED. */
MOE_API moe_status moe_forward_fp8(const void* x, const float* W_g, const uint8_t* W1q,
                                   const uint8_t* W3q, const uint8_t* W2q, const uint8_t* sf1,
                                   const uint8_t* sf3, const uint8_t* sf2, int64_t T, int64_t d,
                                   int64_t F, int n, int K, void* out, void* workspace,
                                   size_t workspace_bytes, void* stream, void* const* events,
                                   int n_events);

/* moe_forward with HOST input and output (the block as in moe_forward; the host copies are
 * plumbing with no counterpart in the pages): copies x_host (pinned recommended) to x_dev,
 * runs the block into out_dev and copies it back to out_host, all on `stream`; returns
 * after enqueueing (synchronise the stream before reading out_host).  x_dev and out_dev
 * are caller-owned device buffers of T*d elements. */
MOE_API moe_status moe_forward_host_io(const void* x_host, void* x_dev, const float* W_g,
                               const void* W1, const void* W3, const void* W2, int64_t T,
                               int64_t d, int64_t F, int n, int K, moe_dtype dt,
                               void* out_dev, void* out_host, void* workspace,
                               size_t workspace_bytes, void* stream);

/* moe_forward that also records caller-created CUDA events (cudaEvent_t, passed as void*)
 * on `stream` at the stage boundaries, for timing each kernel live (measurement plumbing; the
 * stages are those of moe_forward):
 *   events[0] before routing            events[1] after router, scan and permute
 *   events[2] after the gate/up GEMM    events[3] after the split-K reduction (== [2] when
 *                                                  the small-batch tiling is not used)
 *   events[4] after the down GEMM       events[5] after the combine
 * n_events must be 6.  Otherwise identical to moe_forward. */
MOE_API moe_status moe_forward_profiled(const void* x, const float* W_g, const void* W1,
                                        const void* W3, const void* W2, int64_t T, int64_t d,
                                        int64_t F, int n, int K, moe_dtype dt, void* out,
                                        void* workspace, size_t workspace_bytes, void* stream,
                                        void* const* events, int n_events);

/* Work plan chosen for a shape (for reports; no counterpart in the pages):
 *   *small_batch = 1 if the weights are the MMA's 128-row operand (small token counts);
 *   *split13 / *split2 = K-splits of the two expert GEMMs on that path (1 otherwise);
 *   *launches = kernels one forward launches (a stack of them launches one more, the first
 *              block's RMSNorm, on the large-batch tilings);
 *   *tiling = the expert GEMMs' tiling: 0 = 128-row token tiles (or the small-batch tiles
 *             when *small_batch = 1), 1 = CTA pairs (256-row token tiles), 2 = mid-size
 *             weight-stationary tiles (128 weight rows as the MMA's M, up to 256 of an
 *             expert's token rows as its N).
 * Any output may be NULL. */
MOE_API moe_status moe_plan_info(int64_t T, int64_t d, int64_t F, int n, int K, moe_dtype dt,
                                 int* small_batch, int* split13, int* split2, int* launches,
                                 int* tiling);

/* Stack of L blocks on a residual stream (attention omitted), in place on x [T][d]:
 *   for l in 0..L-1:  x <- round(x + MoE_l(RMSNorm(x)))
 * The pages say only that every one of Mixtral's 32 layers replaces its feed-forward block
 * with this MoE block (hada.io page, "Arsitektur Sparse Mixture of Experts"); the RMSNorm ->
 * MoE -> residual stacking with attention left out is the library's stacked-block workload,
 * not a passage of the pages.  RMSNorm has unit gain: x / sqrt(mean(x^2) + eps), rounded to
 * dt; the residual sum is taken in fp32 and rounded once.  W_g, W1, W3, W2 are HOST arrays
 * of L device pointers (per-layer weights, layouts as above).  Only the bf16 path is
 * supported. */
MOE_API size_t moe_stack_workspace_bytes(int64_t T, int64_t d, int64_t F, int n, int K,
                                 moe_dtype dt);
MOE_API moe_status moe_stack_forward(void* x, const float* const* W_g, const void* const* W1,
                             const void* const* W3, const void* const* W2, int L, int64_t T,
                             int64_t d, int64_t F, int n, int K, moe_dtype dt, float eps,
                             void* workspace, size_t workspace_bytes, void* stream);

/* moe_stack_forward that records caller-created CUDA events at every block's stage
 * boundaries (measurement plumbing): events[6*l + j] is block l's event j as in
 * moe_forward_profiled (the block's RMSNorm runs just before events[6*l]).
 * n_events must be 6*L. */
MOE_API moe_status moe_stack_forward_profiled(void* x, const float* const* W_g,
                                              const void* const* W1, const void* const* W3,
                                              const void* const* W2, int L, int64_t T,
                                              int64_t d, int64_t F, int n, int K, moe_dtype dt,
                                              float eps, void* workspace,
                                              size_t workspace_bytes, void* stream,
                                              void* const* events, int n_events);

/* moe_stack_forward with HOST input and output (host copies are plumbing): copies x_host
 * (T*d bf16, pinned recommended) to the caller's device buffer x_dev, runs the L blocks in
 * place on x_dev and copies the result to out_host, all enqueued on `stream`; returns after
 * enqueueing (synchronise the stream before reading out_host). */
MOE_API moe_status moe_stack_forward_host_io(const void* x_host, void* x_dev,
                                             const float* const* W_g, const void* const* W1,
                                             const void* const* W3, const void* const* W2,
                                             int L, int64_t T, int64_t d, int64_t F, int n,
                                             int K, moe_dtype dt, float eps, void* out_host,
                                             void* workspace, size_t workspace_bytes,
                                             void* stream);

/* ---- Expert parallelism: the block's stages as separate calls, so that the experts can be
 * spread over GPUs with an exchange between them ("Mixtral 8x7B: Model Bahasa Sparse Mixture
 * of Experts", id.news.hada.io, section "Implementasi dan Efisiensi Inferensi": tokens are
 * sent to the GPU that holds their expert and the expert outputs return to the tokens'
 * original positions).  The exchanges themselves are the caller's (e.g. NCCL all-to-alls);
 * moe_route -> [dispatch] -> moe_experts_forward -> [return] -> moe_combine on one GPU gives
 * moe_forward's result within rounding.
 *
 * Workspace bytes of moe_route (0 if unsupported). */
MOE_API size_t moe_route_workspace_bytes(int64_t T, int64_t d, int n, int K, moe_dtype dt);

/* The router, TopK and softmax of every token (method section, equation G(x)) and the
 * grouping of the T*K (token, slot) rows by expert, unpadded and stable (by token, then
 * slot): expert e's rows are x_grouped[o_e .. o_e + expert_counts[e]), o_e = sum of the
 * counts of the experts before e.
 *   x [T][d] dt, W_g [d][n] fp32            inputs (x 16-byte aligned)
 *   x_grouped [T*K][d] dt                   the token rows in grouped order (must not alias x)
 *   topk_idx, token_rows [T][K] int32       selected experts; row of each (token, slot)
 *   topk_gate [T][K] fp32                   G(x) over the kept experts
 *   expert_counts [n] int32
 * Requirements as moe_forward (d a multiple of 64 for bf16, 8 for fp32). */
MOE_API moe_status moe_route(const void* x, const float* W_g, int64_t T, int64_t d, int n,
                             int K, moe_dtype dt, void* x_grouped, int32_t* topk_idx,
                             float* topk_gate, int32_t* expert_counts, int32_t* token_rows,
                             void* workspace, size_t workspace_bytes, void* stream);

/* Workspace bytes of moe_experts_forward for `rows` received rows (0 if unsupported). */
MOE_API size_t moe_experts_workspace_bytes(int64_t rows, int64_t d, int64_t F, int n_local,
                                           moe_dtype dt);

/* The SwiGLU experts (method section, equation y; W2 . (silu(W1 . x) * (W3 . x))) of one
 * GPU's n_local experts on rows received from S sources:
 *   x_rows [rows][d] dt         S segments in source order; segment s holds seg_counts[s][e]
 *                               rows for local expert e = 0 .. n_local-1, in expert order
 *   seg_counts [S][n_local]     int32, device (S * n_local <= 2048; they must add up to rows,
 *                               else bit 2 of the status word is set and nothing is computed)
 *   W1, W3 [n_local][F][d], W2 [n_local][d][F] dt   the local experts' weights
 *   y_rows [rows][d] fp32       y_rows[r] = SwiGLU_e(x_rows[r]), same row order, no gate
 * The rows are regrouped on the device into the padded per-expert layout of the grouped
 * GEMMs (the same kernels and tilings as moe_forward for `rows` rows over n_local experts). */
MOE_API moe_status moe_experts_forward(const void* x_rows, int64_t rows,
                                       const int32_t* seg_counts, int S, const void* W1,
                                       const void* W3, const void* W2, int64_t d, int64_t F,
                                       int n_local, moe_dtype dt, float* y_rows, void* workspace,
                                       size_t workspace_bytes, void* stream);

/* The gate-weighted combine back to token order (method section, equation y):
 *   out[t] = sum_k topk_gate[t][k] * y_rows[token_rows[t][k]]
 * summed in fp32 in slot order and rounded once to dt (out [T][d], 16-byte aligned; y_rows
 * fp32, 16-byte aligned; d a multiple of 4).  No workspace. */
MOE_API moe_status moe_combine(const float* y_rows, const int32_t* token_rows,
                               const float* topk_gate, int64_t T, int64_t d, int K, moe_dtype dt,
                               void* out, void* stream);

/* Row gather for the expert-parallel exchange when experts are replicated over ranks (the
 * hada.io page, "Implementasi dan Efisiensi Inferensi": the load across GPUs must be
 * balanced; moving rows is plumbing): out[i] = in[index[i]] for 0 <= i < rows, each row
 * row_bytes bytes (a multiple of 16); in has in_rows rows; an index outside [0, in_rows)
 * leaves out row i unwritten.  Device pointers: in and out 16-byte aligned and distinct,
 * index int32 4-byte aligned.  Enqueued on `stream`; MOE_ERR_INVALID_ARG on bad arguments
 * before any launch. */
MOE_API moe_status moe_gather_rows(const void* in, int64_t in_rows, const int32_t* index,
                                   int64_t rows, int64_t row_bytes, void* out, void* stream);

/* Test hook for the failure path (no counterpart in the pages): moe_forward, except that the
 * one-CTA tensor-core kernel of the gate/up projection issues none of its loads, so its
 * tensor-core thread waits on a barrier that nothing will complete; that wait, and the other
 * pipeline waits of the kernel, give up after wait_limit_cycles (1 .. 4e9 SM clock cycles).
 * The kernel then records bit 0 in the status word, lets nothing in flight outlive it, frees
 * its tensor memory and returns; the rest of the block runs on undefined values.  Expect
 * moe_workspace_status() == MOE_ERR_TIMEOUT afterwards, then call moe_workspace_init().
 * Shapes that take the CTA-pair or fp32 kernels return MOE_ERR_UNSUPPORTED. */
MOE_API moe_status moe_debug_forward_withheld(const void* x, const float* W_g, const void* W1,
                                              const void* W3, const void* W2, int64_t T,
                                              int64_t d, int64_t F, int n, int K, moe_dtype dt,
                                              void* out, void* workspace,
                                              size_t workspace_bytes, void* stream,
                                              int64_t wait_limit_cycles);

/* moe_forward without a caller-supplied workspace, for callers that cannot allocate device
 * memory (e.g. a plugin inside an application whose own pool owns every allocation, or a
 * loop that must never call cudaMalloc because it can synchronise the device).  The paper
 * has no counterpart to this entry point; it exists only for such callers.
 *   - The workspace is a fixed device array of MOE_NOALLOC_WORKSPACE_BYTES inside the
 *     library; every GPU that loads the library holds it until the process exits.  Shapes
 *     whose moe_workspace_bytes() exceeds it return MOE_ERR_WORKSPACE (at Mixtral's sizes it
 *     fits decode batches of up to 24 tokens).
 *   - Every call looks up the array's device address on the current device.  The first call
 *     on a device (and the first after the context was re-created) also zeroes the array's
 *     256-byte header with an asynchronous memset enqueued on `stream`, ahead of that call's
 *     kernels; make that first call before any stream capture.  Nothing is allocated, and
 *     nothing is freed.
 *   - All calls share the one array and it keeps the last call's contents: calls that
 *     overlap on the GPU (other streams, other threads) race on it.
 *   - Faults that kernels detect go to the array's status word: read them with
 *     moe_noalloc_status().
 * Arguments, layouts and errors otherwise as moe_forward. */
#define MOE_NOALLOC_WORKSPACE_BYTES (32u << 20)
MOE_API moe_status moe_forward_noalloc(const void* x, const float* W_g, const void* W1,
                                       const void* W3, const void* W2, int64_t T, int64_t d,
                                       int64_t F, int n, int K, moe_dtype dt, void* out,
                                       void* stream);

/* moe_workspace_status() for the array moe_forward_noalloc uses (the paper has no
 * counterpart): synchronises `stream`, reads and clears the status word.  On an error it
 * also zeroes the array's header (status word and counters) on `stream` and synchronises,
 * so the next moe_forward_noalloc starts clean. */
MOE_API moe_status moe_noalloc_status(void* stream, uint32_t* raw);

/* Short description of a status code (static string). */
MOE_API const char* moe_status_string(moe_status s);

/* Library ABI version (increases when an entry point changes). */
MOE_API int moe_abi_version(void);

#ifdef __cplusplus
}
#endif

#endif /* MOE_B200_H */
