// gemm_tc.cu -- grouped expert GEMMs on the sm_100a tensor cores (tcgen05 + TMEM + TMA).
//
// Each expert is a SwiGLU FFN of intermediate width F ("Mixtral of Experts", method
// section: n = 8 experts of width 14336 on hidden size 4096; glossary: Swish combined with
// an element-wise product):
//   G13:  h = silu(X_e . W1_e^T) * (X_e . W3_e^T)      rounded to bf16
//   G2:   Y = h_e . W2_e^T                              kept in fp32
// where X_e are the rows routed to expert e (grouped by the permute kernel).
//
// Persistent kernels, one CTA (or CTA pair) per SM, warp-specialised:
//   warp 0      TMA producer filling a ring of shared-memory stages,
//   warp 1      owns the TMEM allocation; one thread issues tcgen05.mma,
//   the rest    epilogue: tcgen05.ld of the fp32 accumulators, SwiGLU / store.
// All waits are bounded (see common.cuh).
//
// Tilings (chosen per call from the shape, see make_plan):
//   128-row tiles (tc_grouped_gemm_kernel, !SWAP): tile = 128 permuted rows x (G13: 128
//     columns of W1 and the same 128 of W3, stacked into one N = 256 MMA operand | G2: 256
//     columns of W2), full K per tile, accumulators double-buffered in TMEM.
//   small batch (tc_grouped_gemm_kernel, SWAP): the weights are the 128-row MMA operand and
//     the expert's tokens the N dimension (16..256), K split into `splits` ranges so that
//     every SM streams weights; fp32 partial sums go to per-split slabs reduced in a fixed
//     order afterwards.  With MXFP8 weights the operands are E4M3 codes with E8M0 block
//     scales, applied by the MMA (kind::mxf8f6f4 block_scale).
//   mid-size groups (tc_grouped_gemm_kernel, SWAP with `mid`): the same orientation without
//     the K split: a unit is (expert, 128 weight rows, pass of up to tok_tile of the expert's
//     rows), each weight byte streamed once per pass; G13 writes h itself.
//   CTA pairs (tc_pair_gemm_kernel): cta_group::2 tiles of 256 rows x two 256-column blocks,
//     M = 128 tiles for an expert's last 128 rows (see the section below).
#include <stdio.h>

#include "internal.h"

namespace moe {

enum { KIND_G13 = 0, KIND_G2 = 1 };
constexpr int MAX_STAGES = 16;
constexpr int GEMM_THREADS = 192;
constexpr uint32_t TILE_BYTES = 128 * 128;  // 128 rows x 64 bf16 (one 128-byte row each)

struct TcArgs {
  const int32_t* offsets;  // [n+1] first permuted row of each expert
  int n;
  int num_kb;              // 64-wide K blocks per work unit
  int nw;                  // weight rows (output features) per expert: F (G13) or d (G2)
  int n_tiles;             // prefill: column tiles per row tile (pairs: column-block pairs)
  int n_blocks;            // CTA pairs: column blocks per expert, two per tile
  int wb;                  // small batch: 128-row weight blocks per expert
  int splits;              // small batch: K ranges
  int tok_tile;            // small batch: MMA N
  int stages;
  uint32_t stage_bytes;    // shared-memory bytes per stage (1024-aligned)
  uint32_t tx_bytes;       // bytes the TMA loads of one stage deliver
  uint32_t x_off;          // offset of the activation tile inside a stage
  uint32_t acc_cols, nacc, tmem_cols;
  void* out;
  int64_t out_ld;          // elements per output row
  int64_t split_stride;    // elements between split slabs
  uint32_t* status;
  // CTA pairs reading x directly (G13: row_tok, counts, gather_T) and applying the gates
  // (G2: row_gate); null otherwise
  const int32_t* row_tok;  // token of each permuted row
  const int32_t* counts;   // [n] rows routed to each expert
  int gather_T;            // rows of x (a row index past the end reads zeros)
  const float* row_gate;   // gate of each permuted row
  int gather_rows;         // small batch gathering from x: permuted rows (T*K)
  // one-CTA kernel: cycles a pipeline wait may last before the kernel gives up
  // (WAIT_LIMIT_CYCLES), and the failure-path test hook: withhold_loads = 1 makes the
  // producer issue no load at all, so the MMA thread's first wait is on a barrier nothing
  // will complete and runs out after wait_limit cycles (0 on every forward call)
  long long wait_limit = WAIT_LIMIT_CYCLES;
  int withhold_loads = 0;
  // weight-stationary tiles for mid-size groups (SWAP kernels): an expert's rows are taken
  // in passes of up to tok_tile, each MMA's N is its pass's rows rounded up to 16, B rows come
  // in 64-row boxes, and G13 writes h = bf16(silu(a) b) itself (no split-K)
  int mid = 0;
  // MXFP8 (E4M3 kernels): E8M0 block scales of the A rows (W1 or W2; sfa1: W3) in the tensor
  // cores' tile order, one 512-byte chunk per (128-row tile, 128-wide K block); of the B rows
  // (the expert's token or h rows) one 512-byte chunk per (expert, K block), row slot j at
  // byte 16 (j % 32) + 4 (j / 32); sf_kb K blocks per row; sf_off: their copies in a stage
  // (A0, A1, B at +0, +512, +1024); sf_col: first TMEM column of the scales (A0, A1, B at
  // +0, +4, +8)
  const uint8_t* sfa0 = nullptr;
  const uint8_t* sfa1 = nullptr;
  const uint8_t* sfb = nullptr;
  int sf_kb = 0;
  uint32_t sf_off = 0;
  uint32_t sf_col = 0;
};

struct Ctrl {
  uint64_t full[MAX_STAGES];
  uint64_t empty[MAX_STAGES];
  uint64_t tfull[2];
  uint64_t tempty[2];
  uint64_t mma_done;
  uint32_t issued[MAX_STAGES];
  uint32_t tmem_slot;
  int abort;
  int nact;
  int off[MAX_EXPERTS + 1];
  int act[MAX_EXPERTS];
  int pbase[MAX_EXPERTS + 1];  // mid: passes of the active experts before each
  // small batch gathering from x: the token of each row follows the block (gather_rows ints)
};

struct Work {
  int e, mt, nt, wblk, s, row0, count;
  int m;  // CTA pairs: MMA M of the tile (256, or 128 for an expert's last 128 rows)
          // (and s: the tile's first column block)
};

template <bool SWAP>
__device__ __forceinline__ int total_work(const TcArgs& a, const Ctrl* c) {
  if (SWAP) return a.mid ? c->pbase[c->nact] * a.wb : c->nact * a.wb * a.splits;
  return (c->off[a.n] / TILE_M) * a.n_tiles;
}

// Prefill order: expert-major, then column tile, then row tile (consecutive CTAs share the
// weight tile through L2).  Small-batch order: active expert, weight block, split.
template <bool SWAP>
__device__ __forceinline__ Work decode_work(const TcArgs& a, const Ctrl* c, int id) {
  Work w{};
  if (SWAP && a.mid) {
    // active expert, then weight block, then pass (the passes over one weight block run side
    // by side and share its stream through L2)
    int ai = 0;
    while (ai + 1 < c->nact && id >= c->pbase[ai + 1] * a.wb) ++ai;
    const int np = c->pbase[ai + 1] - c->pbase[ai];
    const int local = id - c->pbase[ai] * a.wb;
    const int pass = local % np;
    w.e = c->act[ai];
    w.wblk = local / np;
    w.s = 0;
    w.row0 = c->off[w.e] + pass * a.tok_tile;
    const int left = c->off[w.e + 1] - w.row0;
    w.count = left < a.tok_tile ? left : a.tok_tile;
  } else if (SWAP) {
    const int per = a.wb * a.splits;
    const int ai = id / per, rem = id % per;
    w.e = c->act[ai];
    w.wblk = rem / a.splits;
    w.s = rem % a.splits;
    w.row0 = c->off[w.e];
    w.count = c->off[w.e + 1] - c->off[w.e];
  } else {
    int e = 0;
    while (e + 1 < a.n && id >= (c->off[e + 1] / TILE_M) * a.n_tiles) ++e;
    const int mt0 = c->off[e] / TILE_M;
    const int mcnt = c->off[e + 1] / TILE_M - mt0;
    const int local = id - mt0 * a.n_tiles;
    w.e = e;
    w.nt = local / mcnt;
    w.mt = mt0 + local % mcnt;
    w.row0 = w.mt * TILE_M;
  }
  return w;
}

// E4M3 (small batch only): operands are FP8 codes (128 per 128-byte row, so a K block is 128
// elements wide) with one E8M0 scale per 32 elements of every row; each stage also brings the
// scales of its K block, which the MMA thread copies into TMEM (tcgen05.cp) ahead of the
// block-scaled MMAs (kind::mxf8f6f4), so the accumulators hold real sums.
template <int KIND, bool SWAP, bool E4M3 = false>
__global__ void __launch_bounds__(GEMM_THREADS, 1)
    tc_grouped_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                           const __grid_constant__ CUtensorMap tmW0,
                           const __grid_constant__ CUtensorMap tmW1, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  Ctrl* c = reinterpret_cast<Ctrl*>(smem + (size_t)a.stages * a.stage_bytes);
  int* gtok = reinterpret_cast<int*>(c + 1);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&c->full[s], 1);
      mbar_init(&c->empty[s], 1);
      c->issued[s] = 0;
    }
    for (int i = 0; i < 2; ++i) {
      mbar_init(&c->tfull[i], 1);
      mbar_init(&c->tempty[i], 128);
    }
    mbar_init(&c->mma_done, 1);
    c->abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW0);
    if (KIND == KIND_G13) tma_prefetch_desc(&tmW1);
  }
  if (warp == 1) {
    tmem_alloc(&c->tmem_slot, a.tmem_cols);
    tmem_relinquish();
  }
  pdl_wait();  // expert offsets and operands come from the previous kernels
  pdl_trigger();
  if (threadIdx.x <= a.n) c->off[threadIdx.x] = a.offsets[threadIdx.x];
  const bool gather = SWAP && KIND == KIND_G13 && a.row_tok != nullptr;
  if (gather)
    for (int i = threadIdx.x; i < a.gather_rows; i += blockDim.x) gtok[i] = a.row_tok[i];
  __syncthreads();
  if (threadIdx.x == 0) {
    int na = 0;
    c->pbase[0] = 0;
    for (int e = 0; e < a.n; ++e)
      if (c->off[e + 1] > c->off[e]) {
        c->act[na] = e;
        c->pbase[na + 1] = c->pbase[na] + (c->off[e + 1] - c->off[e] + a.tok_tile - 1) /
                                              (a.tok_tile > 0 ? a.tok_tile : 1);
        ++na;
      }
    c->nact = na;
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = c->tmem_slot;
  const int total = total_work<SWAP>(a, c);

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer
    if (lane == 0) {
      const uint64_t pol_w = SWAP ? policy_evict_first() : policy_evict_normal();
      const uint64_t pol_x = policy_evict_last();
      int stage = 0;
      uint32_t phase = 0;
      for (int id = blockIdx.x; id < total && !a.withhold_loads; id += gridDim.x) {
        const Work w = decode_work<SWAP>(a, c, id);
        // gathering: only the 4-row groups that hold this expert's rows are loaded; the MMA
        // columns of the other slots read whatever the stage holds and are never stored
        const int ngath = gather ? (w.count + 3) / 4 : 0;
        const int nbox = a.mid ? (w.count + MID_BOX - 1) / MID_BOX : 0;  // mid: boxes of B rows
        const uint32_t tx =
            gather ? a.tx_bytes - (uint32_t)(a.tok_tile / 4 - ngath) * 512u
            : a.mid ? a.tx_bytes - (uint32_t)(a.tok_tile / MID_BOX - nbox) * (MID_BOX * 128u)
                    : a.tx_bytes;
        bool ok = true;
        for (int kb = 0; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&c->empty[stage], phase ^ 1u, a.status, &c->abort, a.wait_limit)) {
            ok = false;
            break;
          }
          uint8_t* st = smem + (size_t)stage * a.stage_bytes;
          uint64_t* fb = &c->full[stage];
          mbar_arrive_expect_tx(fb, tx);
          const int k = (SWAP ? w.s * a.num_kb + kb : kb) * (E4M3 ? 128 : 64);
          if (!SWAP) {
            tma_load_2d(st, &tmX, fb, k, w.mt * TILE_M, pol_x);
            if (KIND == KIND_G13) {
              const int wr = w.e * a.nw + w.nt * 128;
              tma_load_2d(st + TILE_BYTES, &tmW0, fb, k, wr, pol_w);
              tma_load_2d(st + 2 * TILE_BYTES, &tmW1, fb, k, wr, pol_w);
            } else {
              tma_load_2d(st + TILE_BYTES, &tmW0, fb, k, w.e * a.nw + w.nt * 256, pol_w);
            }
          } else {
            const int wr = w.e * a.nw + w.wblk * 128;
            tma_load_2d(st, &tmW0, fb, k, wr, pol_w);
            if (KIND == KIND_G13) tma_load_2d(st + TILE_BYTES, &tmW1, fb, k, wr, pol_w);
            if constexpr (E4M3) {  // the K block's scale chunks (A rows, B row slots)
              const int kbg = w.s * a.num_kb + kb;
              const int64_t rt = ((int64_t)w.e * a.nw + w.wblk * 128) / 128;
              bulk_load(st + a.sf_off, a.sfa0 + (rt * a.sf_kb + kbg) * 512, 512, fb);
              if (KIND == KIND_G13)
                bulk_load(st + a.sf_off + 512, a.sfa1 + (rt * a.sf_kb + kbg) * 512, 512, fb);
              bulk_load(st + a.sf_off + 1024, a.sfb + ((int64_t)w.e * a.sf_kb + kbg) * 512, 512,
                        fb);
            }
            if (gather) {  // the expert's token rows straight from x, four per gather
              for (int g = 0; g < ngath; ++g) {
                int tk[4];
#pragma unroll
                for (int j = 0; j < 4; ++j)
                  tk[j] = 4 * g + j < w.count ? gtok[w.row0 + 4 * g + j] : a.gather_T;
                tma_gather4(st + a.x_off + g * 512, &tmX, fb, k, tk[0], tk[1], tk[2], tk[3],
                            pol_x);
              }
            } else if (a.mid) {
              for (int b = 0; b < nbox; ++b)
                tma_load_2d(st + a.x_off + b * (MID_BOX * 128), &tmX, fb, k,
                            w.row0 + MID_BOX * b, pol_x);
            } else {
              tma_load_2d(st + a.x_off, &tmX, fb, k, w.row0, pol_x);
            }
          }
          c->issued[stage] += 1;
          if (++stage == a.stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
      }
      if (c->abort) {  // let every issued copy land before the CTA's shared memory goes away
        for (int s = 0; s < a.stages; ++s)
          if (c->issued[s]) wait_short(&c->full[s], (c->issued[s] - 1u) & 1u);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer
    if (lane == 0) {
      const uint32_t idesc = umma_idesc_bf16(128, SWAP ? a.tok_tile : 256);
      int stage = 0, it = 0;
      uint32_t phase = 0;
      bool ok = true;
      for (int id = blockIdx.x; id < total && ok; id += gridDim.x, ++it) {
        const uint32_t acc = (uint32_t)it % a.nacc;
        const uint32_t aph = ((uint32_t)it / a.nacc) & 1u;
        if (!mbar_wait(&c->tempty[acc], aph ^ 1u, a.status, &c->abort, a.wait_limit)) break;
        tc_fence_after();
        const uint32_t dtm = tmem_base + acc * a.acc_cols;
        uint32_t idesc_u = idesc;  // mid: N = this pass's rows rounded up to 16
        if (SWAP && !E4M3 && a.mid) {
          const Work wq = decode_work<SWAP>(a, c, id);
          idesc_u = umma_idesc_bf16(128, (wq.count + 15) & ~15);
        }
        for (int kb = 0; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&c->full[stage], phase, a.status, &c->abort, a.wait_limit)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + (size_t)stage * a.stage_bytes);
          if constexpr (E4M3) {
            // the K block's scales into TMEM; the MMAs below read them after the copies (the
            // tensor core runs this thread's tcgen05 operations in order)
            const uint32_t sf = tmem_base + a.sf_col;
            tmem_cp_32x128b_x4(sf, sdesc_rows16(sb + a.sf_off));
            if (KIND == KIND_G13) tmem_cp_32x128b_x4(sf + 4, sdesc_rows16(sb + a.sf_off + 512));
            tmem_cp_32x128b_x4(sf + 8, sdesc_rows16(sb + a.sf_off + 1024));
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {  // 32 codes along K per MMA, scale byte kk
              const uint32_t kofs = kk * 32;
              const uint32_t accum = (kb | kk) != 0;
              const uint32_t id = umma_idesc_mx_e4m3(128, a.tok_tile, (uint32_t)kk);
              const uint32_t sbyte = (uint32_t)kk << 30;
              const uint64_t bd = umma_desc_k128(sb + a.x_off + kofs);
              umma_mx_e4m3(dtm, umma_desc_k128(sb + kofs), bd, id, sf + sbyte, sf + 8 + sbyte,
                           accum);
              if (KIND == KIND_G13)
                umma_mx_e4m3(dtm + a.tok_tile, umma_desc_k128(sb + TILE_BYTES + kofs), bd, id,
                             sf + 4 + sbyte, sf + 8 + sbyte, accum);
            }
          } else {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk) {
              const uint32_t kofs = kk * 32;  // 16 bf16 along K in the 128-byte row
              const uint32_t accum = (kb | kk) != 0;
              if (!SWAP) {
                umma_bf16(dtm, umma_desc_k128(sb + kofs), umma_desc_k128(sb + TILE_BYTES + kofs),
                          idesc, accum);
              } else {
                const uint64_t bd = umma_desc_k128(sb + a.x_off + kofs);
                umma_bf16(dtm, umma_desc_k128(sb + kofs), bd, idesc_u, accum);
                if (KIND == KIND_G13)
                  umma_bf16(dtm + a.tok_tile, umma_desc_k128(sb + TILE_BYTES + kofs), bd,
                            idesc_u, accum);
              }
            }
          }
          umma_commit(&c->empty[stage]);  // frees the stage once these MMAs have read it
          if (++stage == a.stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit(&c->tfull[acc]);  // accumulator complete
      }
      if (c->abort) {
        umma_commit(&c->mma_done);
        wait_short(&c->mma_done, 0);
      }
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (warps 2..5)
    const int q = warp & 3;  // TMEM lane quarter this warp may access
    const int r = q * 32 + lane;
    int it = 0;
    for (int id = blockIdx.x; id < total; id += gridDim.x, ++it) {
      const Work w = decode_work<SWAP>(a, c, id);
      const uint32_t acc = (uint32_t)it % a.nacc;
      const uint32_t aph = ((uint32_t)it / a.nacc) & 1u;
      const bool ok = mbar_wait(&c->tfull[acc], aph, a.status, &c->abort, a.wait_limit);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + acc * a.acc_cols;
      if (!SWAP && KIND == KIND_G13) {
        __nv_bfloat16* h = static_cast<__nv_bfloat16*>(a.out) + (int64_t)(w.row0 + r) * a.out_ld;
#pragma unroll 1
        for (int cc = 0; cc < 4; ++cc) {
          uint32_t va[32], vb[32];
          tmem_ld32(tb + cc * 32, va);
          tmem_ld32(tb + 128 + cc * 32, vb);
          tmem_ld_wait();
          const int col = w.nt * 128 + cc * 32;
          if (col < a.nw) {
            uint32_t pk[16];
#pragma unroll
            for (int i = 0; i < 16; ++i) {
              const float h0 = silu_epilogue(__uint_as_float(va[2 * i])) * __uint_as_float(vb[2 * i]);
              const float h1 =
                  silu_epilogue(__uint_as_float(va[2 * i + 1])) * __uint_as_float(vb[2 * i + 1]);
              pk[i] = pack_bf16x2(h0, h1);
            }
            uint4* dst = reinterpret_cast<uint4*>(h + col);
#pragma unroll
            for (int i = 0; i < 4; ++i)  // streaming: keep L2 for the weight and X tiles
              __stcs(dst + i, make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]));
          }
        }
      } else if (!SWAP && KIND == KIND_G2) {
        float* y = static_cast<float*>(a.out) + (int64_t)(w.row0 + r) * a.out_ld;
#pragma unroll 1
        for (int cc = 0; cc < 8; ++cc) {
          uint32_t v[32];
          tmem_ld32(tb + cc * 32, v);
          tmem_ld_wait();
          const int col = w.nt * 256 + cc * 32;
          if (col < a.nw) {
            float4* dst = reinterpret_cast<float4*>(y + col);
#pragma unroll
            for (int i = 0; i < 8; ++i)
              __stcs(dst + i, make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                          __uint_as_float(v[4 * i + 2]),
                                          __uint_as_float(v[4 * i + 3])));
          }
        }
      } else {
        // small batch: accumulator row = weight row, column = token of this expert
        float* p = static_cast<float*>(a.out) + (int64_t)w.s * a.split_stride;
        const int f = w.wblk * 128 + r;
        const bool frow = f < a.nw;
        // mid: only the pass's rows; G13 writes h = bf16(silu(a) b) straight away
        const int ncc = a.mid ? (w.count + 15) / 16 : a.tok_tile / 16;
        __nv_bfloat16* hm = static_cast<__nv_bfloat16*>(a.out);
#pragma unroll 1
        for (int cc = 0; cc < ncc; ++cc) {
          uint32_t v1[16], v3[16];
          tmem_ld16(tb + cc * 16, v1);
          if (KIND == KIND_G13) tmem_ld16(tb + a.tok_tile + cc * 16, v3);
          tmem_ld_wait();
#pragma unroll
          for (int jj = 0; jj < 16; ++jj) {
            const int j = cc * 16 + jj;
            if (frow && j < w.count) {
              if (KIND == KIND_G13 && a.mid) {
                hm[(int64_t)(w.row0 + j) * a.out_ld + f] = __float2bfloat16_rn(
                    silu_epilogue(__uint_as_float(v1[jj])) * __uint_as_float(v3[jj]));
              } else {
                float* rowp = p + (int64_t)(w.row0 + j) * a.out_ld;
                rowp[f] = __uint_as_float(v1[jj]);
                if (KIND == KIND_G13) rowp[a.nw + f] = __uint_as_float(v3[jj]);
              }
            }
          }
        }
      }
      tc_fence_before();
      mbar_arrive(&c->tempty[acc]);
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  if (warp == 1) tmem_dealloc(tmem_base, a.tmem_cols);
}

// ---------------------------------------------------------------- CTA-pair prefill tiling
// Tile = 256 permuted rows x two 256-column blocks, computed by a cluster of two CTAs with
// tcgen05.mma.cta_group::2 (M = 256, N = 256 per block).  CTA r holds its 128 rows of A and
// half of each block's N = 256 operand -- G13: W1 rows (r = 0) or the same W3 rows (r = 1),
// so a block is 128 columns of h; G2: W2 rows [128r, 128r + 128) of the block's 256 output
// columns.  Both blocks share the A rows, so a CTA stages 48 KB per 64-wide K block for two
// blocks' MMAs: 48 bytes per MMA cycle, where one block per tile needs 64, which is about what
// an SM can pull from L2.  The even CTA (leader) issues every MMA; both CTAs' TMA loads
// complete on the leader's full barrier; the leader's commits arrive on both CTAs' empty and
// accumulator-full barriers.  The two accumulators fill TMEM (2 x 256 columns), so there is
// no second buffer: the eight epilogue warps drain accumulator 0, release it on the leader's
// barrier, then drain accumulator 1, and the next tile's MMAs start on accumulator 0 in the
// meantime.  A tile whose second block lies past the last column block computes one block.  Expert groups are padded to 256 rows on this path.
constexpr int PAIR_ROWS = 256;
constexpr int PAIR_THREADS = 320;

struct PairCtrl {
  uint64_t full[MAX_STAGES];   // leader: the stage's bytes of both CTAs have landed
  uint64_t empty[MAX_STAGES];  // each CTA: its stage may be refilled
  uint64_t tfull;              // each CTA: both accumulators complete
  uint64_t tempty[2];          // leader: accumulator g drained by both CTAs' epilogues
  uint64_t peer_done;          // each CTA: the peer CTA is finished with TMEM
  uint32_t tmem_slot;
  int abort;
  int off[MAX_EXPERTS + 1];
  int tbase[MAX_EXPERTS + 1];  // row tiles of experts before e
  int cnt[MAX_EXPERTS];        // gather: rows routed to each expert
};

// Tile order: expert, then column-block pair, then row tile (the row tiles of a column-block
// pair run side by side and share its weight tiles through L2).  Tiles go round-robin to the
// pairs; when the last round would keep at most half of the pairs busy, its `split` tiles are
// cut into one-block tiles (ids from wide - split on: two per tile) so that it takes half
// as long.  count = 0 marks the missing second half of a one-block tile.
struct PairSchedule {
  int wide;   // two-block tiles
  int split;  // of which the last `split` are cut in two
};

__device__ __forceinline__ PairSchedule pair_schedule(const TcArgs& a, const PairCtrl* c,
                                                      int npairs) {
  PairSchedule ps;
  ps.wide = c->tbase[a.n] * a.n_tiles;
  const int r = ps.wide % npairs;
  ps.split = a.n_blocks > 1 && r > 0 && 2 * r <= npairs ? r : 0;
  return ps;
}

__device__ __forceinline__ Work decode_pair_work(const TcArgs& a, const PairCtrl* c,
                                                 const PairSchedule& ps, int id) {
  int wid = id, part = -1;
  if (id >= ps.wide - ps.split) {
    const int u = id - (ps.wide - ps.split);
    wid = ps.wide - ps.split + (u >> 1);
    part = u & 1;
  }
  Work w{};
  int e = 0;
  while (e + 1 < a.n && wid >= c->tbase[e + 1] * a.n_tiles) ++e;
  const int mcnt = c->tbase[e + 1] - c->tbase[e];
  const int local = wid - c->tbase[e] * a.n_tiles;
  const int mloc = local % mcnt;
  w.e = e;
  w.nt = local / mcnt;  // column-block pair: blocks 2 nt and 2 nt + 1
  w.row0 = c->off[e] + mloc * PAIR_ROWS;
  w.m = c->off[e + 1] - w.row0 < PAIR_ROWS ? 128 : 256;
  w.count = 2 * w.nt + 1 < a.n_blocks ? 2 : 1;  // blocks in this tile
  w.s = 2 * w.nt;                               // first column block
  if (part >= 0) {
    w.s += part;
    w.count = part < w.count ? 1 : 0;
  }
  return w;
}

template <int KIND>
__global__ void __launch_bounds__(PAIR_THREADS, 1)
    tc_pair_gemm_kernel(const __grid_constant__ CUtensorMap tmX,
                        const __grid_constant__ CUtensorMap tmW0,
                        const __grid_constant__ CUtensorMap tmW1,
                        const __grid_constant__ CUtensorMap tmW0h,
                        const __grid_constant__ CUtensorMap tmW1h, const TcArgs a) {
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  PairCtrl* c = reinterpret_cast<PairCtrl*>(smem + (size_t)a.stages * a.stage_bytes);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int pair = (int)(blockIdx.x >> 1), npairs = (int)(gridDim.x >> 1);

  if (threadIdx.x == 0) {
    for (int s = 0; s < a.stages; ++s) {
      mbar_init(&c->full[s], 1);
      mbar_init(&c->empty[s], 1);
    }
    mbar_init(&c->tfull, 1);
    mbar_init(&c->tempty[0], 512);  // 256 epilogue threads in each of the two CTAs
    mbar_init(&c->tempty[1], 512);
    mbar_init(&c->peer_done, 1);
    c->abort = 0;
    fence_mbar_init();
  }
  if (threadIdx.x == 32) {
    tma_prefetch_desc(&tmX);
    tma_prefetch_desc(&tmW0);
    if (KIND == KIND_G13) {
      tma_prefetch_desc(&tmW1);
      tma_prefetch_desc(&tmW0h);
      tma_prefetch_desc(&tmW1h);
    }
  }
  if (warp == 1) {
    tmem_alloc_pair(&c->tmem_slot, 512);
    tmem_relinquish_pair();
  }
  pdl_wait();  // expert offsets and operands come from the previous kernels
  pdl_trigger();
  if (threadIdx.x <= a.n) c->off[threadIdx.x] = a.offsets[threadIdx.x];
  if (a.counts != nullptr && threadIdx.x < a.n) c->cnt[threadIdx.x] = a.counts[threadIdx.x];
  __syncthreads();
  if (threadIdx.x == 0) {
    c->tbase[0] = 0;
    for (int e = 0; e < a.n; ++e)
      c->tbase[e + 1] = c->tbase[e] + (c->off[e + 1] - c->off[e] + PAIR_ROWS - 1) / PAIR_ROWS;
  }
  tc_fence_before();
  cluster_sync_all();  // barrier initialisation and the TMEM allocation, in both CTAs
  tc_fence_after();
  const uint32_t tmem_base = c->tmem_slot;
  const PairSchedule ps = pair_schedule(a, c, npairs);
  const int total = ps.wide + ps.split;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (both CTAs)
    // Lane 0 waits for free stages and loads the weight halves and the X_perm rows.  When G13
    // reads x directly, the whole warp runs the loop and every lane gathers four of the CTA's
    // 128 A rows per stage (one tile::gather4 of the x rows of their tokens; padding rows read
    // zeros).
    const bool gather = KIND == KIND_G13 && a.row_tok != nullptr;
    const uint64_t pol_w = policy_evict_normal();
    const uint64_t pol_x = policy_evict_last();
    const uint32_t full0 = map_to_rank(&c->full[0], 0);
    int stage = 0;
    uint32_t phase = 0;
    bool ok = true;
    for (int id = pair; id < total && ok && (gather || lane == 0); id += npairs) {
      const Work w = decode_pair_work(a, c, ps, id);
      if (w.count == 0) continue;
      const int rows_cta = w.m >> 1;
      const int row = w.row0 + (int)rank * rows_cta;
      int tok[4] = {0, 0, 0, 0};
      if (gather) {
        const int end = c->off[w.e] + c->cnt[w.e];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = 4 * lane + j;
          tok[j] = i < rows_cta && row + i < end ? a.row_tok[row + i] : a.gather_T;
        }
      }
      for (int kb = 0; kb < a.num_kb; ++kb) {
        if (lane == 0) ok = mbar_wait(&c->empty[stage], phase ^ 1u, a.status, &c->abort);
        if (gather) ok = __shfl_sync(0xffffffffu, ok, 0);
        if (!ok) break;
        uint8_t* st = smem + (size_t)stage * a.stage_bytes;
        const uint32_t fb = full0 + (uint32_t)stage * 8u;
        const int k = kb * 64;
        if (lane == 0) {
          if (leader)
            mbar_arrive_expect_tx(&c->full[stage], 2u * (uint32_t)(1 + w.count) * TILE_BYTES);
          if (!gather) tma_load_2d_pair(st, &tmX, fb, k, row, pol_x);
          for (int j = 0; j < w.count; ++j) {
            const int cb = w.s + j;
            uint8_t* bt = st + (1 + j) * TILE_BYTES;
            if (KIND == KIND_G13 && w.m == 128) {  // 64 W1 rows, then the same 64 W3 rows
              const int wr = w.e * a.nw + cb * 128 + (int)rank * 64;
              tma_load_2d_pair(bt, &tmW0h, fb, k, wr, pol_w);
              tma_load_2d_pair(bt + TILE_BYTES / 2, &tmW1h, fb, k, wr, pol_w);
            } else if (KIND == KIND_G13)
              tma_load_2d_pair(bt, rank == 0 ? &tmW0 : &tmW1, fb, k,
                               w.e * a.nw + cb * 128, pol_w);
            else
              tma_load_2d_pair(bt, &tmW0, fb, k, w.e * a.nw + cb * 256 + (int)rank * 128, pol_w);
          }
        }
        if (gather)
          tma_gather4_pair(st + lane * 512, &tmX, fb, k, tok[0], tok[1], tok[2], tok[3], pol_x);
        if (++stage == a.stages) { stage = 0; phase ^= 1u; }
      }
    }
    // every MMA commit aimed at this CTA's empty barriers has landed before it may exit
    if (lane == 0) {
      for (int s = 0; ok && s < a.stages; ++s) {
        if (!mbar_wait(&c->empty[stage], phase ^ 1u, a.status, &c->abort)) break;
        if (++stage == a.stages) { stage = 0; phase ^= 1u; }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader only)
    // The epilogue drains accumulator 0 before accumulator 1, so a tile starts with the first
    // `lead` K blocks of accumulator 0 (their stages are held) while accumulator 1 is still
    // being drained; accumulator 1 then catches up on the held stages, releasing them.
    if (lane == 0 && leader) {
      const int lead = a.stages < a.num_kb ? a.stages : a.num_kb;
      int stage = 0;
      uint32_t it = 0, phase = 0;
      bool ok = true;
      for (int id = pair; id < total && ok; id += npairs) {
        const Work w = decode_pair_work(a, c, ps, id);
        if (w.count == 0) continue;
        const uint32_t idesc = umma_idesc_bf16(w.m, 256);
        const uint32_t tpar = (it & 1u) ^ 1u;  // tile it - 1 drained
        if (!mbar_wait(&c->tempty[0], tpar, a.status, &c->abort)) { ok = false; break; }
        tc_fence_after();
        const int stage0 = stage;
        const uint32_t phase0 = phase;
        for (int kb = 0; kb < lead; ++kb) {
          if (!mbar_wait(&c->full[stage], phase, a.status, &c->abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + (size_t)stage * a.stage_bytes);
#pragma unroll
          for (int kk = 0; kk < 4; ++kk)
            umma_bf16_pair(tmem_base, umma_desc_k128(sb + kk * 32),
                           umma_desc_k128(sb + TILE_BYTES + kk * 32), idesc, (kb | kk) != 0);
          if (++stage == a.stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        if (w.count == 2) {
          if (!mbar_wait(&c->tempty[1], tpar, a.status, &c->abort)) { ok = false; break; }
          tc_fence_after();
        }
        stage = stage0;
        phase = phase0;
        for (int kb = 0; kb < lead; ++kb) {
          if (w.count == 2) {
            const uint32_t sb = smem_u32(smem + (size_t)stage * a.stage_bytes);
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair(tmem_base + 256u, umma_desc_k128(sb + kk * 32),
                             umma_desc_k128(sb + 2 * TILE_BYTES + kk * 32), idesc,
                             (kb | kk) != 0);
          }
          umma_commit_pair(&c->empty[stage], 0x3);
          if (++stage == a.stages) { stage = 0; phase ^= 1u; }
        }
        for (int kb = lead; kb < a.num_kb; ++kb) {
          if (!mbar_wait(&c->full[stage], phase, a.status, &c->abort)) { ok = false; break; }
          tc_fence_after();
          const uint32_t sb = smem_u32(smem + (size_t)stage * a.stage_bytes);
          for (int j = 0; j < w.count; ++j) {
#pragma unroll
            for (int kk = 0; kk < 4; ++kk)
              umma_bf16_pair(tmem_base + (uint32_t)j * 256u, umma_desc_k128(sb + kk * 32),
                             umma_desc_k128(sb + (uint32_t)(1 + j) * TILE_BYTES + kk * 32),
                             idesc, 1u);
          }
          umma_commit_pair(&c->empty[stage], 0x3);
          if (++stage == a.stages) { stage = 0; phase ^= 1u; }
        }
        if (!ok) break;
        umma_commit_pair(&c->tfull, 0x3);
        ++it;
      }
      // both accumulators released before TMEM is torn down
      if (ok && mbar_wait(&c->tempty[0], (it & 1u) ^ 1u, a.status, &c->abort))
        mbar_wait(&c->tempty[1], (it & 1u) ^ 1u, a.status, &c->abort);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    // Two warps per TMEM lane quarter (warps q + 2 and q + 6, q = warp & 3 being the quarter
    // a warp may access) split the columns; accumulator 0 is drained and released first.
    const int half = (warp - 2) >> 2;
    const int q = warp & 3;
    const int r = q * 32 + lane;
    const uint32_t tempty0 = map_to_rank(&c->tempty[0], 0);
    uint32_t it = 0;
    for (int id = pair; id < total; id += npairs, ++it) {
      const Work w = decode_pair_work(a, c, ps, id);
      if (w.count == 0) { --it; continue; }
      const bool ok = mbar_wait(&c->tfull, it & 1u, a.status, &c->abort);
      if (!__all_sync(0xffffffffu, ok)) break;
      tc_fence_after();
      // M = 256: lane r is row r of this CTA's 128, all 256 columns of the block.
      // M = 128: lane r is row r % 64 of this CTA's 64; lanes >= 64 hold the second half of N.
      const bool full = w.m == 256;
      const int sub = full ? 0 : r >> 6;
      const int64_t row = w.row0 + (full ? (int)rank * 128 + r : (int)rank * 64 + (r & 63));
      for (int g = 0; g < 2; ++g) {
        if (g >= w.count) {
          tc_fence_before();
          mbar_arrive_cluster(tempty0 + (uint32_t)g * 8u);
          continue;
        }
        const int cb = w.s + g;
        const uint32_t tb = tmem_base + ((uint32_t)(q * 32) << 16) + (uint32_t)g * 256u;
        // This warp's share of the accumulator goes to registers first; the accumulator is
        // released to the next tile's MMAs before the SwiGLU and the stores.
        uint32_t v[4][32];
        if (KIND == KIND_G13) {
          if (full) {  // a in columns [0,128), b in [128,256); this warp: 64*half + [0,64)
            const uint32_t c0 = 64u * half;
            tmem_ld32(tb + c0, v[0]);
            tmem_ld32(tb + c0 + 32, v[1]);
            tmem_ld32(tb + 128 + c0, v[2]);
            tmem_ld32(tb + 128 + c0 + 32, v[3]);
          } else {     // a in [0,64), b in [64,128); this warp: 32*half + [0,32)
            const uint32_t c0 = 32u * half;
            tmem_ld32(tb + c0, v[0]);
            tmem_ld32(tb + 64 + c0, v[2]);
          }
        } else {       // this warp: 128*half + [0,128) (full) or 64*half + [0,64) (half)
          const uint32_t c0 = full ? 128u * half : 64u * half;
          tmem_ld32(tb + c0, v[0]);
          tmem_ld32(tb + c0 + 32, v[1]);
          if (full) {
            tmem_ld32(tb + c0 + 64, v[2]);
            tmem_ld32(tb + c0 + 96, v[3]);
          }
        }
        tmem_ld_wait();
        tc_fence_before();
        mbar_arrive_cluster(tempty0 + (uint32_t)g * 8u);
        if (KIND == KIND_G13) {
          __nv_bfloat16* h = static_cast<__nv_bfloat16*>(a.out) + row * a.out_ld;
#pragma unroll
          for (int j = 0; j < 2; ++j) {
            if (j == 1 && !full) break;
            const int col = cb * 128 + sub * 64 + (full ? 64 * half + 32 * j : 32 * half);
            if (col < a.nw) {
              uint32_t pk[16];
#pragma unroll
              for (int i = 0; i < 16; ++i) {
                const float h0 = silu_epilogue(__uint_as_float(v[j][2 * i])) *
                                 __uint_as_float(v[2 + j][2 * i]);
                const float h1 = silu_epilogue(__uint_as_float(v[j][2 * i + 1])) *
                                 __uint_as_float(v[2 + j][2 * i + 1]);
                pk[i] = pack_bf16x2(h0, h1);
              }
              uint4* dst = reinterpret_cast<uint4*>(h + col);
#pragma unroll
              for (int i = 0; i < 4; ++i)  // streaming: keep L2 for the weight and X tiles
                __stcs(dst + i,
                       make_uint4(pk[4 * i], pk[4 * i + 1], pk[4 * i + 2], pk[4 * i + 3]));
            }
          }
        } else {
          float* y = static_cast<float*>(a.out) + row * a.out_ld;
          // the row's gate (the combine then only sums); padding rows are never read
          const float g = a.row_gate != nullptr ? a.row_gate[row] : 1.f;
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            if (j >= 2 && !full) break;
            const int col = cb * 256 + sub * 128 + (full ? 128 * half : 64 * half) + 32 * j;
            if (col < a.nw) {
              float4* dst = reinterpret_cast<float4*>(y + col);
#pragma unroll
              for (int i = 0; i < 8; ++i)
                __stcs(dst + i, make_float4(g * __uint_as_float(v[j][4 * i]),
                                            g * __uint_as_float(v[j][4 * i + 1]),
                                            g * __uint_as_float(v[j][4 * i + 2]),
                                            g * __uint_as_float(v[j][4 * i + 3])));
            }
          }
        }
      }
    }
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if (warp == 1) {  // both CTAs are done with TMEM before the pair deallocates it
    if (lane == 0) {
      mbar_arrive_cluster(map_to_rank(&c->peer_done, rank ^ 1u));
      const long long t0 = clock64();
      while (!mbar_try_wait(&c->peer_done, 0))
        if (clock64() - t0 > WAIT_LIMIT_CYCLES) {
          set_status(a.status, DEV_ERR_TIMEOUT);
          break;
        }
    }
    __syncwarp();
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, 512);
  }
}

// Small batch: h = bf16(silu(sum_s A_s) * sum_s B_s), splits summed in order 0..S-1.  A
// thread's loads go out four splits (eight float4) at a time before their sums: holding all
// eight splits' loads took 102 registers, two CTAs per SM, and a second wave for the last
// CTAs of a decode step's 448.

// The four-wide column slice at p of the split sums of A (p[s * split_stride]) and of B (F
// further on), in split order.
__device__ __forceinline__ void sum_splits(const float* __restrict__ p, int S,
                                           int64_t split_stride, int F, float4* a, float4* b) {
  float4 sa = make_float4(0.f, 0.f, 0.f, 0.f), sb = sa;
  for (int s0 = 0; s0 < S; s0 += 4) {
    float4 ta[4], tb[4];
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (s0 + u < S) {
        ta[u] = __ldg(reinterpret_cast<const float4*>(p + (s0 + u) * split_stride));
        tb[u] = __ldg(reinterpret_cast<const float4*>(p + (s0 + u) * split_stride + F));
      }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (s0 + u < S) {
        sa.x += ta[u].x; sa.y += ta[u].y; sa.z += ta[u].z; sa.w += ta[u].w;
        sb.x += tb[u].x; sb.y += tb[u].y; sb.z += tb[u].z; sb.w += tb[u].w;
      }
  }
  *a = sa;
  *b = sb;
}

__global__ void __launch_bounds__(256)
    swiglu_reduce_kernel(const float* __restrict__ p13, int S, int64_t split_stride,
                         int64_t rows, int F, __nv_bfloat16* __restrict__ h) {
  pdl_wait();
  pdl_trigger();
  const int vpr = F / 4;
  const int64_t total = rows * vpr;
  for (int64_t v = (int64_t)blockIdx.x * blockDim.x + threadIdx.x; v < total;
       v += (int64_t)gridDim.x * blockDim.x) {
    const int64_t r = v / vpr;
    const int c = (int)(v % vpr) * 4;
    float4 sa, sb;
    sum_splits(p13 + r * 2 * F + c, S, split_stride, F, &sa, &sb);
    uint2 o;
    o.x = pack_bf16x2(silu_epilogue(sa.x) * sb.x, silu_epilogue(sa.y) * sb.y);
    o.y = pack_bf16x2(silu_epilogue(sa.z) * sb.z, silu_epilogue(sa.w) * sb.w);
    *reinterpret_cast<uint2*>(h + r * F + c) = o;
  }
}

// ---------------------------------------------------------------- FP8 (MXFP8) weights
// Codes E4M3(v / X) in blocks of 32 consecutive elements of a row sharing the scale X = 2^E
// (mx_scale_code / mx_inv_scale: the smallest E with max |v| <= 448 2^E; v / X is exact).
// One warp per (row, 128 columns): lane c holds columns 4c .. 4c + 3, so a 32-element block is
// 8 lanes and the K block's four scale codes are those of lanes 0, 8, 16 and 24.

// The block scale of this lane's 8-lane group and the K block's scale word (codes of the four
// groups, the lowest columns in the lowest byte; the same value on every lane).
__device__ __forceinline__ uint32_t mx_group_scale(float amax, float* inv, uint32_t* word) {
#pragma unroll
  for (int off = 1; off < 8; off <<= 1) amax = fmaxf(amax, __shfl_xor_sync(0xffffffffu, amax, off));
  const uint32_t code = mx_scale_code(amax);
  *inv = mx_inv_scale(code);
  *word = __shfl_sync(0xffffffffu, code, 0) | (__shfl_sync(0xffffffffu, code, 8) << 8) |
          (__shfl_sync(0xffffffffu, code, 16) << 16) | (__shfl_sync(0xffffffffu, code, 24) << 24);
  return code;
}

// FP8 small batch: permuted row r of expert e (rows grouped by offsets, slot j = r -
// offsets[e]): a = sum_s A_s, b = sum_s B_s (splits in order; the block-scaled MMAs already
// applied every scale), h = silu(a) b in binary32, then block-quantised: codes hq[r][f] and
// the K block's scale word at slot j of the G2 B-operand chunk sfh[e][f / 128].
// four CTAs per SM (at most 64 registers), so that a decode step's 448 CTAs take one wave
__global__ void __launch_bounds__(256, 4)
    swiglu_quantize_mx_kernel(const float* __restrict__ p13, int S, int64_t split_stride,
                              int64_t rows, int F, int n, const int32_t* __restrict__ offsets,
                              uint8_t* __restrict__ hq, uint32_t* __restrict__ sfh) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31;
  const int kbs = F / 128;
  const int64_t gw = (int64_t)blockIdx.x * 8 + (threadIdx.x >> 5);
  if (gw >= rows * kbs) return;  // warp-uniform
  const int64_t r = gw / kbs;
  const int kb = (int)(gw % kbs);
  const int c = kb * 128 + lane * 4;
  float4 sa, sb;
  sum_splits(p13 + r * 2 * F + c, S, split_stride, F, &sa, &sb);
  const float h0 = silu_epilogue(sa.x) * sb.x, h1 = silu_epilogue(sa.y) * sb.y;
  const float h2 = silu_epilogue(sa.z) * sb.z, h3 = silu_epilogue(sa.w) * sb.w;
  float inv;
  uint32_t word;
  mx_group_scale(fmaxf(fmaxf(fabsf(h0), fabsf(h1)), fmaxf(fabsf(h2), fabsf(h3))), &inv, &word);
  *reinterpret_cast<uint32_t*>(hq + r * F + c) = e4m3x4_mul(h0, h1, h2, h3, inv);
  if (lane == 0) {
    int e = 0;
    while (e + 1 < n && r >= offsets[e + 1]) ++e;
    const int j = (int)(r - offsets[e]);  // < 128: an expert gets at most T <= 64 rows
    sfh[((int64_t)e * kbs + kb) * 128 + 4 * (j & 31) + (j >> 5)] = word;
  }
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*,
                                  const cuuint64_t*, const cuuint64_t*, const cuuint32_t*,
                                  const cuuint32_t*, CUtensorMapInterleave, CUtensorMapSwizzle,
                                  CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

static EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static bool tried = false;
  if (!tried) {
    tried = true;
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  }
  return fn;
}

// 2-D bf16 tensor [outer][inner] (row-major), box = box_rows x 64 elements, 128-byte swizzle.
static bool make_map(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                     uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner * 2};
  const cuuint32_t box[2] = {64, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

// 2-D E4M3 tensor [outer][inner] of bytes, box = box_rows x 128 codes, 128-byte swizzle.
static bool make_map_u8(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                        uint32_t box_rows) {
  EncodeTiledFn fn = encode_fn();
  if (!fn) return false;
  const cuuint64_t dims[2] = {inner, outer};
  const cuuint64_t strides[1] = {inner};
  const cuuint32_t box[2] = {128, box_rows};
  const cuuint32_t estr[2] = {1, 1};
  return fn(m, CU_TENSOR_MAP_DATA_TYPE_UINT8, 2, const_cast<void*>(base), dims, strides, box,
            estr, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
            CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
            CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE) == CUDA_SUCCESS;
}

bool make_map_bf16(CUtensorMap* m, const void* base, uint64_t inner, uint64_t outer,
                   uint32_t box_rows) {
  return make_map(m, base, inner, outer, box_rows);
}

constexpr uint32_t SMEM_STAGE_BUDGET = 200 * 1024;
// mid-size tiling: the stages may take all the shared memory a CTA can have (227 KB) beside
// the control block (four 56 KB stages of 192-row passes); the weight tiles in flight set the
// rate at which a CTA streams weights
constexpr uint32_t MID_STAGE_BUDGET = 232448 - (uint32_t)sizeof(Ctrl) - 1024;
static_assert(MID_STAGE_BUDGET >= 4 * (2 * TILE_BYTES + 192 * 128), "four 192-row stages");

template <int KIND, bool SWAP, bool E4M3 = false>
static cudaError_t launch_one(const CUtensorMap& mx, const CUtensorMap& mw0,
                              const CUtensorMap& mw1, TcArgs a, int max_work, cudaStream_t s) {
  const size_t gath = SWAP && KIND == KIND_G13 && a.row_tok ? (size_t)a.gather_rows * 4 : 0;
  const size_t smem = (size_t)a.stages * a.stage_bytes + sizeof(Ctrl) + gath + 1024;
  auto kern = tc_grouped_gemm_kernel<KIND, SWAP, E4M3>;
  static int configured[MAX_DEVICES] = {0};
  const cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
  if (e != cudaSuccess) return e;
  const int grid = max_work < num_sms() ? (max_work > 0 ? max_work : 1) : num_sms();
  pdl(kern, grid, GEMM_THREADS, smem, s)(mx, mw0, mw1, a);
  return cudaGetLastError();
}

template <int KIND>
static cudaError_t launch_pair(const CUtensorMap& mx, const CUtensorMap& mw0,
                               const CUtensorMap& mw1, const CUtensorMap& mw0h,
                               const CUtensorMap& mw1h, TcArgs a, int max_work, cudaStream_t s) {
  const size_t smem = (size_t)a.stages * a.stage_bytes + sizeof(PairCtrl) + 1024;
  auto kern = tc_pair_gemm_kernel<KIND>;
  static int configured[MAX_DEVICES] = {0};
  cudaError_t e = ensure_dynamic_smem(kern, smem, configured);
  if (e != cudaSuccess) return e;
  cudaLaunchConfig_t cfg = {};
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.blockDim = dim3(PAIR_THREADS, 1, 1);
  cfg.dynamicSmemBytes = smem;
  cfg.stream = s;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  static int pairs_fit[64] = {0};  // co-resident clusters per device
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev < 0 || dev >= 64) dev = 0;
  if (!pairs_fit[dev]) {
    int nclusters = 0;
    cfg.gridDim = dim3(2 * (num_sms() / 2), 1, 1);
    if (cudaOccupancyMaxActiveClusters(&nclusters, kern, &cfg) != cudaSuccess || nclusters < 1)
      nclusters = num_sms() / 2;
    pairs_fit[dev] = nclusters;
  }
  int pairs = max_work < pairs_fit[dev] ? max_work : pairs_fit[dev];
  if (pairs < 1) pairs = 1;
  cfg.gridDim = dim3(2 * pairs, 1, 1);
  cfg.numAttrs = 2;
  e = cudaLaunchKernelEx(&cfg, kern, mx, mw0, mw1, mw0h, mw1h, a);
  if (e != cudaSuccess) return e;
  return cudaGetLastError();
}

static int stages_for(uint32_t stage_bytes, uint32_t budget = SMEM_STAGE_BUDGET) {
  int st = (int)(budget / stage_bytes);
  return st > MAX_STAGES ? MAX_STAGES : st;
}

static uint32_t pow2_cols(uint32_t c) {
  uint32_t p = 32;
  while (p < c) p <<= 1;
  return p;
}

static cudaError_t record(cudaEvent_t const* ev, int i, cudaStream_t s) {
  return ev ? cudaEventRecord(ev[i], s) : cudaSuccess;
}

cudaError_t launch_expert_gemms_tc(const Plan& p, const void* x, const void* W1,
                                   const void* W3, const void* W2, const Workspace& w,
                                   cudaStream_t s, cudaEvent_t const* ev) {
  CUtensorMap mX, mW1, mW3, mH, mW2;
  const int d = (int)p.d, F = (int)p.F, n = p.n;
  cudaError_t err;
  if (p.pair) {  // 256-row tiles on CTA pairs
    CUtensorMap mW1h, mW3h;  // 64-row boxes for the M = 128 tiles of G13
    // gather_x: G13's A rows are gathered from x (one-row boxes), else loaded from X_perm
    if (!(p.gather_x ? make_map(&mX, x, d, (uint64_t)p.T, 1)
                     : make_map(&mX, w.xperm, d, p.rows_max, 128)) ||
        !make_map(&mW1, W1, d, (uint64_t)n * F, 128) ||
        !make_map(&mW3, W3, d, (uint64_t)n * F, 128) ||
        !make_map(&mW1h, W1, d, (uint64_t)n * F, 64) ||
        !make_map(&mW3h, W3, d, (uint64_t)n * F, 64) ||
        !make_map(&mH, w.h, F, p.rows_max, 128) ||
        !make_map(&mW2, W2, F, (uint64_t)n * d, 128))
      return cudaErrorInvalidValue;
    const int pair_tiles_max = (int)(p.rows_max / 128);  // bound on row tiles (grid size)
    TcArgs a{};
    a.offsets = w.offsets;
    a.n = n;
    a.stage_bytes = 3 * TILE_BYTES;  // A rows + two column blocks' halves
    a.stages = stages_for(a.stage_bytes);
    a.status = w.status;
    a.num_kb = d / 64;
    a.nw = F;
    a.n_blocks = (F + 127) / 128;
    a.n_tiles = (a.n_blocks + 1) / 2;
    a.out = w.h;
    a.out_ld = F;
    if (p.gather_x) {
      a.row_tok = w.row_tok;
      a.counts = w.counts;
      a.gather_T = (int)p.T;
    }
    if ((err = launch_pair<KIND_G13>(mX, mW1, mW3, mW1h, mW3h, a, pair_tiles_max * a.n_tiles,
                                     s)) !=
        cudaSuccess)
      return err;
    if ((err = record(ev, 0, s)) != cudaSuccess || (err = record(ev, 1, s)) != cudaSuccess)
      return err;
    a.num_kb = F / 64;
    a.nw = d;
    a.n_blocks = (d + 255) / 256;
    a.n_tiles = (a.n_blocks + 1) / 2;
    a.out = w.y;
    a.out_ld = d;
    a.row_tok = nullptr;
    a.counts = nullptr;
    if (p.gather_x) a.row_gate = w.row_gate;
    if ((err = launch_pair<KIND_G2>(mH, mW2, mW2, mW2, mW2, a, pair_tiles_max * a.n_tiles, s)) !=
        cudaSuccess)
      return err;
    return record(ev, 2, s);
  }
  if (p.mid) {  // mid-size groups: weight-stationary tiles, the expert's rows as the MMA's N
    const int tok = p.tok_tile;
    if (!make_map(&mX, w.xperm, d, p.rows_max, MID_BOX) ||
        !make_map(&mW1, W1, d, (uint64_t)n * F, 128) ||
        !make_map(&mW3, W3, d, (uint64_t)n * F, 128) ||
        !make_map(&mH, w.h, F, p.rows_max, MID_BOX) ||
        !make_map(&mW2, W2, F, (uint64_t)n * d, 128))
      return cudaErrorInvalidValue;
    // passes over all experts: one per tok rows, plus at most one partial pass per expert
    const int64_t max_passes = n + (p.T * p.K + tok - 1) / tok;
    TcArgs a{};
    a.offsets = w.offsets;
    a.n = n;
    a.tok_tile = tok;
    a.status = w.status;
    a.mid = 1;
    a.splits = 1;
    // G13 with SwiGLU: h = bf16(silu(x.W1) * (x.W3))
    a.num_kb = d / 64;
    a.nw = F;
    a.wb = (F + 127) / 128;
    a.x_off = 2 * TILE_BYTES;
    a.stage_bytes = 2 * TILE_BYTES + (uint32_t)tok * 128;
    a.tx_bytes = a.stage_bytes;
    a.stages = stages_for(a.stage_bytes, MID_STAGE_BUDGET);
    // W1's and W3's accumulators side by side; two such slots (the epilogue of one pass
    // overlapping the next pass's MMAs) while they fit in TMEM's 512 columns
    a.acc_cols = 2 * tok;
    a.nacc = 2 * a.acc_cols <= 512 ? 2 : 1;
    a.tmem_cols = pow2_cols(a.nacc * a.acc_cols);
    a.out = w.h;
    a.out_ld = F;
    if (p.g13_withhold) {
      a.withhold_loads = 1;
      a.wait_limit = p.g13_wait_limit;
    }
    if ((err = launch_one<KIND_G13, true>(mX, mW1, mW3, a, (int)(max_passes * a.wb), s)) !=
        cudaSuccess)
      return err;
    a.withhold_loads = 0;
    a.wait_limit = WAIT_LIMIT_CYCLES;
    if ((err = record(ev, 0, s)) != cudaSuccess || (err = record(ev, 1, s)) != cudaSuccess)
      return err;
    // G2: Y = h.W2 in fp32
    a.num_kb = F / 64;
    a.nw = d;
    a.wb = (d + 127) / 128;
    a.x_off = TILE_BYTES;
    a.stage_bytes = TILE_BYTES + (uint32_t)tok * 128;
    a.tx_bytes = a.stage_bytes;
    a.stages = stages_for(a.stage_bytes, MID_STAGE_BUDGET);
    a.acc_cols = tok;
    a.nacc = 2;
    a.tmem_cols = pow2_cols(2 * tok);
    a.out = w.y;
    a.out_ld = d;
    a.split_stride = 0;
    if ((err = launch_one<KIND_G2, true>(mH, mW2, mW2, a, (int)(max_passes * a.wb), s)) !=
        cudaSuccess)
      return err;
    return record(ev, 2, s);
  }
  if (!p.swap) {
    if (!make_map(&mX, w.xperm, d, p.rows_max, 128) ||
        !make_map(&mW1, W1, d, (uint64_t)n * F, 128) ||
        !make_map(&mW3, W3, d, (uint64_t)n * F, 128) ||
        !make_map(&mH, w.h, F, p.rows_max, 128) ||
        !make_map(&mW2, W2, F, (uint64_t)n * d, 256))
      return cudaErrorInvalidValue;
    const int m_tiles_max = (int)(p.rows_max / TILE_M);
    TcArgs a{};
    a.offsets = w.offsets;
    a.n = n;
    a.stage_bytes = 3 * TILE_BYTES;
    a.tx_bytes = 3 * TILE_BYTES;
    a.stages = stages_for(a.stage_bytes);
    a.acc_cols = 256;
    a.nacc = 2;
    a.tmem_cols = 512;
    a.status = w.status;
    // G13
    a.num_kb = d / 64;
    a.nw = F;
    a.n_tiles = (F + 127) / 128;
    a.out = w.h;
    a.out_ld = F;
    if (p.g13_withhold) {
      a.withhold_loads = 1;
      a.wait_limit = p.g13_wait_limit;
    }
    if ((err = launch_one<KIND_G13, false>(mX, mW1, mW3, a, m_tiles_max * a.n_tiles, s)) !=
        cudaSuccess)
      return err;
    a.withhold_loads = 0;
    a.wait_limit = WAIT_LIMIT_CYCLES;
    if ((err = record(ev, 0, s)) != cudaSuccess || (err = record(ev, 1, s)) != cudaSuccess)
      return err;
    // G2
    a.num_kb = F / 64;
    a.nw = d;
    a.n_tiles = (d + 255) / 256;
    a.out = w.y;
    a.out_ld = d;
    if ((err = launch_one<KIND_G2, false>(mH, mW2, mW2, a, m_tiles_max * a.n_tiles, s)) !=
        cudaSuccess)
      return err;
    return record(ev, 2, s);
  }
  // small batch
  const int tok = p.tok_tile;
  const uint32_t xbytes = (uint32_t)tok * 128;
  const uint32_t xslot = (xbytes + 1023u) & ~1023u;
  // gather_small: G13's token rows come from x by token (one-row boxes), else from X_perm
  if (!(p.gather_small ? make_map(&mX, x, d, (uint64_t)p.T, 1)
                       : make_map(&mX, w.xperm, d, p.rows_max, tok)) ||
      !make_map(&mW1, W1, d, (uint64_t)n * F, 128) ||
      !make_map(&mW3, W3, d, (uint64_t)n * F, 128) || !make_map(&mH, w.h, F, p.rows_max, tok) ||
      !make_map(&mW2, W2, F, (uint64_t)n * d, 128))
    return cudaErrorInvalidValue;
  TcArgs a{};
  a.offsets = w.offsets;
  a.n = n;
  a.tok_tile = tok;
  a.status = w.status;
  // G13: partial sums of x.W1 and x.W3 per split
  a.splits = p.s13;
  a.num_kb = d / 64 / p.s13;
  a.nw = F;
  a.wb = (F + 127) / 128;
  a.x_off = 2 * TILE_BYTES;
  a.stage_bytes = 2 * TILE_BYTES + xslot;
  a.tx_bytes = 2 * TILE_BYTES + xbytes;
  a.stages = stages_for(a.stage_bytes);
  a.acc_cols = 2 * tok;
  a.nacc = 2 * a.acc_cols <= 512 ? 2 : 1;
  a.tmem_cols = pow2_cols(a.nacc * a.acc_cols);
  a.out = w.p13;
  a.out_ld = 2 * (int64_t)F;
  a.split_stride = p.rows_max * 2 * (int64_t)F;
  if (p.gather_small) {
    a.row_tok = w.row_tok;
    a.gather_T = (int)p.T;
    a.gather_rows = (int)(p.T * p.K);
  }
  if (p.g13_withhold) {
    a.withhold_loads = 1;
    a.wait_limit = p.g13_wait_limit;
  }
  if ((err = launch_one<KIND_G13, true>(mX, mW1, mW3, a, n * a.wb * a.splits, s)) !=
      cudaSuccess)
    return err;
  a.row_tok = nullptr;
  a.withhold_loads = 0;
  a.wait_limit = WAIT_LIMIT_CYCLES;
  if ((err = record(ev, 0, s)) != cudaSuccess) return err;
  const int64_t rows = p.T * p.K;
  const int64_t vec = rows * F / 4;
  const int rgrid = (int)((vec + 255) / 256 < 4 * num_sms() ? (vec + 255) / 256 : 4 * num_sms());
  pdl(swiglu_reduce_kernel, rgrid > 0 ? rgrid : 1, 256, 0, s)(
      w.p13, p.s13, a.split_stride, rows, F, static_cast<__nv_bfloat16*>(w.h));
  if ((err = cudaGetLastError()) != cudaSuccess || (err = record(ev, 1, s)) != cudaSuccess)
    return err;
  // G2: per-split partial sums of h.W2
  a.splits = p.s2;
  a.num_kb = F / 64 / p.s2;
  a.nw = d;
  a.wb = (d + 127) / 128;
  a.x_off = TILE_BYTES;
  a.stage_bytes = TILE_BYTES + xslot;
  a.tx_bytes = TILE_BYTES + xbytes;
  a.stages = stages_for(a.stage_bytes);
  a.acc_cols = tok;
  a.nacc = 2 * a.acc_cols <= 512 ? 2 : 1;
  a.tmem_cols = pow2_cols(a.nacc * a.acc_cols);
  a.out = w.y;
  a.out_ld = d;
  a.split_stride = p.rows_max * (int64_t)d;
  if ((err = launch_one<KIND_G2, true>(mH, mW2, mW2, a, n * a.wb * a.splits, s)) !=
      cudaSuccess)
    return err;
  return record(ev, 2, s);
}

// The small-batch tiling of launch_expert_gemms_tc on MXFP8 codes: G13 partial sums (block
// scales applied by the MMAs), SwiGLU with h block-quantised, G2 partial sums.  The token
// rows' codes are gathered from the per-token rows in w.xperm; the block scales of the B rows
// come from the routing kernel (w.sfx) and from the SwiGLU kernel (w.sfh).
cudaError_t launch_expert_gemms_e4m3(const Plan& p, const uint8_t* W1q, const uint8_t* W3q,
                                     const uint8_t* W2q, const uint8_t* sf1,
                                     const uint8_t* sf3, const uint8_t* sf2, const Workspace& w,
                                     cudaStream_t s, cudaEvent_t const* ev) {
  CUtensorMap mX, mW1, mW3, mH, mW2;
  const int d = (int)p.d, F = (int)p.F, n = p.n;
  const int tok = p.tok_tile;  // a multiple of 32 (the B scales' TMEM layout), <= 64
  const uint32_t xbytes = (uint32_t)tok * 128;
  const uint32_t xslot = (xbytes + 1023u) & ~1023u;
  constexpr uint32_t SF_SLOT = 2048;  // three 512-byte scale chunks, stage size 1024-aligned
  if (!make_map_u8(&mX, w.xperm, d, (uint64_t)p.T, 1) ||
      !make_map_u8(&mW1, W1q, d, (uint64_t)n * F, 128) ||
      !make_map_u8(&mW3, W3q, d, (uint64_t)n * F, 128) ||
      !make_map_u8(&mH, w.h, F, p.rows_max, tok) ||
      !make_map_u8(&mW2, W2q, F, (uint64_t)n * d, 128))
    return cudaErrorInvalidValue;
  cudaError_t err;
  TcArgs a{};
  a.offsets = w.offsets;
  a.n = n;
  a.tok_tile = tok;
  a.status = w.status;
  a.splits = p.s13;
  a.num_kb = d / 128 / p.s13;
  a.nw = F;
  a.wb = (F + 127) / 128;
  a.x_off = 2 * TILE_BYTES;
  a.sf_off = 2 * TILE_BYTES + xslot;
  a.stage_bytes = 2 * TILE_BYTES + xslot + SF_SLOT;
  a.tx_bytes = 2 * TILE_BYTES + xbytes + 3 * 512;
  a.stages = stages_for(a.stage_bytes);
  a.acc_cols = 2 * tok;
  a.nacc = 2 * a.acc_cols + 12 <= 512 ? 2 : 1;
  a.sf_col = a.nacc * a.acc_cols;
  a.tmem_cols = pow2_cols(a.sf_col + 12);
  a.sfa0 = sf1;
  a.sfa1 = sf3;
  a.sfb = reinterpret_cast<const uint8_t*>(w.sfx);
  a.sf_kb = d / 128;
  a.out = w.p13;
  a.out_ld = 2 * (int64_t)F;
  a.split_stride = p.rows_max * 2 * (int64_t)F;
  a.row_tok = w.row_tok;
  a.gather_T = (int)p.T;
  a.gather_rows = (int)(p.T * p.K);
  if ((err = launch_one<KIND_G13, true, true>(mX, mW1, mW3, a, n * a.wb * a.splits, s)) !=
      cudaSuccess)
    return err;
  a.row_tok = nullptr;
  if ((err = record(ev, 0, s)) != cudaSuccess) return err;
  {
    const int64_t rows = p.T * p.K;
    const int64_t warps = rows * (F / 128);
    const unsigned blocks = (unsigned)((warps + 7) / 8 > 0 ? (warps + 7) / 8 : 1);
    pdl(swiglu_quantize_mx_kernel, blocks, 256, 0, s)(
        w.p13, p.s13, a.split_stride, rows, F, n, static_cast<const int32_t*>(w.offsets),
        static_cast<uint8_t*>(w.h), w.sfh);
  }
  if ((err = cudaGetLastError()) != cudaSuccess || (err = record(ev, 1, s)) != cudaSuccess)
    return err;
  a.splits = p.s2;
  a.num_kb = F / 128 / p.s2;
  a.nw = d;
  a.wb = (d + 127) / 128;
  a.x_off = TILE_BYTES;
  a.sf_off = TILE_BYTES + xslot;
  a.stage_bytes = TILE_BYTES + xslot + SF_SLOT;
  a.tx_bytes = TILE_BYTES + xbytes + 2 * 512;
  a.stages = stages_for(a.stage_bytes);
  a.acc_cols = tok;
  a.nacc = 2 * a.acc_cols + 12 <= 512 ? 2 : 1;
  a.sf_col = a.nacc * a.acc_cols;
  a.tmem_cols = pow2_cols(a.sf_col + 12);
  a.sfa0 = sf2;
  a.sfa1 = nullptr;
  a.sfb = reinterpret_cast<const uint8_t*>(w.sfh);
  a.sf_kb = F / 128;
  a.out = w.y;
  a.out_ld = d;
  a.split_stride = p.rows_max * (int64_t)d;
  if ((err = launch_one<KIND_G2, true, true>(mH, mW2, mW2, a, n * a.wb * a.splits, s)) !=
      cudaSuccess)
    return err;
  return record(ev, 2, s);
}

}  // namespace moe
