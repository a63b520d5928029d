// Internal kernel interfaces of the MoE layer library (not part of the C ABI).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "../../include/moe_mxfp4.h"

namespace moe {

// --- grouped MXFP4 GEMV (decode) -------------------------------------------
struct GateUpArgs {
  const __half* x16;         // [T, W] f16 activation rows (one per token)
  const float* xscale;       // [T] power-of-two row scales
  const int32_t* offsets;    // [E+1]
  const int32_t* expert_list;  // [E+1]: count, then active experts
  const int32_t* row_token;  // [R]
  const uint8_t *wg_q, *wg_s, *wu_q, *wu_s;
  __half* h16;               // [R, I]
  float* hscale;             // [R, I/16]
  int W, I, E, R;
  int min_tokens;            // experts with fewer tokens are left to the CUDA-core path
};

// Gate/up of the experts with 2+ tokens through a CTA-wide TMA ring (W and I
// multiples of 512, gemv_mma.cu): codes by 2-D tensor maps over [E*I, W/2]
// bytes (boxes of 128 bytes x 64 rows, 128-byte swizzle), scales over
// [E*I, W/32] bytes (boxes of 16 bytes x 64 rows), token rows by bulk copies;
// h written as fp32 rows (g.h16 / g.hscale unused).
constexpr int kMmaConsumers = 16;    // consumer warps plus one producer warp
constexpr int kMmaStages = 3;
struct MmaGateUpArgs {
  CUtensorMap map_gq, map_uq, map_gs, map_us;
  GateUpArgs g;
  float* h32;                // [R, I]
  int32_t* status;
};
__global__ void k_mma_gateup(const __grid_constant__ MmaGateUpArgs a);
size_t mma_gateup_smem_bytes();
// h rows of the experts with >= min_tokens tokens: fp32 [R, I] -> f16 [R, I]
// with one power-of-two scale per row (hrs [R])
__global__ void k_h_rowscale(const float* h32, const int32_t* offsets, int E, int R, int I,
                             int min_tokens, __half* h16, float* hrs);
// Down projection of the experts with 2+ tokens, the same ring: down codes
// [E*W, I/2] (boxes of 128 bytes x 128 rows) and scales [E*W, I/32] (16 bytes
// x 128 rows) by tensor maps, the tokens' f16 h rows by bulk copies.
struct MmaDownArgs {
  CUtensorMap map_dq, map_ds;
  const __half* h16;         // [R, I]
  const float* hrs;          // [R] h row scales
  const int32_t* offsets;
  const int32_t* expert_list;
  float* y_perm;             // [R, W]
  int32_t* status;
  int W, I, E, R;
  int min_tokens;
};
__global__ void k_mma_down(const __grid_constant__ MmaDownArgs a);
size_t mma_down_smem_bytes();

struct DownArgs {
  const __half* h16;
  const float* hscale;
  const int32_t* offsets;
  const int32_t* expert_list;
  const uint8_t *wd_q, *wd_s;
  float* y_perm;             // [R, W]
  int W, I, E, R;
  int min_tokens;
};

// tensor-core path: experts with >= 2 tokens
__global__ void k_gateup_mxfp4(GateUpArgs a);
__global__ void k_down_mxfp4(DownArgs a);
size_t gemv_mxfp4_smem_bytes();
// CUDA-core path: experts with exactly 1 token (gemv_fma.cu)
constexpr int kFmaConsumers = 16;  // consumer warps per CTA (plus one producer warp)
constexpr int kFmaMaxStages = 8;
struct FmaArgs {
  const __half* x16;         // gate/up: [T, W] f16 rows, xscale [T]
  const float* xscale;
  float* h32;                // gate/up writes, down reads: [R, I] fp32
  const int32_t* offsets;
  const int32_t* expert_list;
  const int32_t* row_token;
  const uint8_t *wg_q, *wg_s, *wu_q, *wu_s, *wd_q, *wd_s;
  float* y_perm;             // down: [R, W]
  int32_t* status;           // device status word
  int32_t* sync;             // one-token launch: [0] finished CTAs, [1 + s] h row pairs of expert slot s
  // one-token launch: bytes the next kernel of the stream reads (16-byte
  // aligned, a multiple of 16), prefetched into L2 by each CTA as the chunks
  // run out (its 1/gridDim share); NULL: none
  const void* l2_next;
  uint64_t l2_next_bytes;
  int W, I, E, R;
};
// Launch geometry: rps rows per consumer warp of a down stage, units per stage
// (gate/up: row pairs; down: rows), code_bytes = one matrix's codes of a
// stage, sbuf_off / sbuf2_off = offsets of the E8M0 spans (the second:
// gate/up only), nst ring stages, act_off = the activation row buffer.
// act_stride: the one-token launch's down role keeps two f16 h buffers
// (f16 row, then K/32 fp32 block scales) act_stride bytes apart.
struct FmaGeometry {
  int ok, rps, nst, units;
  uint32_t code_bytes, sbuf_off, sbuf2_off, stage_bytes, act_off, smem_bytes, act_stride;
};
FmaGeometry fma_geometry(int K, bool gate_up, size_t smem_budget, bool routed1 = false);
template <int BPL, bool kGateUp, int RPS> __global__ void k_fma_gemv(FmaArgs a, FmaGeometry g);
// One token: gate/up and down of all its experts in one launch, chunks taken
// from device counters (gate/up first); gg / gd share the ring (stage_bytes,
// nst) and the activation region (act_off). sync holds 3 + kRouted1MaxK words.
constexpr int kRouted1MaxK = 32;     // experts of the token (k <= 32)
constexpr int kRouted1SyncWords = 3 + kRouted1MaxK;
constexpr int kRouted1Warps = kFmaConsumers + 2;   // producer, consumers, signal warp
template <int BG, int BD, int RPSD>
__global__ void k_fma_routed1(FmaArgs a, FmaGeometry gg, FmaGeometry gd);
// the common geometry of k_fma_routed1 (ok = 0 when it does not fit)
void routed1_geometry(int W, int I, size_t smem_budget, FmaGeometry& gg, FmaGeometry& gd);

// --- grouped MXFP4 GEMM on tcgen05 (many tokens per expert) ----------------
// Token rows are grouped in tiles of at most kTileRows consecutive permuted
// rows of one expert (the MMA's N side). Weight codes are read through 2-D
// tensor maps over [E*M, K/2] bytes (boxes of 128 rows x 128 bytes, 128-byte
// swizzle), token codes through a map over [R, K/2] (boxes of kTileRows rows);
// all scales are in the tiled layout of sf_tiled_offset (weights: 128-row
// tiles; tokens: the tiles of the tile list).
constexpr int kTileRows = 112;
struct Mxf4GemmArgs {
  CUtensorMap map_a0;        // gate/up: gate weights; down: down weights
  CUtensorMap map_a1;        // gate/up: up weights
  CUtensorMap map_b;         // token codes: x rows (gate/up) or h rows (down), [R, K/2]
  const uint8_t* sa0;        // tiled weight scales
  const uint8_t* sa1;
  const uint8_t* bs;         // tiled token scales
  const int4* tiles;         // k_tile_list output
  const int32_t* n_tiles;
  uint8_t* hq;               // gate/up out: h codes [R, M/2]
  uint8_t* hs;               // gate/up out: h scales, tiled (K = M)
  float* y;                  // down out: y_perm [R, M]
  int32_t* status;           // device status word
  int K, M;                  // reduction length; weight rows per expert (a multiple of 128)
};
__global__ void k_tile_list(const int32_t* offsets, const int32_t* expert_list, int4* tiles,
                            int32_t* tile_base, int32_t* n_tiles);
__global__ void k_tile_scales(const uint8_t* src, long rows, int K, uint8_t* dst);
template <bool kGateUp> __global__ void k_mxf4_gemm(const __grid_constant__ Mxf4GemmArgs a);
size_t mxf4_gemm_smem_bytes(bool gate_up);
int mxf4_gemm_threads();

// --- single-token bf16 GEMV (contiguous row ranges per CTA, mma.sync) ------
constexpr int kRowsConsumers = 16;   // consumer warps (plus one producer warp)
constexpr int kRowsMaxStages = 8;
struct RowsArgs {
  const uint16_t* w[3];      // bf16 [rows[i], K]; SwiGLU: w[0] gate, w[1] up
  int rows[3];               // plain: segment rows (0: unused); SwiGLU: rows[0] = row pairs
  float* out[3];             // plain: out[i][row] per segment; SwiGLU: out[0][i] = h_i
  const void* x;             // [K] bf16, or fp32 (k_rows_bf16<*, true>)
  int32_t* status;
  int K, nst;
  int slots;                 // row slots of a stage: 1..16 (plain), 2..16 (SwiGLU), a power of two
  // optional combine of one token (plain mode): instead of
  // out[0][row], y[row] = sum_j topk_w[j] * y_perm[slot_row[j], row]
  //                      + sigmoid(gate_logit[0]) * (Wx)[row]
  float* y;                  // [rows[0]] or NULL
  const float* y_perm;       // [R, rows[0]]
  const int32_t* slot_row;   // [k]
  const float* topk_w;       // [k]
  const float* gate_logit;   // [1]
  int k;
  // optional, plain mode with bf16 x: CTA 0 also writes x as the f16
  // activation operand of the single-token expert GEMVs (the row's largest
  // |x| mapped into [2^14, 2^15) by a power-of-two scale, written to xscale)
  __half* x16;               // [K] or NULL
  float* xscale;             // [1]
};
template <bool kSwiGLU, bool kXF32> __global__ void k_rows_bf16(RowsArgs a);
// K a power of two in 1024..8192: a stage holds `slots` row slots (plain:
// rows; SwiGLU: half gate, half up rows) of a K chunk of about 64 KB over the
// slots, each slot 16 bytes longer than the chunk (conflict-free ldmatrix);
// after the ring the activation (bf16 x [K], or the bf16 hi/lo pair [2][K]
// of fp32 x)
__host__ __device__ constexpr int rows_chunk(int K, int slots) { return K < 32768 / slots ? K : 32768 / slots; }
__host__ __device__ constexpr size_t rows_stage_bytes(int K, int slots) {
  return (size_t)slots * ((size_t)rows_chunk(K, slots) * 2 + 16);
}
__host__ __device__ constexpr size_t rows_act_bytes(int K, bool x_f32) { return (size_t)K * (x_f32 ? 4 : 2); }
int rows_stages(int K, int slots, bool x_f32, size_t smem_budget);

// --- dense bf16 GEMM on tcgen05 -----------------------------------------------
// Weights [rows, K] and tokens [T, K] bf16 through 2-D tensor maps (weights:
// boxes of 128 rows x 64 elements; tokens: N rows x 64 elements; 128-byte
// swizzle). K / S a multiple of 64; N (tokens per tile, the MMA's N) a
// multiple of 16 in 16..128.
constexpr int kBf16Plain = 0;     // out[(s*T + t)*ld + col] fp32 partial sums over K split s
constexpr int kBf16SwiGLU = 1;    // h = silu(Wg x) * (Wu x) as a bf16 hi/lo pair [T, M]
struct Bf16GemmArgs {
  CUtensorMap map_a[3];      // plain: up to three row segments of W; SwiGLU: [0] Wg, [1] Wu
  CUtensorMap map_b0;        // tokens (pass 0)
  CUtensorMap map_b1;        // tokens of pass 1 (plain, passes == 2: the lo half)
  float* out;                // plain
  uint16_t* h_hi;            // SwiGLU: [T, M]
  uint16_t* h_lo;
  int32_t* status;
  int mode, K, T, S, passes, N;
  int seg_rows[3];           // plain: rows of each segment (0: unused); SwiGLU: seg_rows[0] = M
  int ld;                    // plain: row stride of out; segment i starts at column rows(0..i-1)
};
__global__ void k_bf16_gemm(const __grid_constant__ Bf16GemmArgs a);
// Stage = two 128-row weight tiles + one N-row token tile per pass; as many
// stages (at most 8) as fit in the budget: all of a CTA's shared memory for
// large token tiles, 144 KB for N <= 64 so that the small kernels of the
// routing chain still fit on an SM beside a CTA of a weight-streaming GEMM.
constexpr int kBf16SmemBudget = 232448 - 1024 - 256;
constexpr int kBf16SmallBudget = 144 * 1024;
__host__ __device__ constexpr int bf16_stage_bytes(int N, int passes) { return 32768 + passes * N * 128; }
__host__ __device__ constexpr int bf16_stages(int N, int passes) {
  return ((N <= 64 ? kBf16SmallBudget : kBf16SmemBudget) / bf16_stage_bytes(N, passes)) < 8
             ? (N <= 64 ? kBf16SmallBudget : kBf16SmemBudget) / bf16_stage_bytes(N, passes)
             : 8;
}
size_t bf16_gemm_smem_bytes(int N, int passes);
int bf16_gemm_threads();

// --- dense bf16 GEMV with split-K partial sums (moe_route_noalloc's router) -
struct DenseArgs {
  const uint16_t* w[3];      // row segments of the weight matrix, each [rows, K]
  int rows[3];
  int N;                     // rows[0] + rows[1] + rows[2]
  const void* x;             // [T, K] bf16 bits, or fp32 when x_f32
  int x_f32;
  float* part;               // [S, T, N] partial sums
  int T, K, S, kper;         // kper = K / S, a multiple of 32
};
__global__ void k_dense_gemv(DenseArgs a);
constexpr int kDenseWarps = 4;   // warps (16-row tiles) per CTA

// --- router tail ------------------------------------------------------------
constexpr int kTopkThreads = 1024;
// One token with bf16 activations: k_topk can also write what k_permute and
// k_act_to_f16 write for it (the dispatch of its k experts and the f16 row
// with its power-of-two scale); x == NULL: top-k only.
struct TopkFuse {
  int32_t *counts, *offsets, *expert_list, *row_token, *row_slot, *slot_row;
  const uint16_t* x;         // [W] bf16
  int W;                     // a multiple of 8
  __half* x16;               // [W], or NULL when the router launch writes the operand
  float* xscale;             // [1]
};
// How k_topk scores and selects (the default is the softmax router):
// score_fn 0: softmax (selection by logit, weights the softmax renormalised
//   over the selected experts);
// score_fn 1: sigmoid (s = sigmoid(logit); selection by s + bias[e] with
//   bias nullable; weights s / sum of the selected s);
// n_group > 1: group-limited selection (E / n_group consecutive experts per
//   group, a group scored by the sum of its two largest expert scores, the
//   softmax probability or the biased sigmoid score; the topk_group best
//   groups kept, ties to the lower group; top-k among their experts);
// the weights are multiplied by scale.
struct RouteCfg {
  const float* bias;         // [E] or nullptr
  float scale;
  int score_fn, n_group, topk_group;
};
constexpr int kMaxGroups = 64;
// part [S, T, ld] router partial sums (ld >= E); with gate_logit set, column E
// holds the sigmoid-gate row's partials and gate_logit[t] gets their sum;
// f.x set: T == 1 and the fused dispatch above
__global__ void k_topk(const float* part, int S, int T, int E, int ld, int k, int32_t* idx, float* w,
                       float* logits, float* gate_logit, TopkFuse f, RouteCfg rc);

// --- permutation and activation operands ------------------------------------
__global__ void k_permute(const int32_t* idx, int T, int k, int E, int32_t* counts,
                          int32_t* offsets, int32_t* expert_list, int32_t* row_token,
                          int32_t* row_slot, int32_t* slot_row, int32_t* status);
size_t permute_smem_bytes(int E, int R);
__global__ void k_act_to_f16(const uint16_t* x, int W, __half* x16, float* xscale);
__global__ void k_act_to_mxfp4_perm(const uint16_t* x, int W, int k, const int32_t* idx,
                                    const int32_t* slot_row, const int32_t* offsets,
                                    const int32_t* expert_list, const int32_t* tile_base,
                                    uint8_t* q, uint8_t* sf);

// --- finalisers of split-K partials ----------------------------------------
constexpr int kFinThreads = 64;
__global__ void k_shared_swiglu(const float* part, int S, int T, int Is, uint16_t* h_hi,
                                uint16_t* h_lo, float* gate_logit);
// out[t, n] = bf16(sum_s part[(s * T + t) * ld + n]), n < N
__global__ void k_round_bf16(const float* part, int S, int T, int N, int ld, uint16_t* out);
__global__ void k_sum_column(const float* part, int S, int T, int ld, int col, float* out);

struct CombineArgs {
  const float* y_perm;       // [R, width] or NULL
  const int32_t* slot_row;   // [T, k]
  const float* topk_w;       // [T, k]
  int k;
  const float* add1;         // [S1, T, width] partials added as is, or NULL
  int S1;
  const float* add2;         // [S2, T, width] partials scaled by sigmoid(gate_logit[t]), or NULL
  int S2;
  const float* gate_logit;   // [T]
  float* out;                // [T, width] fp32, or NULL when out_hi is set
  uint16_t* out_hi;          // [T, width] bf16 pair hi = bf16(y), lo = bf16(y - hi), or NULL
  uint16_t* out_lo;
  int T, width;
};
constexpr int kCombineThreads = 64;
__global__ void k_combine(CombineArgs a);

// one-line reason for moe_last_error() (defined with the C ABI in api.cu)
moe_status record_error(moe_status s, const char* msg);

}  // namespace moe
