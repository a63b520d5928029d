// Grouped MXFP4 GEMV for the routed experts that received 2 or more tokens
// (decode batches); single-token experts take the CUDA-core path (gemv_fma.cu).
//
// The "expert matmul" of the rabbit README phase breakdown: for every active
// expert e and its n_e tokens, gate/up projections with a fused SwiGLU
// epilogue, then the down projection. Weights are OCP MXFP4 (E2M1 nibbles,
// one E8M0 scale per 32 elements of a row), read once from HBM.
//
// Design (B200, memory-bound):
// * one warp per CTA; persistent CTAs walk the work items (active expert from
//   the permutation's expert list, 16-row tile of its matrices, full K), so a
//   1-token decode step spreads 1280 gate/up items over the 148 SMs;
// * each warp streams its rows through a private 4-stage cp.async ring in
//   shared memory (128 B of every row per stage = 8 scale blocks, stored with
//   the 128-byte XOR swizzle so ldmatrix is conflict-free);
// * ldmatrix.x4 hands every lane 4 bytes (8 E2M1 codes) of one 32-element
//   block for rows g and g+8 of the tile, exactly the A-fragment shape of
//   mma.m16n8k16 with K permuted inside the block: one MMA pair never mixes
//   two scale blocks, so the E8M0 scale is applied once per block to the
//   fp32 MMA result;
// * E2M1 pairs become f16x2 with one cvt.rn.f16x2.e2m1x2 each (exact);
// * activations enter as f16: x with one power-of-two scale per token row
//   (exact for bf16 x), h with one power-of-two scale per group of 16
//   elements that one MMA of the down projection consumes.
#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

constexpr int kStages = 4;
constexpr int kRowsPerStage = 32;                  // 2 m16 tiles
constexpr int kRowBytes = 128;                     // 256 K elements
constexpr int kStageWBytes = kRowsPerStage * kRowBytes;
constexpr int kStageSBytes = kRowsPerStage * 8;    // 8 E8M0 codes per row
constexpr int kStageBytes = kStageWBytes + kStageSBytes;

// Global row (relative to the tile base) of tile-local row r (0..15). A gate/up
// tile takes the interleaved set {8a + j : a = 0..3, j = 0..3} of its 32-row
// block (its partner tile, based 4 rows further, takes j = 4..7): exactly the
// K elements one mma.m16n8k16 of the down projection covers in a 32-element
// block, so the power-of-two scale of each 16-element h group is per MMA.
MOE_DEV int tile_row(int r, bool interleaved) { return interleaved ? 8 * (r >> 2) + (r & 3) : r; }

// Issue the cp.async copies of one stage: tile rows 0..15 from (q0, s0), rows
// 16..31 from (q1, s1); `kb` = first K element of the slab, `nblk` = 4 or 8 blocks.
MOE_DEV void issue_stage(uint8_t* st, const uint8_t* __restrict__ q0, const uint8_t* __restrict__ s0,
                         const uint8_t* __restrict__ q1, const uint8_t* __restrict__ s1,
                         size_t qrow, size_t srow, int kb, int nblk, bool interleaved, int lane) {
#pragma unroll
  for (int m = 0; m < 8; ++m) {
    const int idx = lane + 32 * m;
    const int row = idx >> 3, c = idx & 7;
    if (c < nblk) {
      const int gr = tile_row(row & 15, interleaved);
      const uint8_t* src = (row < 16 ? q0 : q1) + gr * qrow + (kb >> 1) + c * 16;
      cp_async_16(smem_u32(st + row * kRowBytes + ((c ^ (row & 7)) << 4)), src);
    }
  }
#pragma unroll
  for (int m = 0; m < 2; ++m) {
    const int idx = lane + 32 * m;
    const int row = idx >> 1, wd = idx & 1;
    if (wd * 4 < nblk) {
      const int gr = tile_row(row & 15, interleaved);
      const uint8_t* src = (row < 16 ? s0 : s1) + gr * srow + (kb >> 5) + wd * 4;
      cp_async_4(smem_u32(st + kStageWBytes + row * 8 + wd * 4), src);
    }
  }
}

// ldmatrix.x4 of block pair (2*bp, 2*bp+1) for the m16 tile starting at smem row r16.
MOE_DEV void load_tile_pair(uint32_t (&r)[4], const uint8_t* st, int r16, int bp, int lane) {
  const int q = lane >> 3, rr = lane & 7;
  const int row = r16 + (q & 1) * 8 + rr;
  const int chunk = 2 * bp + (q >> 1);
  ldmatrix_x4(r, smem_u32(st + row * kRowBytes + ((chunk ^ (row & 7)) << 4)));
}

// A fragments of the two k16 halves of one block from the row-g / row-g+8 words.
MOE_DEV void decode_block(uint32_t wg, uint32_t wg8, uint32_t (&a0)[4], uint32_t (&a1)[4]) {
  uint32_t lo[4], hi[4];
  e2m1x8_to_f16x8(wg, lo);
  e2m1x8_to_f16x8(wg8, hi);
  a0[0] = lo[0]; a0[1] = hi[0]; a0[2] = lo[1]; a0[3] = hi[1];
  a1[0] = lo[2]; a1[1] = hi[2]; a1[2] = lo[3]; a1[3] = hi[3];
}

// power-of-two scale mapping a block maximum m into [2^14, 2^15) as f16
MOE_DEV void f16_block_scale(float m, float& scale, float& inv) {
  if (!(m > 0.0f) || !isfinite(m)) { scale = 1.0f; inv = 1.0f; return; }
  const int ex = max(-100, min(127, frexp_exponent(m)));   // m = f * 2^ex, f in [0.5, 1)
  scale = pow2_f32(ex - 15);
  inv = pow2_f32(15 - ex);
}

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU
// persistent grid, block 32, dynamic smem kStages*kStageBytes; work item =
// (active expert, 16-row tile), item = ai * (I/16) + tile
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) k_gateup_mxfp4(GateUpArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;
  const int tiles = a.I >> 4;
  const int items = __ldg(a.expert_list) * tiles;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
  const int ai = item / tiles, tile = item - ai * tiles;
  const int e = __ldg(a.expert_list + 1 + ai);
  const int r0 = __ldg(a.offsets + e);
  const int n_all = __ldg(a.offsets + e + 1) - r0;
  if (n_all < a.min_tokens) continue;          // single-token experts: CUDA-core path
  // tile q covers rows {32*(q/2) + 4*(q%2) + 8a + j : a, j = 0..3}; its h group is q
  const int i0 = 32 * (tile >> 1) + 4 * (tile & 1);
  const size_t qrow = (size_t)a.W / 2, srow = (size_t)a.W / 32;
  const uint8_t* gq = a.wg_q + ((size_t)e * a.I + i0) * qrow;
  const uint8_t* gs = a.wg_s + ((size_t)e * a.I + i0) * srow;
  const uint8_t* uq = a.wu_q + ((size_t)e * a.I + i0) * qrow;
  const uint8_t* us = a.wu_s + ((size_t)e * a.I + i0) * srow;
  const int nslab = (a.W + 255) / 256;

  for (int c0 = 0; c0 < n_all; c0 += 32) {
    const int n = min(32, n_all - c0);
    const int ng = (n + 7) >> 3;
    const __half* xrow[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const int slot = min(gi * 8 + g, n - 1);
      xrow[gi] = a.x16 + (size_t)__ldg(a.row_token + r0 + c0 + slot) * a.W + 8 * t;
    }
    float accG[4][4], accU[4][4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi)
#pragma unroll
      for (int j = 0; j < 4; ++j) accG[gi][j] = accU[gi][j] = 0.0f;

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
      if (s < nslab)
        issue_stage(smem + s * kStageBytes, gq, gs, uq, us, qrow, srow, s * 256,
                    min(8, (a.W - s * 256) >> 5), true, lane);
      cp_async_commit();
    }
    for (int slab = 0; slab < nslab; ++slab) {
      cp_async_wait<kStages - 2>();
      __syncwarp();
      {
        const int nx = slab + kStages - 1;
        if (nx < nslab)
          issue_stage(smem + (nx % kStages) * kStageBytes, gq, gs, uq, us, qrow, srow, nx * 256,
                      min(8, (a.W - nx * 256) >> 5), true, lane);
        cp_async_commit();
      }
      const uint8_t* st = smem + (slab % kStages) * kStageBytes;
      const uint8_t* ss = st + kStageWBytes;
      const int kb = slab * 256;
      const int nbp = min(8, (a.W - kb) >> 5) >> 1;
      // the slab's activations of token group 0, all loads in flight at once
      uint4 xpre[8];
#pragma unroll
      for (int b = 0; b < 8; ++b)
        xpre[b] = (b < 2 * nbp) ? ldg16(xrow[0] + kb + 32 * b) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
      for (int bp = 0; bp < 4; ++bp) {
        if (bp < nbp) {
          uint32_t Rg[4], Ru[4];
          load_tile_pair(Rg, st, 0, bp, lane);
          load_tile_pair(Ru, st, 16, bp, lane);
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const int b = 2 * bp + hb;
            uint32_t ag0[4], ag1[4], au0[4], au1[4];
            decode_block(Rg[2 * hb], Rg[2 * hb + 1], ag0, ag1);
            decode_block(Ru[2 * hb], Ru[2 * hb + 1], au0, au1);
            const float sg0 = e8m0_to_f32(ss[g * 8 + b]);
            const float sg8 = e8m0_to_f32(ss[(g + 8) * 8 + b]);
            const float su0 = e8m0_to_f32(ss[(g + 16) * 8 + b]);
            const float su8 = e8m0_to_f32(ss[(g + 24) * 8 + b]);
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              if (gi < ng) {
                const uint4 xv = gi == 0 ? xpre[b] : ldg16(xrow[gi] + kb + 32 * b);
                float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16(cg, ag0, xv.x, xv.y);
                mma_f16(cg, ag1, xv.z, xv.w);
                mma_f16(cu, au0, xv.x, xv.y);
                mma_f16(cu, au1, xv.z, xv.w);
                accG[gi][0] = fmaf(cg[0], sg0, accG[gi][0]);
                accG[gi][1] = fmaf(cg[1], sg0, accG[gi][1]);
                accG[gi][2] = fmaf(cg[2], sg8, accG[gi][2]);
                accG[gi][3] = fmaf(cg[3], sg8, accG[gi][3]);
                accU[gi][0] = fmaf(cu[0], su0, accU[gi][0]);
                accU[gi][1] = fmaf(cu[1], su0, accU[gi][1]);
                accU[gi][2] = fmaf(cu[2], su8, accU[gi][2]);
                accU[gi][3] = fmaf(cu[3], su8, accU[gi][3]);
              }
            }
          }
        }
      }
    }
    cp_async_wait<0>();
    __syncwarp();

    // epilogue: h = silu(G) * U, one power-of-two scale per (token, 16 rows)
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      if (gi < ng) {
        float h[4];
        float xs[2];
#pragma unroll
        for (int c = 0; c < 2; ++c) {
          const int col = gi * 8 + 2 * t + c;
          xs[c] = (col < n) ? __ldg(a.xscale + __ldg(a.row_token + r0 + c0 + col)) : 0.0f;
        }
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const float G = accG[gi][j] * xs[j & 1];
          const float U = accU[gi][j] * xs[j & 1];
          h[j] = silu_f32(G) * U;
        }
        float m0 = fmaxf(fabsf(h[0]), fabsf(h[2]));
        float m1 = fmaxf(fabsf(h[1]), fabsf(h[3]));
#pragma unroll
        for (int off = 4; off < 32; off <<= 1) {
          m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, off));
          m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, off));
        }
        float sc[2], inv[2];
        f16_block_scale(m0, sc[0], inv[0]);
        f16_block_scale(m1, sc[1], inv[1]);
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int col = gi * 8 + 2 * t + (j & 1);
          if (col < n) {
            const int row = tile_row(g + 8 * (j >> 1), true);
            a.h16[(size_t)(r0 + c0 + col) * a.I + i0 + row] = __float2half_rn(h[j] * inv[j & 1]);
          }
        }
        if (g == 0) {
#pragma unroll
          for (int c = 0; c < 2; ++c) {
            const int col = gi * 8 + 2 * t + c;
            if (col < n) a.hscale[(size_t)(r0 + c0 + col) * (a.I >> 4) + tile] = sc[c];
          }
        }
      }
    }
  }
  }  // items
}

// ---------------------------------------------------------------------------
// down projection
// persistent grid, block 32, dynamic smem kStages*kStageBytes; work item =
// (active expert, 32-row tile of W), item = ai * (W/32) + tile
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32) k_down_mxfp4(DownArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x;
  const int g = lane >> 2, t = lane & 3;
  const int tiles = a.W >> 5;
  const int items = __ldg(a.expert_list) * tiles;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
  const int ai = item / tiles, tile = item - ai * tiles;
  const int e = __ldg(a.expert_list + 1 + ai);
  const int r0 = __ldg(a.offsets + e);
  const int n_all = __ldg(a.offsets + e + 1) - r0;
  if (n_all < a.min_tokens) continue;          // single-token experts: CUDA-core path
  const int n0 = tile * 32;
  const size_t qrow = (size_t)a.I / 2, srow = (size_t)a.I / 32;
  const uint8_t* dq = a.wd_q + ((size_t)e * a.W + n0) * qrow;
  const uint8_t* ds = a.wd_s + ((size_t)e * a.W + n0) * srow;
  const int nslab = (a.I + 255) / 256;

  for (int c0 = 0; c0 < n_all; c0 += 32) {
    const int n = min(32, n_all - c0);
    const int ng = (n + 7) >> 3;
    const __half* hrow[4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      const int slot = min(gi * 8 + g, n - 1);
      hrow[gi] = a.h16 + (size_t)(r0 + c0 + slot) * a.I + 8 * t;
    }
    float acc[4][2][4];
#pragma unroll
    for (int gi = 0; gi < 4; ++gi)
#pragma unroll
      for (int tt = 0; tt < 2; ++tt)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[gi][tt][j] = 0.0f;

#pragma unroll
    for (int s = 0; s < kStages - 1; ++s) {
      if (s < nslab)
        issue_stage(smem + s * kStageBytes, dq, ds, dq + 16 * qrow, ds + 16 * srow, qrow, srow,
                    s * 256, min(8, (a.I - s * 256) >> 5), false, lane);
      cp_async_commit();
    }
    for (int slab = 0; slab < nslab; ++slab) {
      cp_async_wait<kStages - 2>();
      __syncwarp();
      {
        const int nx = slab + kStages - 1;
        if (nx < nslab)
          issue_stage(smem + (nx % kStages) * kStageBytes, dq, ds, dq + 16 * qrow, ds + 16 * srow,
                      qrow, srow, nx * 256, min(8, (a.I - nx * 256) >> 5), false, lane);
        cp_async_commit();
      }
      const uint8_t* st = smem + (slab % kStages) * kStageBytes;
      const uint8_t* ss = st + kStageWBytes;
      const int kb = slab * 256;
      const int nbp = min(8, (a.I - kb) >> 5) >> 1;
      // the slab's h of token group 0 and its group scales, all loads in flight at once
      uint4 hpre[8];
      float hspre[8][2][2];
#pragma unroll
      for (int b = 0; b < 8; ++b) {
        const bool in = b < 2 * nbp;
        hpre[b] = in ? ldg16(hrow[0] + kb + 32 * b) : make_uint4(0u, 0u, 0u, 0u);
#pragma unroll
        for (int cc = 0; cc < 2; ++cc) {
          const int col = 2 * t + cc;
          const bool ok = in && col < n;
          const float* hsr = a.hscale + (size_t)(r0 + c0 + col) * (a.I >> 4) + 2 * ((kb >> 5) + b);
          hspre[b][0][cc] = ok ? __ldg(hsr) : 0.0f;
          hspre[b][1][cc] = ok ? __ldg(hsr + 1) : 0.0f;
        }
      }
#pragma unroll
      for (int bp = 0; bp < 4; ++bp) {
        if (bp < nbp) {
          uint32_t R0[4], R1[4];
          load_tile_pair(R0, st, 0, bp, lane);
          load_tile_pair(R1, st, 16, bp, lane);
#pragma unroll
          for (int hb = 0; hb < 2; ++hb) {
            const int b = 2 * bp + hb;
            uint32_t a00[4], a01[4], a10[4], a11[4];
            decode_block(R0[2 * hb], R0[2 * hb + 1], a00, a01);
            decode_block(R1[2 * hb], R1[2 * hb + 1], a10, a11);
            float ws[2][2];
            ws[0][0] = e8m0_to_f32(ss[g * 8 + b]);
            ws[0][1] = e8m0_to_f32(ss[(g + 8) * 8 + b]);
            ws[1][0] = e8m0_to_f32(ss[(g + 16) * 8 + b]);
            ws[1][1] = e8m0_to_f32(ss[(g + 24) * 8 + b]);
            const int hb16 = 2 * ((kb >> 5) + b);   // h group of the first MMA of this block
#pragma unroll
            for (int gi = 0; gi < 4; ++gi) {
              if (gi < ng) {
                uint4 hv;
                float hs0[2], hs1[2];
                if (gi == 0) {
                  hv = hpre[b];
#pragma unroll
                  for (int c = 0; c < 2; ++c) { hs0[c] = hspre[b][0][c]; hs1[c] = hspre[b][1][c]; }
                } else {
                  hv = ldg16(hrow[gi] + kb + 32 * b);
#pragma unroll
                  for (int c = 0; c < 2; ++c) {
                    const int col = gi * 8 + 2 * t + c;
                    const bool ok = col < n;
                    const float* hsr = a.hscale + (size_t)(r0 + c0 + col) * (a.I >> 4) + hb16;
                    hs0[c] = ok ? __ldg(hsr) : 0.0f;
                    hs1[c] = ok ? __ldg(hsr + 1) : 0.0f;
                  }
                }
                float c00[4] = {0.f, 0.f, 0.f, 0.f}, c01[4] = {0.f, 0.f, 0.f, 0.f};
                float c10[4] = {0.f, 0.f, 0.f, 0.f}, c11[4] = {0.f, 0.f, 0.f, 0.f};
                mma_f16(c00, a00, hv.x, hv.y);
                mma_f16(c01, a01, hv.z, hv.w);
                mma_f16(c10, a10, hv.x, hv.y);
                mma_f16(c11, a11, hv.z, hv.w);
#pragma unroll
                for (int j = 0; j < 4; ++j) {
                  const float v0 = fmaf(c01[j], hs1[j & 1], c00[j] * hs0[j & 1]);
                  const float v1 = fmaf(c11[j], hs1[j & 1], c10[j] * hs0[j & 1]);
                  acc[gi][0][j] = fmaf(v0, ws[0][j >> 1], acc[gi][0][j]);
                  acc[gi][1][j] = fmaf(v1, ws[1][j >> 1], acc[gi][1][j]);
                }
              }
            }
          }
        }
      }
    }
    cp_async_wait<0>();
    __syncwarp();
#pragma unroll
    for (int gi = 0; gi < 4; ++gi) {
      if (gi < ng) {
#pragma unroll
        for (int tt = 0; tt < 2; ++tt)
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int col = gi * 8 + 2 * t + (j & 1);
            if (col < n)
              a.y_perm[(size_t)(r0 + c0 + col) * a.W + n0 + tt * 16 + g + 8 * (j >> 1)] =
                  acc[gi][tt][j];
          }
      }
    }
  }
  }  // items
}

// ---------------------------------------------------------------------------
// gate/up + SwiGLU of the experts with 2+ tokens, CTA-wide TMA ring
// block = 32 * (kMmaConsumers + 1), one CTA per SM, dynamic smem
// mma_gateup_smem_bytes(); work item = (multi-token expert, 64-row group of
// I), numbered group-major so that every CTA's contiguous share mixes
// experts with many and few tokens (the MMA work grows with them); a stage holds one 512-element K slice: gate and up codes (two 128-byte
// boxes x 64 rows each, 128-byte swizzle, the layout ldmatrix reads), their
// scales (16 bytes x 64 rows), and the slice of every token row (f16, rows
// 1040 bytes apart so the B-fragment loads spread over the banks). Consumer
// warp w takes row tile w % 4 (the interleaved 16-row set whose h group is
// one MMA of the down projection) over K half w / 4 of the slice; the two
// halves are added through shared memory at the end of the item.
// ---------------------------------------------------------------------------
namespace {
constexpr int kMgRows = 64;                          // weight rows per item and matrix
constexpr int kMgBox = kMgRows * 128;                // one code box
constexpr int kMgCodes = 2 * kMgBox;                 // one matrix's codes of a stage (512 K)
constexpr int kMgScales = kMgRows * 16;              // one matrix's scales of a stage
constexpr int kMgXStride = 1040;                     // token row stride in the stage
constexpr int kMgXOff = 2 * kMgCodes + 2 * kMgScales;
constexpr int kMgTok = 32;                           // tokens per pass over the weights
constexpr int kMgStage = (kMgXOff + kMgTok * kMgXStride + 1023) / 1024 * 1024;
constexpr int kMgRed = 4 * 32 * 32 * 4;              // K-half partial sums [tile][lane][32]
}  // namespace

__global__ void __launch_bounds__(32 * (kMmaConsumers + 1), 1) k_mma_gateup(const __grid_constant__ MmaGateUpArgs A) {
  pdl_wait();
  pdl_trigger();
  const GateUpArgs& a = A.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_red = reinterpret_cast<float*>(smem + kMmaStages * kMgStage);
  __shared__ int16_t s_list[1024];      // experts with >= min_tokens tokens, in expert-list order
  __shared__ int s_wsum[kMmaConsumers + 1];
  __shared__ uint64_t s_bars[2 * kMmaStages];
  __shared__ int s_abort;
  constexpr int kWarps = kMmaConsumers + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = a.W, I = a.I;

  // 1) the multi-token experts
  const int n_act = __ldg(a.expert_list);
  int n_multi = 0;
  for (int base = 0; base < n_act; base += 32 * kWarps) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < n_act) {
      e = __ldg(a.expert_list + 1 + i);
      if (__ldg(a.offsets + e + 1) - __ldg(a.offsets + e) < a.min_tokens) e = -1;
    }
    const unsigned m = __ballot_sync(0xFFFFFFFFu, e >= 0);
    if (lane == 0) s_wsum[warp] = __popc(m);
    __syncthreads();
    int before = n_multi;
    for (int w = 0; w < warp; ++w) before += s_wsum[w];
    if (e >= 0) s_list[before + __popc(m & ((1u << lane) - 1u))] = (int16_t)e;
    for (int w = 0; w < kWarps; ++w) n_multi += s_wsum[w];
    __syncthreads();
  }
  // 2) this CTA's items: contiguous share of n_multi * (I / 64)
  const int groups = I / kMgRows;
  const long total = (long)n_multi * groups;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kMmaStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmaStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMmaConsumers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  const int nslice = (W + 511) / 512;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      uint32_t last_ph[kMmaStages];
      bool filled[kMmaStages];
      for (int s = 0; s < kMmaStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      bool ok = true;
      for (long it = lo; it < hi && ok; ++it) {
        const int e = s_list[it % n_multi], rg = (int)(it / n_multi);   // group-major: hot and cold experts mix
        const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
        const int wrow = e * I + rg * kMgRows;
        for (int c0 = 0; c0 < n_all && ok; c0 += kMgTok) {
          const int nt = min(kMgTok, n_all - c0);
          for (int s = 0; s < nslice; ++s) {
            if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) { ok = false; break; }
            uint8_t* st = smem + (size_t)slot * kMgStage;
            const uint32_t xb = (uint32_t)min(512, W - s * 512) * 2u;
            fence_proxy_async_smem();
            mbar_expect_tx(&full[slot], 2 * kMgCodes + 2 * kMgScales + nt * xb);
            tc::tma_load_2d(st, &A.map_gq, s * 256, wrow, &full[slot]);
            tc::tma_load_2d(st + kMgBox, &A.map_gq, s * 256 + 128, wrow, &full[slot]);
            tc::tma_load_2d(st + kMgCodes, &A.map_uq, s * 256, wrow, &full[slot]);
            tc::tma_load_2d(st + kMgCodes + kMgBox, &A.map_uq, s * 256 + 128, wrow, &full[slot]);
            tc::tma_load_2d(st + 2 * kMgCodes, &A.map_gs, s * 16, wrow, &full[slot]);
            tc::tma_load_2d(st + 2 * kMgCodes + kMgScales, &A.map_us, s * 16, wrow, &full[slot]);
            for (int c = 0; c < nt; ++c) {
              const int tok = __ldg(a.row_token + r0 + c0 + c);
              bulk_g2s(st + kMgXOff + c * kMgXStride, a.x16 + (size_t)tok * W + s * 512, xb, &full[slot]);
            }
            last_ph[slot] = ph;
            filled[slot] = true;
            if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
          }
        }
      }
      if (*abort) {
        for (int s = 0; s < kMmaStages; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int tt = w & 3, kh = w >> 2;                 // row tile, K half of the slice
    const int g = lane >> 2, t4 = lane & 3;
    const int i0t = 32 * (tt >> 1) + 4 * (tt & 1);     // first row of the tile in the group
    // smem rows of this lane's ldmatrix address and of its fragment rows g, g + 8
    const int lq = lane >> 3, lr = lane & 7;
    const int ldrow = i0t + tile_row((lq & 1) * 8 + lr, true);
    const int row_g = i0t + tile_row(g, true), row_g8 = i0t + tile_row(g + 8, true);
    int slot = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long it = lo; it < hi && ok; ++it) {
      const int e = s_list[it % n_multi], rg = (int)(it / n_multi);   // group-major: hot and cold experts mix
      const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
      const int q = rg * 4 + tt;                        // the 16-row tile (h group) index within I
      const int i0 = 32 * (q >> 1) + 4 * (q & 1);
      for (int c0 = 0; c0 < n_all; c0 += kMgTok) {
        const int n = min(kMgTok, n_all - c0);
        const int ng = (n + 7) >> 3;
        float accG[4][4], accU[4][4];
#pragma unroll
        for (int gi = 0; gi < 4; ++gi)
#pragma unroll
          for (int j = 0; j < 4; ++j) accG[gi][j] = accU[gi][j] = 0.0f;
        for (int s = 0; s < nslice; ++s) {
          if (!tc::wait_or_abort(&full[slot], ph, abort)) { ok = false; break; }
          const uint8_t* st = smem + (size_t)slot * kMgStage;
          const uint32_t gbox = smem_u32(st + kh * kMgBox), ubox = smem_u32(st + kMgCodes + kh * kMgBox);
          const uint8_t* gsc = st + 2 * kMgCodes;
          const uint8_t* usc = gsc + kMgScales;
          const uint32_t xs0 = smem_u32(st + kMgXOff);
          const int nblk = min(16, (W - s * 512) >> 5);   // valid 32-element blocks of the slice
#pragma unroll
          for (int bp = 0; bp < 4; ++bp) {
            const int b0 = 8 * kh + 2 * bp;
            if (b0 < nblk) {
              uint32_t Rg[4], Ru[4];
              const int ch = 2 * bp + (lq >> 1);           // 16-byte chunk within the box row
              ldmatrix_x4(Rg, gbox + ldrow * 128 + ((ch ^ (ldrow & 7)) << 4));
              ldmatrix_x4(Ru, ubox + ldrow * 128 + ((ch ^ (ldrow & 7)) << 4));
#pragma unroll
              for (int hb = 0; hb < 2; ++hb) {
                const int b = b0 + hb;
                uint32_t ag0[4], ag1[4], au0[4], au1[4];
                decode_block(Rg[2 * hb], Rg[2 * hb + 1], ag0, ag1);
                decode_block(Ru[2 * hb], Ru[2 * hb + 1], au0, au1);
                const float sg0 = e8m0_to_f32(gsc[row_g * 16 + b]);
                const float sg8 = e8m0_to_f32(gsc[row_g8 * 16 + b]);
                const float su0 = e8m0_to_f32(usc[row_g * 16 + b]);
                const float su8 = e8m0_to_f32(usc[row_g8 * 16 + b]);
#pragma unroll
                for (int gi = 0; gi < 4; ++gi) {
                  if (gi < ng) {
                    const int tok = min(gi * 8 + g, n - 1);
                    const uint4 xv = lds16(xs0 + tok * kMgXStride + (32 * b + 8 * t4) * 2);
                    float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
                    mma_f16(cg, ag0, xv.x, xv.y);
                    mma_f16(cg, ag1, xv.z, xv.w);
                    mma_f16(cu, au0, xv.x, xv.y);
                    mma_f16(cu, au1, xv.z, xv.w);
                    accG[gi][0] = fmaf(cg[0], sg0, accG[gi][0]);
                    accG[gi][1] = fmaf(cg[1], sg0, accG[gi][1]);
                    accG[gi][2] = fmaf(cg[2], sg8, accG[gi][2]);
                    accG[gi][3] = fmaf(cg[3], sg8, accG[gi][3]);
                    accU[gi][0] = fmaf(cu[0], su0, accU[gi][0]);
                    accU[gi][1] = fmaf(cu[1], su0, accU[gi][1]);
                    accU[gi][2] = fmaf(cu[2], su8, accU[gi][2]);
                    accU[gi][3] = fmaf(cu[3], su8, accU[gi][3]);
                  }
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&empty[slot]);
          if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        // the two K halves of tile tt: half 1 hands its sums to half 0
        float* red = s_red + (size_t)(tt * 32 + lane) * 32;
        if (kh == 1) {
#pragma unroll
          for (int gi = 0; gi < 4; ++gi)
#pragma unroll
            for (int j = 0; j < 4; ++j) { red[gi * 4 + j] = accG[gi][j]; red[16 + gi * 4 + j] = accU[gi][j]; }
        }
        asm volatile("bar.sync %0, 64;\n" ::"r"(1 + tt) : "memory");
        if (kh == 0) {
#pragma unroll
          for (int gi = 0; gi < 4; ++gi)
#pragma unroll
            for (int j = 0; j < 4; ++j) { accG[gi][j] += red[gi * 4 + j]; accU[gi][j] += red[16 + gi * 4 + j]; }
          // epilogue: h = silu(G) * U, one power-of-two scale per (token, 16 rows)
#pragma unroll
          for (int gi = 0; gi < 4; ++gi) {
            if (gi < ng) {
              float h[4];
              float xs[2];
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int col = gi * 8 + 2 * t4 + c;
                xs[c] = (col < n) ? __ldg(a.xscale + __ldg(a.row_token + r0 + c0 + col)) : 0.0f;
              }
#pragma unroll
              for (int j = 0; j < 4; ++j) h[j] = silu_f32(accG[gi][j] * xs[j & 1]) * (accU[gi][j] * xs[j & 1]);
              float m0 = fmaxf(fabsf(h[0]), fabsf(h[2]));
              float m1 = fmaxf(fabsf(h[1]), fabsf(h[3]));
#pragma unroll
              for (int off = 4; off < 32; off <<= 1) {
                m0 = fmaxf(m0, __shfl_xor_sync(0xFFFFFFFFu, m0, off));
                m1 = fmaxf(m1, __shfl_xor_sync(0xFFFFFFFFu, m1, off));
              }
              float sc[2], inv[2];
              f16_block_scale(m0, sc[0], inv[0]);
              f16_block_scale(m1, sc[1], inv[1]);
#pragma unroll
              for (int j = 0; j < 4; ++j) {
                const int col = gi * 8 + 2 * t4 + (j & 1);
                if (col < n) {
                  const int row = tile_row(g + 8 * (j >> 1), true);
                  a.h16[(size_t)(r0 + c0 + col) * I + i0 + row] = __float2half_rn(h[j] * inv[j & 1]);
                }
              }
              if (g == 0) {
#pragma unroll
                for (int c = 0; c < 2; ++c) {
                  const int col = gi * 8 + 2 * t4 + c;
                  if (col < n) a.hscale[(size_t)(r0 + c0 + col) * (I >> 4) + q] = sc[c];
                }
              }
            }
          }
        }
        asm volatile("bar.sync %0, 64;\n" ::"r"(1 + tt) : "memory");   // red free again
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(A.status, kStatusWaitTimeout);
}

size_t mma_gateup_smem_bytes() { return 1024 + (size_t)kMmaStages * kMgStage + kMgRed; }

// ---------------------------------------------------------------------------
// down projection of the experts with 2+ tokens, CTA-wide TMA ring
// block = 32 * (kMmaConsumers + 1), one CTA per SM; work item = (multi-token
// expert, 128-row group of W), numbered group-major as in k_mma_gateup; a stage holds one 512-element K slice: the
// down codes (two 128-byte boxes x 128 rows, 128-byte swizzle), their scales
// (16 bytes x 128 rows), every token's h slice (f16, rows 1040 bytes apart)
// and its 32 group scales; warp w takes the 16-row tile w over the whole
// slice (the items are short: K = I is a few slices).
// ---------------------------------------------------------------------------
namespace {
constexpr int kMdRows = 128;
constexpr int kMdBox = kMdRows * 128;
constexpr int kMdCodes = 2 * kMdBox;
constexpr int kMdScales = kMdRows * 16;
constexpr int kMdHsOff = kMdCodes + kMdScales;                   // h rows
constexpr int kMdScOff = kMdHsOff + kMgTok * kMgXStride;         // h group scales, 128 bytes per token
constexpr int kMdStage = (kMdScOff + kMgTok * 128 + 1023) / 1024 * 1024;
}  // namespace

__global__ void __launch_bounds__(32 * (kMmaConsumers + 1), 1) k_mma_down(const __grid_constant__ MmaDownArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  __shared__ int16_t s_list[1024];
  __shared__ int s_wsum[kMmaConsumers + 1];
  __shared__ uint64_t s_bars[2 * kMmaStages];
  __shared__ int s_abort;
  constexpr int kWarps = kMmaConsumers + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = a.W, I = a.I;

  const int n_act = __ldg(a.expert_list);
  int n_multi = 0;
  for (int base = 0; base < n_act; base += 32 * kWarps) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < n_act) {
      e = __ldg(a.expert_list + 1 + i);
      if (__ldg(a.offsets + e + 1) - __ldg(a.offsets + e) < a.min_tokens) e = -1;
    }
    const unsigned m = __ballot_sync(0xFFFFFFFFu, e >= 0);
    if (lane == 0) s_wsum[warp] = __popc(m);
    __syncthreads();
    int before = n_multi;
    for (int w = 0; w < warp; ++w) before += s_wsum[w];
    if (e >= 0) s_list[before + __popc(m & ((1u << lane) - 1u))] = (int16_t)e;
    for (int w = 0; w < kWarps; ++w) n_multi += s_wsum[w];
    __syncthreads();
  }
  const int groups = W / kMdRows;
  const long total = (long)n_multi * groups;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kMmaStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmaStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMmaConsumers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  const int nslice = I / 512;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      uint32_t last_ph[kMmaStages];
      bool filled[kMmaStages];
      for (int s = 0; s < kMmaStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      bool ok = true;
      for (long it = lo; it < hi && ok; ++it) {
        const int e = s_list[it % n_multi], rg = (int)(it / n_multi);   // group-major: hot and cold experts mix
        const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
        const int wrow = e * W + rg * kMdRows;
        for (int c0 = 0; c0 < n_all && ok; c0 += kMgTok) {
          const int nt = min(kMgTok, n_all - c0);
          for (int s = 0; s < nslice; ++s) {
            if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) { ok = false; break; }
            uint8_t* st = smem + (size_t)slot * kMdStage;
            fence_proxy_async_smem();
            mbar_expect_tx(&full[slot], kMdCodes + kMdScales + nt * (1024 + 128));
            tc::tma_load_2d(st, &a.map_dq, s * 256, wrow, &full[slot]);
            tc::tma_load_2d(st + kMdBox, &a.map_dq, s * 256 + 128, wrow, &full[slot]);
            tc::tma_load_2d(st + kMdCodes, &a.map_ds, s * 16, wrow, &full[slot]);
            for (int c = 0; c < nt; ++c) {
              const size_t r = (size_t)(r0 + c0 + c);
              bulk_g2s(st + kMdHsOff + c * kMgXStride, a.h16 + r * I + s * 512, 1024u, &full[slot]);
              bulk_g2s(st + kMdScOff + c * 128, a.hscale + r * (I >> 4) + s * 32, 128u, &full[slot]);
            }
            last_ph[slot] = ph;
            filled[slot] = true;
            if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
          }
        }
      }
      if (*abort) {
        for (int s = 0; s < kMmaStages; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int tt = warp - 1;                            // 16-row tile of the item
    const int g = lane >> 2, t4 = lane & 3;
    const int lq = lane >> 3, lr = lane & 7;
    const int ldrow = 16 * tt + (lq & 1) * 8 + lr;
    const int row_g = 16 * tt + g, row_g8 = row_g + 8;
    int slot = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long it = lo; it < hi && ok; ++it) {
      const int e = s_list[it % n_multi], rg = (int)(it / n_multi);   // group-major: hot and cold experts mix
      const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
      const int n0 = rg * kMdRows + 16 * tt;             // first output column (row of Wd) of the tile
      for (int c0 = 0; c0 < n_all; c0 += kMgTok) {
        const int n = min(kMgTok, n_all - c0);
        const int ng = (n + 7) >> 3;
        float acc[4][4];
#pragma unroll
        for (int gi = 0; gi < 4; ++gi)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[gi][j] = 0.0f;
        for (int s = 0; s < nslice; ++s) {
          if (!tc::wait_or_abort(&full[slot], ph, abort)) { ok = false; break; }
          const uint8_t* st = smem + (size_t)slot * kMdStage;
          const uint32_t cod = smem_u32(st);
          const uint8_t* wsc = st + kMdCodes;
          const uint32_t hs0a = smem_u32(st + kMdHsOff);
          const float* hsc = reinterpret_cast<const float*>(st + kMdScOff);
#pragma unroll 2
          for (int bp = 0; bp < 8; ++bp) {
            uint32_t R[4];
            const int ch = 2 * (bp & 3) + (lq >> 1);
            ldmatrix_x4(R, cod + (bp >> 2) * kMdBox + ldrow * 128 + ((ch ^ (ldrow & 7)) << 4));
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
              const int b = 2 * bp + hb;
              uint32_t a0[4], a1[4];
              decode_block(R[2 * hb], R[2 * hb + 1], a0, a1);
              const float ws0 = e8m0_to_f32(wsc[row_g * 16 + b]);
              const float ws8 = e8m0_to_f32(wsc[row_g8 * 16 + b]);
#pragma unroll
              for (int gi = 0; gi < 4; ++gi) {
                if (gi < ng) {
                  const int tok = min(gi * 8 + g, n - 1);
                  const uint4 hv = lds16(hs0a + tok * kMgXStride + (32 * b + 8 * t4) * 2);
                  float hq0[2], hq1[2];
#pragma unroll
                  for (int cc = 0; cc < 2; ++cc) {
                    const int col = min(gi * 8 + 2 * t4 + cc, n - 1);
                    hq0[cc] = hsc[col * 32 + 2 * b];
                    hq1[cc] = hsc[col * 32 + 2 * b + 1];
                  }
                  float c00[4] = {0.f, 0.f, 0.f, 0.f}, c01[4] = {0.f, 0.f, 0.f, 0.f};
                  mma_f16(c00, a0, hv.x, hv.y);
                  mma_f16(c01, a1, hv.z, hv.w);
#pragma unroll
                  for (int j = 0; j < 4; ++j) {
                    const float v = fmaf(c01[j], hq1[j & 1], c00[j] * hq0[j & 1]);
                    acc[gi][j] = fmaf(v, (j >> 1) ? ws8 : ws0, acc[gi][j]);
                  }
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&empty[slot]);
          if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          if (gi < ng) {
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const int col = gi * 8 + 2 * t4 + (j & 1);
              if (col < n) a.y_perm[(size_t)(r0 + c0 + col) * W + n0 + g + 8 * (j >> 1)] = acc[gi][j];
            }
          }
        }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
}

size_t mma_down_smem_bytes() { return 1024 + (size_t)kMmaStages * kMdStage; }

size_t gemv_mxfp4_smem_bytes() { return (size_t)kStages * kStageBytes; }

}  // namespace moe
