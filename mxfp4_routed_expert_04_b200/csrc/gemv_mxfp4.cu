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

size_t gemv_mxfp4_smem_bytes() { return (size_t)kStages * kStageBytes; }

}  // namespace moe
