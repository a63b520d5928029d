// MXFP4 GEMV on the CUDA cores for experts that received exactly one token
// (every expert of a 1-token decode step; most experts of small batches).
//
// With one token a tensor-core MMA would use 1 of its 8 columns, and the
// legacy mma.sync rate of sm_100 then caps the kernel near half the HBM
// bandwidth. Here every thread owns BPT fixed 32-element K blocks of the
// activation row (kept in registers as f16) and streams the matching 16-byte
// slices of each weight row: a warp-wide load of one row is 512 contiguous
// bytes. Per 32 weights a thread spends 16 cvt.rn.f16x2.e2m1x2 (exact decode)
// and 32 fma.rn.f32.f16 (exact f16 x f16 product, fp32 accumulation), then one
// fp32 FMA applies the E8M0 block scale. Row sums are reduced across the CTA
// by a warp reduce-scatter and a shared-memory pass.
//
// The h produced here is f16 with one power-of-two scale per group of 16
// CONSECUTIVE intermediate rows (the tensor-core path uses interleaved groups;
// an expert's gate/up and down always take the same path).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

// Dot products of the two 16-element halves of one MXFP4 block with 32 f16
// activations (block scale not applied).
MOE_DEV void dot_block_halves(uint4 w, const uint32_t (&x)[16], float& p0, float& p1) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4];
    e2m1x8_to_f16x8(words[q], h);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a[(q >> 1) * 2] = fma_f16lo(h[j], x[4 * q + j], a[(q >> 1) * 2]);
      a[(q >> 1) * 2 + 1] = fma_f16hi(h[j], x[4 * q + j], a[(q >> 1) * 2 + 1]);
    }
  }
  p0 = a[0] + a[1];
  p1 = a[2] + a[3];
}

template <int BPT>
MOE_DEV void load_act_blocks(uint32_t (&xr)[BPT][16], const __half* row, int KB) {
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int b = threadIdx.x + j * blockDim.x;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (b < KB) v = ldg16(row + b * 32 + 8 * q);
      xr[j][4 * q] = v.x; xr[j][4 * q + 1] = v.y; xr[j][4 * q + 2] = v.z; xr[j][4 * q + 3] = v.w;
    }
  }
}

// CTA-wide sum of acc[32] (one value per row): returns row `lane`'s total in
// every lane of warp 0. `red` holds 32 x 33 floats.
MOE_DEV float cta_row_sums(float (&acc)[32], float (*red)[33]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float v = warp_reduce_scatter32(acc, lane);
  red[warp][lane] = v;
  __syncthreads();
  float s = 0.f;
  if (warp == 0)
    for (int w = 0; w < nw; ++w) s += red[w][lane];
  return s;
}

constexpr int kRowChunk = 8;   // weight rows whose loads are in flight together

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU for single-token experts
// persistent grid; block = KB/BPT threads rounded up to a warp (<= 256);
// work item = (active expert, 16-row tile of I), rows 0..15 gate, 16..31 up
// ---------------------------------------------------------------------------
template <int BPT>
__global__ void __launch_bounds__(kFmaMaxThreads) k_gateup_fma(GateUpArgs a) {
  __shared__ float red[32][33];
  const int KB = a.W >> 5;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tiles = a.I >> 4;
  const int items = __ldg(a.expert_list) * tiles;
  const size_t qrow = (size_t)a.W / 2, srow = (size_t)a.W / 32;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int ai = item / tiles, tile = item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const int r0 = __ldg(a.offsets + e);
    if (__ldg(a.offsets + e + 1) - r0 != 1) continue;      // tensor-core path
    const int tok = __ldg(a.row_token + r0);
    const int i0 = tile * 16;
    uint32_t xr[BPT][16];
    load_act_blocks<BPT>(xr, a.x16 + (size_t)tok * a.W, KB);
    const uint8_t* gq = a.wg_q + ((size_t)e * a.I + i0) * qrow;
    const uint8_t* gs = a.wg_s + ((size_t)e * a.I + i0) * srow;
    const uint8_t* uq = a.wu_q + ((size_t)e * a.I + i0) * qrow;
    const uint8_t* us = a.wu_s + ((size_t)e * a.I + i0) * srow;
    float acc[32];
#pragma unroll
    for (int rc = 0; rc < 32; rc += kRowChunk) {
      uint4 w[kRowChunk][BPT];
      uint32_t sc[kRowChunk][BPT];
#pragma unroll
      for (int rr = 0; rr < kRowChunk; ++rr) {
        const int r = rc + rr;
        const uint8_t* q = (r < 16 ? gq + r * qrow : uq + (r - 16) * qrow);
        const uint8_t* s = (r < 16 ? gs + r * srow : us + (r - 16) * srow);
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          const int b = threadIdx.x + j * blockDim.x;
          w[rr][j] = make_uint4(0u, 0u, 0u, 0u);
          sc[rr][j] = 127u;
          if (b < KB) {
            w[rr][j] = ldg_stream(q + b * 16);
            sc[rr][j] = __ldg(s + b);
          }
        }
      }
#pragma unroll
      for (int rr = 0; rr < kRowChunk; ++rr) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          float p0, p1;
          dot_block_halves(w[rr][j], xr[j], p0, p1);
          v = fmaf(p0 + p1, e8m0_to_f32(sc[rr][j]), v);
        }
        acc[rc + rr] = v;
      }
    }
    const float s = cta_row_sums(acc, red);
    if (warp == 0) {
      // lanes 0..15: gate row i0+lane; lanes 16..31: up row i0+lane-16
      const float xs = __ldg(a.xscale + tok);
      const float u = __shfl_down_sync(0xFFFFFFFFu, s, 16);
      const float h = silu_f32(s * xs) * (u * xs);
      float m = (lane < 16) ? fabsf(h) : 0.0f;
#pragma unroll
      for (int off = 8; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      float scale = 1.0f, inv = 1.0f;
      if (m > 0.0f && isfinite(m)) {
        int ex;
        frexpf(m, &ex);
        ex = max(-100, min(127, ex));
        scale = ldexpf(1.0f, ex - 15);
        inv = ldexpf(1.0f, 15 - ex);
      }
      if (lane < 16) a.h16[(size_t)r0 * a.I + i0 + lane] = __float2half_rn(h * inv);
      if (lane == 0) a.hscale[(size_t)tile * a.R + r0] = scale;
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// down projection for single-token experts
// persistent grid; block = KB/BPT threads (K = I); work item = (active
// expert, 32-row tile of W)
// ---------------------------------------------------------------------------
template <int BPT>
__global__ void __launch_bounds__(kFmaMaxThreads) k_down_fma(DownArgs a) {
  __shared__ float red[32][33];
  const int KB = a.I >> 5;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tiles = a.W >> 5;
  const int items = __ldg(a.expert_list) * tiles;
  const size_t qrow = (size_t)a.I / 2, srow = (size_t)a.I / 32;
  for (int item = blockIdx.x; item < items; item += gridDim.x) {
    const int ai = item / tiles, tile = item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const int r0 = __ldg(a.offsets + e);
    if (__ldg(a.offsets + e + 1) - r0 != 1) continue;      // tensor-core path
    const int n0 = tile * 32;
    uint32_t xr[BPT][16];
    load_act_blocks<BPT>(xr, a.h16 + (size_t)r0 * a.I, KB);
    float hs[BPT][2];
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      const int b = threadIdx.x + j * blockDim.x;
      hs[j][0] = hs[j][1] = 0.0f;
      if (b < KB) {
        hs[j][0] = __ldg(a.hscale + (size_t)(2 * b) * a.R + r0);
        hs[j][1] = __ldg(a.hscale + (size_t)(2 * b + 1) * a.R + r0);
      }
    }
    const uint8_t* dq = a.wd_q + ((size_t)e * a.W + n0) * qrow;
    const uint8_t* ds = a.wd_s + ((size_t)e * a.W + n0) * srow;
    float acc[32];
#pragma unroll
    for (int rc = 0; rc < 32; rc += kRowChunk) {
      uint4 w[kRowChunk][BPT];
      uint32_t sc[kRowChunk][BPT];
#pragma unroll
      for (int rr = 0; rr < kRowChunk; ++rr) {
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          const int b = threadIdx.x + j * blockDim.x;
          w[rr][j] = make_uint4(0u, 0u, 0u, 0u);
          sc[rr][j] = 127u;
          if (b < KB) {
            w[rr][j] = ldg_stream(dq + (rc + rr) * qrow + b * 16);
            sc[rr][j] = __ldg(ds + (rc + rr) * srow + b);
          }
        }
      }
#pragma unroll
      for (int rr = 0; rr < kRowChunk; ++rr) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          float p0, p1;
          dot_block_halves(w[rr][j], xr[j], p0, p1);
          v = fmaf(fmaf(p1, hs[j][1], p0 * hs[j][0]), e8m0_to_f32(sc[rr][j]), v);
        }
        acc[rc + rr] = v;
      }
    }
    const float s = cta_row_sums(acc, red);
    if (warp == 0) a.y_perm[(size_t)r0 * a.W + n0 + lane] = s;
    __syncthreads();
  }
}

template __global__ void k_gateup_fma<1>(GateUpArgs);
template __global__ void k_gateup_fma<2>(GateUpArgs);
template __global__ void k_down_fma<1>(DownArgs);
template __global__ void k_down_fma<2>(DownArgs);

}  // namespace moe
