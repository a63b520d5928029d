// Dense bf16 GEMV / skinny GEMM with split-K partial sums (router logits, the
// shared expert, the latent projections).
//
// Y_part[s, t, n] = sum_{k in split s} W[n, k] * X[t, k]
//
// One warp per 16-row tile of W, one K split and up to 32 tokens. Weights are
// read straight from HBM into registers with 16-byte streaming loads: lane
// (g, t) of the warp loads 8 consecutive K elements of rows g and g+8, which
// is an mma.m16n8k16 A fragment once K is permuted inside each 32-element step
// (the same permutation is applied to the activation fragment, so the dot
// products are unchanged). Products of bf16 values are exact and accumulate
// in fp32. An fp32 activation (h of the shared expert, the latent weighted
// sum) is split into bf16 hi + lo parts and multiplied twice, which keeps
// about 16 significant bits of it.
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

MOE_DEV const uint16_t* dense_row(const DenseArgs& a, int n) {
  if (n < a.rows[0]) return a.w[0] + (size_t)n * a.K;
  n -= a.rows[0];
  if (n < a.rows[1]) return a.w[1] + (size_t)n * a.K;
  n -= a.rows[1];
  return a.w[2] + (size_t)n * a.K;
}

MOE_DEV uint32_t pack_bf16(uint32_t lo, uint32_t hi) { return lo | (hi << 16); }

// hi/lo bf16 split of 8 floats -> (hi words, lo words), 4 each
MOE_DEV void split8(const float (&v)[8], uint32_t (&hw)[4], uint32_t (&lw)[4]) {
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const uint32_t h0 = f32_to_bf16_rne(v[2 * i]), h1 = f32_to_bf16_rne(v[2 * i + 1]);
    const uint32_t l0 = f32_to_bf16_rne(v[2 * i] - bf16_to_f32(h0));
    const uint32_t l1 = f32_to_bf16_rne(v[2 * i + 1] - bf16_to_f32(h1));
    hw[i] = pack_bf16(h0, h1);
    lw[i] = pack_bf16(l0, l1);
  }
}

}  // namespace

// grid (ceil(N / (16*kDenseWarps)), S, ceil(T/32)), block 32*kDenseWarps
__global__ void __launch_bounds__(32 * kDenseWarps) k_dense_gemv(DenseArgs a) {
  pdl_wait();
  pdl_trigger();
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int g = lane >> 2, t = lane & 3;
  const int n0 = (blockIdx.x * kDenseWarps + warp) * 16;
  if (n0 >= a.N) return;
  const int s = blockIdx.y;
  const int tok0 = blockIdx.z * 32;
  const int nt = min(32, a.T - tok0);
  const int ng = (nt + 7) >> 3;
  const int na = min(n0 + g, a.N - 1), nb = min(n0 + g + 8, a.N - 1);
  const int kbeg = s * a.kper;
  const uint16_t* wa = dense_row(a, na) + kbeg + 8 * t;
  const uint16_t* wb = dense_row(a, nb) + kbeg + 8 * t;

  // activation row of this lane for each token group
  const char* xr[4];
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    const int tok = tok0 + min(gi * 8 + g, nt - 1);
    xr[gi] = a.x_f32
                 ? reinterpret_cast<const char*>(static_cast<const float*>(a.x) + (size_t)tok * a.K + kbeg + 8 * t)
                 : reinterpret_cast<const char*>(static_cast<const uint16_t*>(a.x) + (size_t)tok * a.K + kbeg + 8 * t);
  }
  float acc[4][4];
#pragma unroll
  for (int gi = 0; gi < 4; ++gi)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[gi][j] = 0.0f;

  constexpr int U = 4;   // k-steps of 32 in flight
  const int nsteps = a.kper >> 5;
  for (int k0 = 0; k0 < nsteps; k0 += U) {
    uint4 va[U], vb[U];
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k0 + u < nsteps) {
        va[u] = ldg_stream(wa + (k0 + u) * 32);
        vb[u] = ldg_stream(wb + (k0 + u) * 32);
      }
    }
#pragma unroll
    for (int u = 0; u < U; ++u) {
      if (k0 + u < nsteps) {
        const uint32_t A0[4] = {va[u].x, vb[u].x, va[u].y, vb[u].y};
        const uint32_t A1[4] = {va[u].z, vb[u].z, va[u].w, vb[u].w};
        const int koff = (k0 + u) * 32;
#pragma unroll
        for (int gi = 0; gi < 4; ++gi) {
          if (gi < ng) {
            if (!a.x_f32) {
              const uint4 xv = ldg16(reinterpret_cast<const uint16_t*>(xr[gi]) + koff);
              mma_bf16(acc[gi], A0, xv.x, xv.y);
              mma_bf16(acc[gi], A1, xv.z, xv.w);
            } else {
              const float* xf = reinterpret_cast<const float*>(xr[gi]) + koff;
              const float4 p = __ldg(reinterpret_cast<const float4*>(xf));
              const float4 q = __ldg(reinterpret_cast<const float4*>(xf + 4));
              const float v[8] = {p.x, p.y, p.z, p.w, q.x, q.y, q.z, q.w};
              uint32_t hw[4], lw[4];
              split8(v, hw, lw);
              mma_bf16(acc[gi], A0, hw[0], hw[1]);
              mma_bf16(acc[gi], A1, hw[2], hw[3]);
              mma_bf16(acc[gi], A0, lw[0], lw[1]);
              mma_bf16(acc[gi], A1, lw[2], lw[3]);
            }
          }
        }
      }
    }
  }
#pragma unroll
  for (int gi = 0; gi < 4; ++gi) {
    if (gi < ng) {
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int col = gi * 8 + 2 * t + (j & 1);
        const int n = n0 + g + 8 * (j >> 1);
        if (col < nt && n < a.N)
          a.part[((size_t)s * a.T + tok0 + col) * a.N + n] = acc[gi][j];
      }
    }
  }
}

}  // namespace moe
