// Combine and the finalisers of split-K partial sums.
//
// k_combine: y[t] = sum_j w[t, j] * y_perm[slot_row[t, j]]          (routed, slots in order)
//                 + sum_s add1[s, t]                                 (e.g. latent up-projection)
//                 + sigmoid(gate_logit[t]) * sum_s add2[s, t]        (gated shared expert)
// Every sum runs in a fixed order, so the output is reproducible bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// grid (ceil(width/4/256), T), block 256; width a multiple of 4
__global__ void __launch_bounds__(256) k_combine(CombineArgs a) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int c = (blockIdx.x * 256 + threadIdx.x) * 4;
  if (c >= a.width) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  if (a.y_perm) {
    for (int j = 0; j < a.k; ++j) {
      const int r = __ldg(a.slot_row + (size_t)t * a.k + j);
      const float wj = __ldg(a.topk_w + (size_t)t * a.k + j);
      const float4 v = __ldg(reinterpret_cast<const float4*>(a.y_perm + (size_t)r * a.width + c));
      acc.x = fmaf(wj, v.x, acc.x);
      acc.y = fmaf(wj, v.y, acc.y);
      acc.z = fmaf(wj, v.z, acc.z);
      acc.w = fmaf(wj, v.w, acc.w);
    }
  }
  if (a.add1) {
    for (int s = 0; s < a.S1; ++s) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(a.add1 + ((size_t)s * a.T + t) * a.width + c));
      acc.x += v.x; acc.y += v.y; acc.z += v.z; acc.w += v.w;
    }
  }
  if (a.add2) {
    float4 sh = make_float4(0.f, 0.f, 0.f, 0.f);
    for (int s = 0; s < a.S2; ++s) {
      const float4 v = __ldg(reinterpret_cast<const float4*>(a.add2 + ((size_t)s * a.T + t) * a.width + c));
      sh.x += v.x; sh.y += v.y; sh.z += v.z; sh.w += v.w;
    }
    const float gt = sigmoid_f32(__ldg(a.gate_logit + t));
    acc.x = fmaf(gt, sh.x, acc.x);
    acc.y = fmaf(gt, sh.y, acc.y);
    acc.z = fmaf(gt, sh.z, acc.z);
    acc.w = fmaf(gt, sh.w, acc.w);
  }
  *reinterpret_cast<float4*>(a.out + (size_t)t * a.width + c) = acc;
}

// Shared expert SwiGLU from the partials of its gate/up GEMV, whose rows are
// [Ws_gate (Is rows); Ws_up (Is rows); w_sgate (1 row)]:
//   hs[t, i] = silu(G[t, i]) * U[t, i],  gate_logit[t] = x[t] . w_sgate
// grid (ceil(Is/256), T), block 256
__global__ void __launch_bounds__(256) k_shared_swiglu(const float* __restrict__ part, int S, int T,
                                                     int Is, float* __restrict__ hs,
                                                     float* __restrict__ gate_logit) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int i = blockIdx.x * 256 + threadIdx.x;
  const int N = 2 * Is + 1;
  if (i < Is) {
    float G = 0.f, U = 0.f;
    for (int s = 0; s < S; ++s) {
      G += __ldg(part + ((size_t)s * T + t) * N + i);
      U += __ldg(part + ((size_t)s * T + t) * N + Is + i);
    }
    hs[(size_t)t * Is + i] = silu_f32(G) * U;
  }
  if (blockIdx.x == 0 && threadIdx.x == 0) {
    float gl = 0.f;
    for (int s = 0; s < S; ++s) gl += __ldg(part + ((size_t)s * T + t) * N + 2 * Is);
    gate_logit[t] = gl;
  }
}

// out[t, n] = bf16_rne( sum_s part[s, t, n] )   (latent down-projection)
// grid (ceil(N/256), T), block 256
__global__ void __launch_bounds__(256) k_round_bf16(const float* __restrict__ part, int S, int T,
                                                  int N, uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int n = blockIdx.x * 256 + threadIdx.x;
  if (n >= N) return;
  float v = 0.f;
  for (int s = 0; s < S; ++s) v += __ldg(part + ((size_t)s * T + t) * N + n);
  out[(size_t)t * N + n] = (uint16_t)f32_to_bf16_rne(v);
}

}  // namespace moe
