// Router tail: softmax top-k with renormalised weights (rabbit README, model
// table row "MoE routing": softmax top-10 of 512).
//
// One warp per token. The router logits arrive as split-K partial sums
// [S, T, E] from k_dense_gemv and are summed in a fixed order (s = 0..S-1),
// so the logits, and with them the selection, are reproducible run to run.
// Selection ranks by fp32 logit (the softmax is monotone); equal logits go to
// the lower expert index. Weights: w_j = exp(l_j - l_max) / sum_sel exp(l - l_max),
// which equals the full softmax renormalised over the selected experts.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kMaxPerLane = 32;   // E <= 1024

// grid ceil(T/8), block 256 (8 warps, one token each)
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ part, int S, int T, int E,
                                              int k, int32_t* __restrict__ idx,
                                              float* __restrict__ w, float* __restrict__ logits) {
  const int lane = threadIdx.x & 31;
  const int tok = blockIdx.x * 8 + (threadIdx.x >> 5);
  if (tok >= T) return;
  float v[kMaxPerLane];
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int e = lane + 32 * j;
    float acc = -INFINITY;
    if (e < E) {
      acc = 0.0f;
      for (int s = 0; s < S; ++s) acc += __ldg(part + ((size_t)s * T + tok) * E + e);
      if (logits) logits[(size_t)tok * E + e] = acc;
      if (isnan(acc)) acc = -INFINITY;      // a NaN logit never wins
    }
    v[j] = acc;
  }
  uint32_t taken = 0;
  float selv[32];
  int sele[32];
  for (int r = 0; r < k; ++r) {
    float bv = -INFINITY;
    int be = 0x7FFFFFFF;
#pragma unroll
    for (int j = 0; j < kMaxPerLane; ++j) {
      const int e = lane + 32 * j;
      if (e < E && !((taken >> j) & 1u)) {
        if (v[j] > bv || be == 0x7FFFFFFF) { bv = v[j]; be = e; }
      }
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) {
      const float ov = __shfl_xor_sync(0xFFFFFFFFu, bv, off);
      const int oe = __shfl_xor_sync(0xFFFFFFFFu, be, off);
      if (ov > bv || (ov == bv && oe < be)) { bv = ov; be = oe; }
    }
    if ((be & 31) == lane) taken |= 1u << (be >> 5);
    selv[r] = bv;
    sele[r] = be;
  }
  if (lane == 0) {
    const float m = selv[0];
    float den = 0.0f;
    for (int r = 0; r < k; ++r) den += expf(selv[r] - m);
    for (int r = 0; r < k; ++r) {
      idx[(size_t)tok * k + r] = sele[r];
      w[(size_t)tok * k + r] = expf(selv[r] - m) / den;
    }
  }
}

}  // namespace moe
