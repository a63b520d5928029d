// Router tail: softmax top-k with renormalised weights (rabbit README, model
// table row "MoE routing": softmax top-10 of 512).
//
// One CTA per token. The router logits arrive as split-K partial sums
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

// grid T, block 256: the CTA sums the S partial logits of its token (all
// threads, independent loads), then warp 0 selects the top k.
__global__ void __launch_bounds__(256) k_topk(const float* __restrict__ part, int S, int T, int E,
                                              int k, int32_t* __restrict__ idx,
                                              float* __restrict__ w, float* __restrict__ logits) {
  pdl_wait();
  pdl_trigger();
  __shared__ float lg[1024];
  const int tok = blockIdx.x;
  for (int e = threadIdx.x; e < E; e += 256) {
    const float* p = part + (size_t)tok * E + e;
    const size_t stride = (size_t)T * E;
    float acc = 0.0f;
    int s = 0;
    for (; s + 4 <= S; s += 4) {                // fixed summation order s = 0, 1, 2, ...
      const float v0 = __ldg(p + (s + 0) * stride), v1 = __ldg(p + (s + 1) * stride);
      const float v2 = __ldg(p + (s + 2) * stride), v3 = __ldg(p + (s + 3) * stride);
      acc += v0; acc += v1; acc += v2; acc += v3;
    }
    for (; s < S; ++s) acc += __ldg(p + s * stride);
    if (logits) logits[(size_t)tok * E + e] = acc;
    lg[e] = isnan(acc) ? -INFINITY : acc;      // a NaN logit never wins
  }
  __syncthreads();
  if (threadIdx.x >= 32) return;
  const int lane = threadIdx.x;
  float v[kMaxPerLane];
#pragma unroll
  for (int j = 0; j < kMaxPerLane; ++j) {
    const int e = lane + 32 * j;
    v[j] = (e < E) ? lg[e] : -INFINITY;
  }
  uint32_t taken = 0;
  float selv = 0.0f;     // lane r keeps the r-th selection
  int sele = 0;
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
    if (lane == r) { selv = bv; sele = be; }
  }
  const float m = __shfl_sync(0xFFFFFFFFu, selv, 0);
  const float ex = (lane < k) ? expf(selv - m) : 0.0f;
  float den = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, off);
  if (lane < k) {
    idx[(size_t)tok * k + lane] = sele;
    w[(size_t)tok * k + lane] = ex / den;
  }
}

}  // namespace moe
