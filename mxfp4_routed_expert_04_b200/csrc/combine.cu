// Combine and the finalisers of split-K partial sums.
//
// k_combine: y[t] = sum_j w[t, j] * y_perm[slot_row[t, j]]          (routed, slots in order)
//                 + sum_s add1[s, t]                                 (e.g. latent up-projection)
//                 + sigmoid(gate_logit[t]) * sum_s add2[s, t]        (gated shared expert)
// Every sum runs in a fixed order, so the output is reproducible bit for bit.
#include "common.cuh"
#include "kernels.h"

namespace moe {

// grid (ceil(width/4/kCombineThreads), T), block kCombineThreads; width a
// multiple of 4. Loads are issued in groups of four before their sums, which
// keep the order of the formula above.
__global__ void __launch_bounds__(kCombineThreads) k_combine(CombineArgs a) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int c = (blockIdx.x * kCombineThreads + threadIdx.x) * 4;
  if (c >= a.width) return;
  float4 acc = make_float4(0.f, 0.f, 0.f, 0.f);
  auto fma4 = [](float w, const float4& v, float4& o) {
    o.x = fmaf(w, v.x, o.x);
    o.y = fmaf(w, v.y, o.y);
    o.z = fmaf(w, v.z, o.z);
    o.w = fmaf(w, v.w, o.w);
  };
  auto add4 = [](const float4& v, float4& o) { o.x += v.x; o.y += v.y; o.z += v.z; o.w += v.w; };
  auto row4 = [&](const float* base, size_t row) {
    return __ldg(reinterpret_cast<const float4*>(base + row * a.width + c));
  };
  if (a.y_perm) {
    const int32_t* sr = a.slot_row + (size_t)t * a.k;
    const float* tw = a.topk_w + (size_t)t * a.k;
    int j = 0;
    for (; j + 4 <= a.k; j += 4) {
      int r[4];
      float w[4];
      float4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) { r[i] = __ldg(sr + j + i); w[i] = __ldg(tw + j + i); }
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = row4(a.y_perm, (size_t)r[i]);
#pragma unroll
      for (int i = 0; i < 4; ++i) fma4(w[i], v[i], acc);
    }
    for (; j < a.k; ++j) fma4(__ldg(tw + j), row4(a.y_perm, (size_t)__ldg(sr + j)), acc);
  }
  auto split_sum = [&](const float* part, int S, float4& o) {
    int s = 0;
    for (; s + 4 <= S; s += 4) {
      float4 v[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) v[i] = row4(part, (size_t)(s + i) * a.T + t);
#pragma unroll
      for (int i = 0; i < 4; ++i) add4(v[i], o);
    }
    for (; s < S; ++s) add4(row4(part, (size_t)s * a.T + t), o);
  };
  if (a.add1) split_sum(a.add1, a.S1, acc);
  if (a.add2) {
    float4 sh = make_float4(0.f, 0.f, 0.f, 0.f);
    split_sum(a.add2, a.S2, sh);
    fma4(sigmoid_f32(__ldg(a.gate_logit + t)), sh, acc);
  }
  if (a.out_hi) {
    // the operand pair of a bf16 tensor-core GEMM: hi + lo carries 16
    // significant bits of the fp32 sum
    const float v[4] = {acc.x, acc.y, acc.z, acc.w};
    uint32_t hi[4], lo[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      hi[i] = f32_to_bf16_rne(v[i]);
      lo[i] = f32_to_bf16_rne(v[i] - bf16_to_f32(hi[i]));
    }
    const size_t o = (size_t)t * a.width + c;
    *reinterpret_cast<uint2*>(a.out_hi + o) = make_uint2(hi[0] | hi[1] << 16, hi[2] | hi[3] << 16);
    *reinterpret_cast<uint2*>(a.out_lo + o) = make_uint2(lo[0] | lo[1] << 16, lo[2] | lo[3] << 16);
    return;
  }
  *reinterpret_cast<float4*>(a.out + (size_t)t * a.width + c) = acc;
}

// Shared expert SwiGLU from the split-K partials of its gate/up GEMM, whose
// rows are [Ws_gate (Is rows); Ws_up (Is rows); w_sgate (1 row)]:
//   h[t, i] = silu(G[t, i]) * U[t, i]   written as a bf16 pair hi = bf16(h),
//                                        lo = bf16(h - hi) (the down GEMM's operand)
//   gate_logit[t] = x[t] . w_sgate
// grid (ceil(Is/kFinThreads), T), block kFinThreads
__global__ void __launch_bounds__(kFinThreads) k_shared_swiglu(const float* __restrict__ part, int S,
                                                             int T, int Is, uint16_t* __restrict__ h_hi,
                                                             uint16_t* __restrict__ h_lo,
                                                             float* __restrict__ gate_logit) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int i = blockIdx.x * kFinThreads + threadIdx.x;
  const int N = 2 * Is + 1;
  if (i < Is) {
    const size_t stride = (size_t)T * N;
    const float G = sum_splits(part + (size_t)t * N + i, S, stride);
    const float U = sum_splits(part + (size_t)t * N + Is + i, S, stride);
    const float h = silu_f32(G) * U;
    const uint32_t hi = f32_to_bf16_rne(h);
    h_hi[(size_t)t * Is + i] = (uint16_t)hi;
    h_lo[(size_t)t * Is + i] = (uint16_t)f32_to_bf16_rne(h - bf16_to_f32(hi));
  }
  if (blockIdx.x == 0 && threadIdx.x == 0)
    gate_logit[t] = sum_splits(part + (size_t)t * N + 2 * Is, S, (size_t)T * N);
}

// out[t] = sum_s part[(s * T + t) * ld + col]   (the sigmoid-gate logit from
// the split-K partials of its row, summed in the order the top-k kernel uses)
// grid ceil(T/kFinThreads), block kFinThreads
__global__ void __launch_bounds__(kFinThreads) k_sum_column(const float* __restrict__ part, int S, int T,
                                                          int ld, int col, float* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.x * kFinThreads + threadIdx.x;
  if (t < T) out[t] = sum_splits(part + (size_t)t * ld + col, S, (size_t)T * ld);
}

// out[t, n] = bf16_rne( sum_s part[s, t, n] )   (latent down-projection;
// partial rows of ld floats)
// grid (ceil(N/kFinThreads), T), block kFinThreads
__global__ void __launch_bounds__(kFinThreads) k_round_bf16(const float* __restrict__ part, int S,
                                                          int T, int N, int ld,
                                                          uint16_t* __restrict__ out) {
  pdl_wait();
  pdl_trigger();
  const int t = blockIdx.y;
  const int n = blockIdx.x * kFinThreads + threadIdx.x;
  if (n >= N) return;
  const float v = sum_splits(part + (size_t)t * ld + n, S, (size_t)T * ld);
  out[(size_t)t * N + n] = (uint16_t)f32_to_bf16_rne(v);
}

}  // namespace moe
