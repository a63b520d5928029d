// Router tail: softmax top-k with renormalised weights (rabbit README, model
// table row "MoE routing": a softmax router keeping 10 of 512 experts), and the two other routers
// the same table names: "noaux_tc sigmoid" (GLM-5.2; read as sigmoid scores,
// a per-expert bias that steers the selection only, weights renormalised over
// the unbiased scores and scaled) and "grouped routing" (Kimi Linear; read as
// group-limited selection: the experts' groups ranked by the sum of their two
// best scores, top-k inside the best groups).
//
// One CTA per token, one thread per expert. The router logits arrive as
// split-K partial sums [S, T, E] from the router GEMM and are summed in a
// fixed order (s = 0..S-1),
// so the logits, and with them the selection, are reproducible run to run.
// Selection ranks by fp32 logit (the softmax is monotone); equal logits go to
// the lower expert index. Weights: w_j = exp(l_j - l_max) / sum_sel exp(l - l_max),
// which equals the full softmax renormalised over the selected experts.
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

// grid T, block kTopkThreads (one thread per expert, E <= 1024):
// 1) thread e sums the S partial logits of expert e in a fixed order (and
//    thread E the sigmoid-gate row's, when it rides along);
// 2) the k-th largest logit is found by a bitwise search over order-preserving
//    32-bit keys (one CTA-wide count per bit);
// 3) the experts above it are taken, then experts equal to it by ascending
//    index until k are taken;
// 4) warp 0 orders the k by descending logit, equal logits by ascending index,
//    and computes the renormalised weights;
// with f.x set (one token): step 3 also writes the dispatch (expert e's row =
// its rank among the selected by index, as k_permute places a lone token's
// pairs) and step 4 the slot <-> row maps, while warps 1..31 write the f16
// activation row with its power-of-two scale (the arithmetic of
// k_act_to_f16).
__global__ void __launch_bounds__(kTopkThreads) k_topk(const float* __restrict__ part, int S, int T,
                                                     int E, int ld, int k, int32_t* __restrict__ idx,
                                                     float* __restrict__ w,
                                                     float* __restrict__ logits,
                                                     float* __restrict__ gate_logit, TopkFuse f,
                                                     RouteCfg rc) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_cnt[kTopkThreads / 32];
  __shared__ uint32_t s_key[32];
  __shared__ int s_exp[32];
  __shared__ float s_val[32];
  const int tok = blockIdx.x;
  const int e = threadIdx.x, lane = e & 31, warp = e >> 5;
  const bool live = e < E;
  float acc = 0.0f;
  if (live) {
    acc = sum_splits(part + (size_t)tok * ld + e, S, (size_t)T * ld);
    if (logits) logits[(size_t)tok * E + e] = acc;
  }
  if (gate_logit && e == E) gate_logit[tok] = sum_splits(part + (size_t)tok * ld + E, S, (size_t)T * ld);
  // a NaN logit never wins; -0 ranks equal to +0
  const bool finite_in = live && !isnan(acc);
  const float v = finite_in ? (acc == 0.0f ? 0.0f : acc) : -INFINITY;
  // selection score (`choice`) and the value the weights use (`wval`):
  // softmax: the logit for both; sigmoid: s + bias and s
  float choice = v, wval = v;
  if (rc.score_fn == 1) {
    const float sg = finite_in ? 1.0f / (1.0f + expf(-acc)) : 0.0f;
    float c = finite_in ? sg + (rc.bias ? rc.bias[e] : 0.0f) : -INFINITY;
    if (isnan(c)) c = -INFINITY;
    choice = c == 0.0f ? 0.0f : c;
    wval = sg;
  }
  bool elig = live;
  if (rc.n_group > 1) {
    // group scores: the sum of the two largest expert scores of each group
    // (the softmax probability up to its common denominator, exp(l - l_max),
    // or the biased sigmoid score); then the rank of this expert's group
    __shared__ float s_gv[kTopkThreads];
    __shared__ float s_red[kTopkThreads / 32];
    __shared__ float s_gscore[kMaxGroups];
    float gv = choice;
    if (rc.score_fn == 0) {
      float m = v;
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      if (lane == 0) s_red[warp] = m;
      __syncthreads();
      m = s_red[0];
      for (int w2 = 1; w2 < kTopkThreads / 32; ++w2) m = fmaxf(m, s_red[w2]);
      gv = finite_in ? expf(v - m) : 0.0f;
    }
    s_gv[e] = live ? gv : -INFINITY;
    __syncthreads();
    const int gsize = E / rc.n_group;
    for (int g = warp; g < rc.n_group; g += kTopkThreads / 32) {
      float m1 = -INFINITY, m2 = -INFINITY;
      for (int i = lane; i < gsize; i += 32) {
        const float x = s_gv[g * gsize + i];
        if (x > m1) { m2 = m1; m1 = x; } else if (x > m2) { m2 = x; }
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) {
        const float o1 = __shfl_xor_sync(0xFFFFFFFFu, m1, off);
        const float o2 = __shfl_xor_sync(0xFFFFFFFFu, m2, off);
        m2 = fmaxf(fminf(m1, o1), fmaxf(m2, o2));
        m1 = fmaxf(m1, o1);
      }
      if (lane == 0) s_gscore[g] = gsize > 1 ? m1 + m2 : m1;
    }
    __syncthreads();
    if (live) {
      const int g = e / gsize;
      const float sg = s_gscore[g];
      int grank = 0;
      for (int j = 0; j < rc.n_group; ++j) {
        const float sj = s_gscore[j];
        grank += (sj > sg || (sj == sg && j < g)) ? 1 : 0;
      }
      elig = grank < rc.topk_group;
    }
  }
  const uint32_t u = __float_as_uint(choice);
  const uint32_t key = (u & 0x80000000u) ? ~u : (u | 0x80000000u);

  // largest thr with #{key >= thr} >= k among the eligible: the k-th largest key
  uint32_t thr = 0;
  for (int b = 31; b >= 0; --b) {
    const uint32_t c = thr | (1u << b);
    if (__syncthreads_count(elig && key >= c) >= k) thr = c;
  }
  const bool gt = elig && key > thr, eq = elig && key == thr;
  const int n_gt = __syncthreads_count(gt);
  const uint32_t lt_mask = (1u << lane) - 1u;
  const unsigned eq_m = __ballot_sync(0xFFFFFFFFu, eq);
  if (lane == 0) s_cnt[warp] = __popc(eq_m);
  __syncthreads();
  int before = __popc(eq_m & lt_mask);
  for (int w2 = 0; w2 < warp; ++w2) before += s_cnt[w2];
  const bool sel = gt || (eq && before < k - n_gt);
  const unsigned sel_m = __ballot_sync(0xFFFFFFFFu, sel);
  __syncthreads();
  if (lane == 0) s_cnt[warp] = __popc(sel_m);
  __syncthreads();
  int pos = __popc(sel_m & lt_mask);                     // selected experts below e
  for (int w2 = 0; w2 < warp; ++w2) pos += s_cnt[w2];
  if (sel) {
    s_key[pos] = key;
    s_exp[pos] = e;
    s_val[pos] = wval;
  }
  const bool fuse = f.x != nullptr;
  if (fuse) {
    if (live) {
      f.counts[e] = sel ? 1 : 0;
      f.offsets[e] = pos;
      if (sel) f.expert_list[1 + pos] = e;
    }
    if (e == 0) {
      f.offsets[E] = k;
      f.expert_list[0] = k;
    }
  }
  __syncthreads();
  if (warp != 0) {
    if (fuse && f.x16) {
      // the activation operand: the row's largest magnitude, then f16 with
      // the power-of-two scale that maps it into [2^14, 2^15)
      __shared__ float s_max[kTopkThreads / 32];
      const int tid = threadIdx.x - 32, nthr = kTopkThreads - 32;
      float m = 0.0f;
      for (int i = tid * 8; i < f.W; i += nthr * 8) {
        const uint4 xv = ldg16(f.x + i);
        const uint32_t wv[4] = {xv.x, xv.y, xv.z, xv.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16lo(wv[j])), fabsf(bf16hi(wv[j]))));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      if (lane == 0) s_max[warp] = m;
      asm volatile("bar.sync 1, %0;\n" ::"n"(kTopkThreads - 32) : "memory");
      m = s_max[1];
      for (int w2 = 2; w2 < kTopkThreads / 32; ++w2) m = fmaxf(m, s_max[w2]);
      float scale, inv;
      f16_block_scale(m, scale, inv, kF16OpTop);
      for (int i = tid * 8; i < f.W; i += nthr * 8) {
        const uint4 xv = ldg16(f.x + i);
        const uint32_t wv[4] = {xv.x, xv.y, xv.z, xv.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = __floats2half2_rn(bf16lo(wv[j]) * inv, bf16hi(wv[j]) * inv);
          o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(f.x16 + i) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      if (tid == 0) f.xscale[0] = scale;
    }
    return;
  }
  // lane i < k: its rank among the k taken (descending key, then ascending index)
  uint32_t ki = 0;
  int ei = 0;
  float vi = 0.0f;
  if (lane < k) { ki = s_key[lane]; ei = s_exp[lane]; vi = s_val[lane]; }
  int rank = 0;
  for (int j = 0; j < k; ++j) {
    const uint32_t kj = s_key[j];
    const int ej = s_exp[j];
    rank += (kj > ki || (kj == ki && ej < ei)) ? 1 : 0;
  }
  __syncwarp();
  if (fuse && lane < k) {          // row `lane` (ascending expert) holds slot `rank`
    f.row_token[lane] = 0;
    f.row_slot[lane] = rank;
    f.slot_row[rank] = lane;
  }
  if (lane < k) { s_exp[rank] = ei; s_val[rank] = vi; }
  __syncwarp();
  // lane r now holds the r-th selection
  const float selv = (lane < k) ? s_val[lane] : 0.0f;
  const int sele = (lane < k) ? s_exp[lane] : 0;
  // softmax: exp(l - l_top) over the selected (l_top = slot 0's logit, the
  // largest selected); sigmoid: the unbiased scores themselves
  const float m = __shfl_sync(0xFFFFFFFFu, selv, 0);
  const float ex = (lane < k) ? (rc.score_fn == 1 ? selv : expf(selv - m)) : 0.0f;
  float den = ex;
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) den += __shfl_xor_sync(0xFFFFFFFFu, den, off);
  if (lane < k) {
    idx[(size_t)tok * k + lane] = sele;
    w[(size_t)tok * k + lane] = ex / den * rc.scale;
  }
}

}  // namespace moe
