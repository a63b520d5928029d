// bf16 GEMV for a single token on the CUDA cores: the router logits and the
// sigmoid-gate logit (rabbit README, model table row "MoE routing"; "+ gated
// shared expert"), and the shared expert's SwiGLU and down projection.
//
// With one token a tensor-core MMA uses one column, and split-K across SMs
// cuts every weight row into short pieces read far apart. Here one CTA per SM
// streams a contiguous range of whole weight rows through a ring of shared
// memory stages filled by bulk TMA copies (contiguous multi-kilobyte reads),
// so no partial sums leave the CTA:
//
// * wpr = K / 2048 warps share a row (one for K <= 2048), so a stage holds
//   16 / wpr row slots of K bf16 each: plain -> consecutive rows of one
//   segment (up to three matrices stacked along the output); SwiGLU -> gate
//   rows i.. in the first half of the slots, up rows i.. in the second;
// * 16 consumer warps: warp w takes slot w / wpr over K part w % wpr; lane l
//   owns the 8-element chunks l, l+32, ... of that part, the activation
//   chunks kept in registers; products in fp32 (exact for bf16 x bf16),
//   sums in fp32, a 5-step shuffle reduction per warp; the parts of a row are
//   added in order through shared memory one stage later (after every warp
//   has released the stage), so no warp waits inside a stage;
// * plain writes out[s][row]; SwiGLU writes h[i] = silu(g_i) * u_i (fp32);
//   for the shared down projection of one token the plain mode can instead
//   finish the layer's combine for its rows (k <= 32 routed slots gathered
//   by lanes, summed by every lane in slot order).
// Every wait is bounded as in the other streaming kernels.
#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

MOE_DEV float warp_sum_rows(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}

// 8 bf16 weights (one 16-byte chunk) times 8 activations
MOE_DEV void dot8_bf16(const uint4& w, const uint4& x, float& a0, float& a1) {
  const uint32_t ww[4] = {w.x, w.y, w.z, w.w}, xx[4] = {x.x, x.y, x.z, x.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    a0 = fmaf(__uint_as_float(ww[i] << 16), __uint_as_float(xx[i] << 16), a0);
    a1 = fmaf(__uint_as_float(ww[i] & 0xFFFF0000u), __uint_as_float(xx[i] & 0xFFFF0000u), a1);
  }
}
MOE_DEV void dot8_f32(const uint4& w, const float4& xl, const float4& xh, float& a0, float& a1) {
  a0 = fmaf(__uint_as_float(w.x << 16), xl.x, a0);
  a1 = fmaf(__uint_as_float(w.x & 0xFFFF0000u), xl.y, a1);
  a0 = fmaf(__uint_as_float(w.y << 16), xl.z, a0);
  a1 = fmaf(__uint_as_float(w.y & 0xFFFF0000u), xl.w, a1);
  a0 = fmaf(__uint_as_float(w.z << 16), xh.x, a0);
  a1 = fmaf(__uint_as_float(w.z & 0xFFFF0000u), xh.y, a1);
  a0 = fmaf(__uint_as_float(w.w << 16), xh.z, a0);
  a1 = fmaf(__uint_as_float(w.w & 0xFFFF0000u), xh.w, a1);
}

}  // namespace

// block = 32 * (kRowsConsumers + 1) threads (warp 0: producer), one CTA per
// SM; dynamic shared memory = nst * rows_stage_bytes(K)
template <bool kSwiGLU, bool kXF32>
__global__ void __launch_bounds__(32 * (kRowsConsumers + 1), 1) k_rows_bf16(RowsArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int D = kRowsMaxStages + 2;      // depth of the partial-sum exchange
  __shared__ uint64_t s_bars[2 * kRowsMaxStages];
  __shared__ int s_abort;
  __shared__ float s_part[D][kRowsConsumers];   // [stage % D][row slot * wpr + part]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = a.K;
  const int wpr = rows_warps_per_row(K);              // warps sharing one row (K split)
  const int SL = kRowsConsumers / wpr;                // row slots per stage
  const uint32_t row_bytes = (uint32_t)K * 2;
  const uint32_t stage_bytes = (uint32_t)SL * row_bytes;
  const int nst = a.nst;
  // units: plain -> rows of the stacked segments; SwiGLU -> row pairs (gate i, up i)
  const int U0 = a.rows[0], U1 = kSwiGLU ? 0 : a.rows[1], U2 = kSwiGLU ? 0 : a.rows[2];
  const long total = (long)U0 + U1 + U2;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;                                   // uniform across the CTA
  const int P = kSwiGLU ? SL / 2 : SL;                    // units per stage
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kRowsMaxStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kRowsConsumers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  // the cursor (segment, row in it) of unit lo; a stage takes at most P
  // units, never past the segment's end or the range's
  auto seg_units = [&](int s) { return s == 0 ? U0 : s == 1 ? U1 : U2; };
  int seg0 = 0;
  long r_lo = lo;
  while (seg0 < 2 && r_lo >= seg_units(seg0)) {
    r_lo -= seg_units(seg0);
    ++seg0;
  }

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      uint32_t last_ph[kRowsMaxStages];
      bool filled[kRowsMaxStages];
#pragma unroll
      for (int s = 0; s < kRowsMaxStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      int seg = seg0, slot = 0;
      int r = (int)r_lo;
      uint32_t ph = 0;
      for (long u = lo; u < hi;) {
        const int n = (int)min((long)min(P, seg_units(seg) - r), hi - u);
        if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) break;
        uint8_t* st = smem + (size_t)slot * stage_bytes;
        fence_proxy_async_smem();            // the consumers' reads of the slot come first
        const uint32_t cb = n * row_bytes;
        if (kSwiGLU) {                       // gate rows in slots 0.., up rows in slots SL/2..
          mbar_expect_tx(&full[slot], 2 * cb);
          bulk_g2s(st, a.w[0] + (size_t)r * K, cb, &full[slot]);
          bulk_g2s(st + (SL / 2) * row_bytes, a.w[1] + (size_t)r * K, cb, &full[slot]);
        } else {
          mbar_expect_tx(&full[slot], cb);
          bulk_g2s(st, a.w[seg] + (size_t)r * K, cb, &full[slot]);
        }
        last_ph[slot] = ph;
        filled[slot] = true;
        u += n;
        r += n;
        while (seg < 2 && r == seg_units(seg)) { r = 0; ++seg; }   // skips empty segments
        if (++slot == nst) { slot = 0; ph ^= 1u; }
      }
      if (*abort) {     // let every issued copy land before the CTA can exit
        for (int s = 0; s < nst; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int rs = w / wpr, part = w - rs * wpr;         // row slot, K part
    const int Kw = K / wpr;                              // elements per warp
    const int nch = Kw / 256;                            // 8-element chunks per lane
    const int q0 = part * Kw;                            // first element of the part
    // this lane's activations: elements q0 + (j * 32 + lane) * 8 .. + 7
    uint4 xb[kRowsMaxChunks];
    float4 xf[kRowsMaxChunks][2];
#pragma unroll
    for (int j = 0; j < kRowsMaxChunks; ++j) {
      if (j < nch) {
        const int el = q0 + (j * 32 + lane) * 8;
        if (kXF32) {
          const float4* xp = reinterpret_cast<const float4*>(static_cast<const float*>(a.x) + el);
          xf[j][0] = __ldg(xp);
          xf[j][1] = __ldg(xp + 1);
        } else {
          xb[j] = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x) + el));
        }
      }
    }
    // outputs of a stage are written one stage later, by warp i for unit i,
    // once every warp has arrived on the stage's empty barrier (so its
    // partial sums are in s_part): nobody waits in the middle of a stage
    const bool direct = !kSwiGLU && wpr == 1;            // the warp's sum is the output
    int seg = seg0, slot = 0, k = 0;
    int r = (int)r_lo;
    uint32_t ph = 0;
    int pn = 0, pr = 0, pseg = 0, pslot = 0;             // the previous stage
    uint32_t pph = 0;
    auto emit = [&](int kk) {                            // outputs of stage kk (lane 0 of warp w < pn)
      const float* sp = s_part[kk % D];
      if (kSwiGLU) {
        float g = 0.0f, uu = 0.0f;
        for (int i = 0; i < wpr; ++i) g += sp[w * wpr + i];
        for (int i = 0; i < wpr; ++i) uu += sp[(SL / 2 + w) * wpr + i];
        a.out[0][pr + w] = silu_f32(g) * uu;
      } else {
        float g = 0.0f;
        for (int i = 0; i < wpr; ++i) g += sp[w * wpr + i];
        a.out[pseg][pr + w] = g;
      }
    };
    bool ok = true;
    for (long u = lo; u < hi; ++k) {
      const int n = (int)min((long)min(P, seg_units(seg) - r), hi - u);
      if (!tc::wait_or_abort(&full[slot], ph, abort)) { ok = false; break; }
      // slots in use: plain -> 0..n-1; SwiGLU -> gate 0..n-1, up SL/2..SL/2+n-1
      const bool active = kSwiGLU ? ((rs % (SL / 2)) < n) : (rs < n);
      if (active) {
        const uint32_t base = smem_u32(smem + (size_t)slot * stage_bytes) + rs * row_bytes + q0 * 2;
        float a0 = 0.0f, a1 = 0.0f;
#pragma unroll
        for (int j = 0; j < kRowsMaxChunks; ++j) {
          if (j < nch) {
            const uint4 wv = lds16(base + (uint32_t)(j * 32 + lane) * 16u);
            if (kXF32) dot8_f32(wv, xf[j][0], xf[j][1], a0, a1);
            else dot8_bf16(wv, xb[j], a0, a1);
          }
        }
        const float sum = warp_sum_rows(a0 + a1);
        if (direct && a.y) {
          // the layer's combine for this output row, in the combine's own
          // order: routed slots j = 0.. (fma), then the gated shared term
          const int row = r + rs;
          float v = 0.0f, wj = 0.0f;
          if (lane < a.k) {
            v = __ldg(a.y_perm + (size_t)__ldg(a.slot_row + lane) * a.rows[0] + row);
            wj = __ldg(a.topk_w + lane);
          }
          float acc = 0.0f;
          for (int j = 0; j < a.k; ++j)
            acc = fmaf(__shfl_sync(0xFFFFFFFFu, wj, j), __shfl_sync(0xFFFFFFFFu, v, j), acc);
          acc = fmaf(sigmoid_f32(__ldg(a.gate_logit)), sum, acc);
          if (lane == 0) a.y[row] = acc;
        } else if (lane == 0) {
          if (direct) a.out[seg][r + rs] = sum;
          else s_part[k % D][w] = sum;
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[slot]);   // this warp is done with the slot
      if (!direct && k > 0 && w < pn) {
        if (!tc::wait_or_abort(&empty[pslot], pph, abort)) { ok = false; break; }
        if (lane == 0) emit(k - 1);
      }
      pn = n; pr = r; pseg = seg; pslot = slot; pph = ph;
      u += n;
      r += n;
      while (seg < 2 && r == seg_units(seg)) { r = 0; ++seg; }
      if (++slot == nst) { slot = 0; ph ^= 1u; }
    }
    if (ok && !direct && k > 0 && w < pn && tc::wait_or_abort(&empty[pslot], pph, abort) && lane == 0)
      emit(k - 1);
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
}

template __global__ void k_rows_bf16<false, false>(RowsArgs);
template __global__ void k_rows_bf16<true, false>(RowsArgs);
template __global__ void k_rows_bf16<false, true>(RowsArgs);

// stages of the ring for reduction length K within the shared-memory budget
int rows_stages(int K, size_t smem_budget) {
  const size_t sb = rows_stage_bytes(K);
  const size_t n = smem_budget / sb;
  return n < 2 ? 0 : (int)(n > kRowsMaxStages ? kRowsMaxStages : n);
}

}  // namespace moe
