// MXFP4 GEMV on the CUDA cores for experts that received exactly one token
// (every expert of a 1-token decode step; most experts of small batches).
//
// With one token a tensor-core MMA would use 1 of its 8 columns, and the
// legacy mma.sync rate of sm_100 then caps the kernel near half the HBM
// bandwidth. Here one CTA per SM streams a contiguous share of the weight rows
// of all single-token experts through a ring of shared-memory stages:
//
// * the rows of all single-token experts form one list (gate/up: I row pairs
//   per expert; down: W rows per expert); CTA c takes the c-th equal share;
// * a producer warp fills each stage with a few large bulk TMA copies
//   (cp.async.bulk): gate/up -> kFmaConsumers/2 gate rows and the same up rows,
//   down -> kFmaConsumers * RPS rows, each with the covering 16-byte-aligned
//   span of E8M0 codes; a stage never crosses an expert, so every stage has
//   one activation row;
// * kFmaConsumers consumer warps share each stage: gate/up -> warps 2p and
//   2p+1 take row pair p, each over one half of K, and add their partial
//   sums in shared memory; down -> warp w takes rows RPS*w .. RPS*w+RPS-1;
//   lane l owns the 32-element K blocks l, l+32, ... of its warp's K range of
//   the activation row, kept in registers as f16;
// * per 32 weights a lane spends 16 cvt.rn.f16x2.e2m1x2 (exact decode), 32
//   fma.rn.f32.f16 (exact f16 x f16 products, fp32 sums) and one fp32 FMA for
//   the block scale (E8M0 decoded without a branch, codes 0 and 255 included);
//   the rows of a warp are computed interleaved for independent FMA chains;
//   a row's sum is a 5-step warp shuffle reduction.
//
// gate/up writes h = silu(g) * u in fp32 to h32; down reads h32 of the
// expert's token and converts it to f16 with one power-of-two scale per row
// (the largest |h| maps into [2^14, 2^15): relative rounding <= 2^-11).
// Every wait is bounded: on a timeout the CTA raises an abort flag, the
// status word gets kStatusWaitTimeout and every role stops (the results are
// then undefined); copies in flight land before the CTA exits.
#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

// Dot product of one 32-element MXFP4 block with 32 f16 activations (block
// scale not applied).
MOE_DEV float dot_block(uint4 w, const uint32_t (&x)[16]) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  float a0 = 0.f, a1 = 0.f;
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4];
    e2m1x8_to_f16x8(words[q], h);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a0 = fma_f16lo(h[j], x[4 * q + j], a0);
      a1 = fma_f16hi(h[j], x[4 * q + j], a1);
    }
  }
  return a0 + a1;
}

// E8M0 code -> fp32 without a branch: 2^(c-127) for c = 1..254, the
// subnormal 2^-127 for c = 0, NaN for c = 255 (0x7F800000 | 0x400000).
MOE_DEV float e8m0_exact(uint32_t c) {
  const uint32_t special = (c - 1u) > 253u ? 0x00400000u : 0u;
  return __uint_as_float((c << 23) | special);
}

MOE_DEV float warp_sum(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, off);
  return v;
}
MOE_DEV float warp_max(float v) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  return v;
}

}  // namespace

// ---------------------------------------------------------------------------
// block = 32 * (kFmaConsumers + 1) threads (warp 0: producer); one CTA per SM;
// dynamic shared memory = g.nst * g.stage_bytes
// ---------------------------------------------------------------------------
template <int BPL, bool kGateUp, int RPS>
__global__ void __launch_bounds__(32 * (kFmaConsumers + 1), 1) k_fma_gemv(FmaArgs a, FmaGeometry g) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int16_t s_list[1024];      // single-token experts, ascending (E <= 1024)
  __shared__ int s_wsum[kFmaConsumers + 1];
  __shared__ uint64_t s_bars[2 * kFmaMaxStages];
  __shared__ int s_abort;
  __shared__ float2 s_part[2][kFmaConsumers / 2][2];   // gate/up partial sums [stage&1][pair][half]
  constexpr int kWarps = kFmaConsumers + 1;
  constexpr int P = kGateUp ? kFmaConsumers / 2 : kFmaConsumers * RPS;   // units per stage
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = kGateUp ? a.W : a.I;
  const int KB = K >> 5;
  const uint32_t qrow = (uint32_t)K / 2, srow = (uint32_t)K / 32;
  const int N = kGateUp ? a.I : a.W;                      // rows of one matrix
  const size_t s_total = (size_t)a.E * N * srow;          // bytes of a stacked E8M0 array

  // 1) the single-token experts, in the order of the expert list
  const int n_act = __ldg(a.expert_list);
  int n_single = 0;
  for (int base = 0; base < n_act; base += 32 * kWarps) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < n_act) {
      e = __ldg(a.expert_list + 1 + i);
      if (__ldg(a.offsets + e + 1) - __ldg(a.offsets + e) != 1) e = -1;
    }
    const unsigned m = __ballot_sync(0xFFFFFFFFu, e >= 0);
    if (lane == 0) s_wsum[warp] = __popc(m);
    __syncthreads();
    int before = n_single;
    for (int w = 0; w < warp; ++w) before += s_wsum[w];
    if (e >= 0) s_list[before + __popc(m & ((1u << lane) - 1u))] = (int16_t)e;
    for (int w = 0; w < kWarps; ++w) n_single += s_wsum[w];
    __syncthreads();
  }

  // 2) this CTA's share of the units (gate/up: row pairs; down: rows)
  const long total = (long)n_single * N;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;                                   // uniform across the CTA
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kFmaMaxStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < g.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFmaConsumers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  // a stage takes at most P units, never crossing an expert or the range end;
  // both roles walk the stages with the same incremental cursor (expert slot
  // si, row r within it, ring slot and phase): no division per stage
  const int si0 = (int)(lo / N), r_lo = (int)(lo - (long)si0 * N);
  auto stage_units = [&](long u, int r) -> int { return (int)min((long)min(P, N - r), hi - u); };

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      uint32_t last_ph[kFmaMaxStages];
      bool filled[kFmaMaxStages];
#pragma unroll
      for (int s = 0; s < kFmaMaxStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      int si = si0, r = r_lo, slot = 0;
      uint32_t ph = 0;
      for (long u = lo; u < hi;) {
        const int n = stage_units(u, r);
        if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) break;
        const size_t row = (size_t)s_list[si] * N + r;
        const uint32_t cb = n * qrow;
        const size_t s0 = row * srow, s1 = (row + n) * srow;
        const size_t a0 = s0 & ~(size_t)15, a1 = min((s1 + 15) & ~(size_t)15, s_total);
        const uint32_t sb = (uint32_t)(a1 - a0);
        uint8_t* st = smem + (size_t)slot * g.stage_bytes;
        fence_proxy_async_smem();            // the consumers' reads of the slot come first
        if (kGateUp) {
          mbar_expect_tx(&full[slot], 2 * cb + 2 * sb);
          bulk_g2s(st, a.wg_q + row * qrow, cb, &full[slot]);
          bulk_g2s(st + g.code_bytes, a.wu_q + row * qrow, cb, &full[slot]);
          bulk_g2s(st + g.sbuf_off, a.wg_s + a0, sb, &full[slot]);
          bulk_g2s(st + g.sbuf2_off, a.wu_s + a0, sb, &full[slot]);
        } else {
          mbar_expect_tx(&full[slot], cb + sb);
          bulk_g2s(st, a.wd_q + row * qrow, cb, &full[slot]);
          bulk_g2s(st + g.sbuf_off, a.wd_s + a0, sb, &full[slot]);
        }
        last_ph[slot] = ph;
        filled[slot] = true;
        u += n;
        r += n;
        if (r == N) { r = 0; ++si; }
        if (++slot == g.nst) { slot = 0; ph ^= 1u; }
      }
      if (*abort) {     // let every issued copy land before the CTA can exit
        for (int s = 0; s < g.nst; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    // gate/up: warps 2p and 2p+1 share row pair p of a stage, each over one
    // half of K (half the activation registers), and combine their partial
    // sums through shared memory; down: warp w takes rows RPS*w ... of a stage
    const int w = warp - 1;
    constexpr int BW = kGateUp ? (BPL + 1) / 2 : BPL;    // blocks per lane of this warp
    const int half = kGateUp ? (w & 1) : 0;
    const int KBw = kGateUp ? KB / 2 : KB;                // blocks of this warp's K range
    const int kb0 = half * KBw;                           // its first block
    uint32_t xr[BW][16];
    float xs = 1.0f;
    int cur_e = -1, r0 = 0;
    int si = si0, r = r_lo, slot = 0, k = 0;
    uint32_t ph = 0;
    for (long u = lo; u < hi; ++k) {
      const int n = stage_units(u, r);
      const int e = s_list[si];
      if (e != cur_e) {                     // new expert: load its activation row
        cur_e = e;
        r0 = __ldg(a.offsets + e);
        if (kGateUp) {
          const int tok = __ldg(a.row_token + r0);
          const __half* xrow = a.x16 + (size_t)tok * a.W;
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            const int b = lane + 32 * j;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              uint4 t = make_uint4(0u, 0u, 0u, 0u);
              if (b < KBw) t = ldg16(xrow + (kb0 + b) * 32 + 8 * q);
              xr[j][4 * q] = t.x; xr[j][4 * q + 1] = t.y; xr[j][4 * q + 2] = t.z; xr[j][4 * q + 3] = t.w;
            }
          }
          xs = __ldg(a.xscale + tok);
        } else {
          // h32 row -> f16 with one power-of-two scale for the row
          const float* hrow = a.h32 + (size_t)r0 * a.I;
          float m = 0.0f;
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            const int b = lane + 32 * j;
            if (b < KB)
              for (int q = 0; q < 8; ++q) {
                const float4 t = __ldg(reinterpret_cast<const float4*>(hrow + b * 32) + q);
                m = fmaxf(m, fmaxf(fmaxf(fabsf(t.x), fabsf(t.y)), fmaxf(fabsf(t.z), fabsf(t.w))));
              }
          }
          m = warp_max(m);
          float inv = 1.0f;
          xs = 1.0f;
          if (m > 0.0f && isfinite(m)) {
            int ex;
            frexpf(m, &ex);
            ex = max(-100, min(127, ex));
            xs = ldexpf(1.0f, ex - 15);
            inv = ldexpf(1.0f, 15 - ex);
          }
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            const int b = lane + 32 * j;
#pragma unroll
            for (int q = 0; q < 8; ++q) {
              float4 t = make_float4(0.f, 0.f, 0.f, 0.f);
              if (b < KB) t = __ldg(reinterpret_cast<const float4*>(hrow + b * 32) + q);
              const __half2 l2 = __floats2half2_rn(t.x * inv, t.y * inv);
              const __half2 h2 = __floats2half2_rn(t.z * inv, t.w * inv);
              xr[j][2 * q] = *reinterpret_cast<const uint32_t*>(&l2);
              xr[j][2 * q + 1] = *reinterpret_cast<const uint32_t*>(&h2);
            }
          }
        }
      }
      if (!tc::wait_or_abort(&full[slot], ph, abort)) break;
      const uint32_t st = smem_u32(smem + (size_t)slot * g.stage_bytes);
      const uint32_t soff = (uint32_t)((((size_t)e * N + r) * srow) & 15u);
      // rows of this warp: gate/up -> row 0 = gate, row 1 = up of pair w/2;
      // down -> rows RPS*w ... (codes qrow apart, scales srow apart)
      constexpr int NR = kGateUp ? 2 : RPS;
      const int u0 = kGateUp ? (w >> 1) : RPS * w;
      float acc[NR];
#pragma unroll
      for (int rr = 0; rr < NR; ++rr) acc[rr] = 0.0f;
      if (u0 < n) {
        uint32_t cb[NR], sbs[NR];
#pragma unroll
        for (int rr = 0; rr < NR; ++rr) {
          if (kGateUp) {
            cb[rr] = st + rr * g.code_bytes + u0 * qrow + 16u * (kb0 + lane);
            sbs[rr] = st + (rr ? g.sbuf2_off : g.sbuf_off) + soff + u0 * srow + kb0 + lane;
          } else {
            cb[rr] = st + (u0 + rr) * qrow + 16u * lane;
            sbs[rr] = st + g.sbuf_off + soff + (u0 + rr) * srow + lane;
          }
        }
#pragma unroll
        for (int j = 0; j < BW; ++j) {
          if (lane + 32 * j < KBw) {
#pragma unroll
            for (int rr = 0; rr < NR; ++rr) {
              if (kGateUp || u0 + rr < n) {
                const uint4 wv = lds16(cb[rr] + 512u * j);
                const uint32_t code = lds8(sbs[rr] + 32u * j);
                acc[rr] = fmaf(dot_block(wv, xr[j]), e8m0_exact(code), acc[rr]);
              }
            }
          }
        }
        if (kGateUp) {
          const float gs = warp_sum(acc[0]), us = warp_sum(acc[1]);
          float2* part = s_part[k & 1][u0];
          if (lane == 0) part[half] = make_float2(gs, us);
          asm volatile("bar.sync %0, 64;\n" ::"r"(1 + u0) : "memory");   // the two warps of the pair
          if (half == 0 && lane == 0) {
            const float2 o = part[1];
            a.h32[(size_t)r0 * a.I + r + u0] = silu_f32((gs + o.x) * xs) * ((us + o.y) * xs);
          }
        } else {
#pragma unroll
          for (int rr = 0; rr < NR; ++rr) {
            if (u0 + rr < n) {
              const float sum = warp_sum(acc[rr]);
              if (lane == 0) a.y_perm[(size_t)r0 * a.W + r + u0 + rr] = sum * xs;
            }
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(&empty[slot]);   // this warp is done with the slot
      u += n;
      r += n;
      if (r == N) { r = 0; ++si; }
      if (++slot == g.nst) { slot = 0; ph ^= 1u; }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
}

// Geometry for reduction length K (host side): rows per consumer warp in a
// down stage rps = max(1, 8 / BPL); a stage holds kFmaConsumers / 2 row pairs
// (gate/up: the gate rows, then the up rows, then the two E8M0 spans) or
// kFmaConsumers * rps rows (down: codes, then their span); every span with 32
// bytes of alignment slack; ring depth nst from the shared-memory budget.
FmaGeometry fma_geometry(int K, bool gate_up, size_t smem_budget) {
  FmaGeometry g{};
  const size_t qrow = K / 2, srow = K / 32;
  const int bpl = (K + 1023) / 1024;
  if (bpl > 8) return g;
  const int rps = gate_up ? 1 : (bpl > 4 ? 1 : bpl > 2 ? 2 : bpl > 1 ? 4 : 8);
  const int units = gate_up ? kFmaConsumers / 2 : kFmaConsumers * rps;
  g.rps = rps;
  g.units = units;
  g.code_bytes = (uint32_t)((units * qrow + 127) / 128 * 128);
  const uint32_t code_all = gate_up ? 2 * g.code_bytes : g.code_bytes;
  const uint32_t span = (uint32_t)((units * srow + 32 + 127) / 128 * 128);
  g.sbuf_off = code_all;
  g.sbuf2_off = code_all + span;
  g.stage_bytes = code_all + (gate_up ? 2 : 1) * span;
  int nst = (int)(smem_budget / g.stage_bytes);
  if (nst < 2) return g;
  g.nst = nst > kFmaMaxStages ? kFmaMaxStages : nst;
  g.smem_bytes = (uint32_t)(g.nst * g.stage_bytes);
  g.ok = 1;
  return g;
}

#define MOE_FMA_INST(BPL, RPS)                                                 \
  template __global__ void k_fma_gemv<BPL, true, 1>(FmaArgs, FmaGeometry);    \
  template __global__ void k_fma_gemv<BPL, false, RPS>(FmaArgs, FmaGeometry);
MOE_FMA_INST(1, 8)
MOE_FMA_INST(2, 4)
MOE_FMA_INST(4, 2)
MOE_FMA_INST(8, 1)
#undef MOE_FMA_INST

}  // namespace moe
