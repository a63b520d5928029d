// MXFP4 GEMV on the CUDA cores for experts that received exactly one token
// (every expert of a 1-token decode step; most experts of small batches).
//
// With one token a tensor-core MMA would use 1 of its 8 columns, and the
// legacy mma.sync rate of sm_100 then caps the kernel near half the HBM
// bandwidth. Here every warp works alone on a contiguous range of weight rows:
//
// * the rows of all single-token experts form one list (gate/up: I row pairs
//   per expert; down: W rows per expert); warp w of the grid takes the w-th
//   equal share of it, so the load is balanced to one row and a warp reloads
//   its activation row only when its range crosses into another expert;
// * lane l owns the 32-element K blocks l, l+32, l+64, ... of the activation
//   row (BPL of them), kept in registers as f16;
// * the warp streams its rows through a private ring of shared-memory stages
//   filled by bulk TMA copies (cp.async.bulk of the packed codes and of the
//   covering 16-byte-aligned span of E8M0 codes) that lane 0 issues NST stages
//   ahead, completing on one mbarrier per stage;
// * per 32 weights a lane spends 16 cvt.rn.f16x2.e2m1x2 (exact decode) and
//   32 fma.rn.f32.f16 (exact f16 x f16 products, fp32 sums) and one fp32 FMA
//   for the block scale; a row's sum is a 5-step warp shuffle reduction;
// * no barrier couples the warps after the CTA has listed the experts.
//
// gate/up writes h = silu(g) * u in fp32 to h32; down reads h32 of the
// expert's token and converts it to f16 with one power-of-two scale per row
// (the largest |h| maps into [2^14, 2^15): relative rounding <= 2^-11).
// Every wait is bounded: on timeout the status word gets kStatusWaitTimeout
// and the warp stops waiting (its results are then undefined).
#include "common.cuh"
#include "kernels.h"

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

// E8M0 code -> fp32 scale for codes 1..254 (one shift); codes 0 and 255 go
// through e8m0_to_f32 (a stage holding either takes the exact path).
MOE_DEV float e8m0_fast(uint32_t c) { return __uint_as_float(c << 23); }

// true when any of the n bytes at p (16-byte aligned span) is 0x00 or 0xFF;
// every lane checks 16-byte pieces, the warp votes
MOE_DEV bool span_has_special(const uint8_t* p, int n, int lane) {
  bool any = false;
  for (int i = lane * 16; i < n; i += 32 * 16) {
    const uint4 v = *reinterpret_cast<const uint4*>(p + i);
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int k = 0; k < 4; ++k) any |= (__vcmpeq4(w[k], 0u) | __vcmpeq4(w[k], 0xFFFFFFFFu)) != 0u;
  }
  return __any_sync(0xFFFFFFFFu, any);
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
// block = kFmaWarps warps; grid sized so that every warp has work; dynamic
// shared memory = kFmaWarps * g.nst * (g.stage_bytes + 8)
// ---------------------------------------------------------------------------
template <int BPL, bool kGateUp>
__global__ void __launch_bounds__(32 * kFmaWarps, 3) k_fma_gemv(FmaArgs a, FmaGeometry g) {
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int16_t s_list[1024];      // single-token experts, ascending (E <= 1024)
  __shared__ int s_wsum[kFmaWarps];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = kGateUp ? a.W : a.I;
  const int KB = K >> 5;
  const size_t qrow = (size_t)K / 2, srow = (size_t)K / 32;
  const int N = kGateUp ? a.I : a.W;                      // rows of one matrix
  const size_t s_total = (size_t)a.E * N * srow;          // bytes of a stacked E8M0 array

  // 1) the single-token experts, in the order of the expert list
  const int n_act = __ldg(a.expert_list);
  int n_single = 0;
  for (int base = 0; base < n_act; base += 32 * kFmaWarps) {
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
    for (int w = 0; w < kFmaWarps; ++w) n_single += s_wsum[w];
    __syncthreads();
  }

  // 2) this warp's share of the units (gate/up: row pairs; down: rows)
  const int total = n_single * N;                        // < 2^27
  const int nwarps = gridDim.x * kFmaWarps;
  const int gw = blockIdx.x * kFmaWarps + warp;
  const int lo = (int)((long)total * gw / nwarps), hi = (int)((long)total * (gw + 1) / nwarps);
  if (lo >= hi) return;
  const int hi_si = hi / N, hi_r = hi - hi_si * N;       // end of the range as (expert, row)

  uint8_t* ring = smem + (size_t)warp * g.nst * g.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kFmaWarps * g.nst * g.stage_bytes) +
                   warp * g.nst;
  if (lane == 0) {
    for (int i = 0; i < g.nst; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // A cursor walks the stage sequence: gate/up -> for each row pair the gate
  // row, then the up row; down -> up to g.rps rows of one expert per stage.
  struct Cursor { int si, r, half; };
  auto rows_in_stage = [&](const Cursor& c) -> int {
    if (kGateUp) return 1;
    const int left = (c.si == hi_si) ? hi_r - c.r : N - c.r;
    return min(g.rps, left);
  };
  auto advance = [&](Cursor& c, int n) {
    if (kGateUp) {
      c.half ^= 1;
      if (c.half) return;
      n = 1;
    }
    c.r += n;
    if (c.r == N) { c.r = 0; ++c.si; }
  };
  auto done = [&](const Cursor& c) { return c.si > hi_si || (c.si == hi_si && c.r >= hi_r); };

  // producer (lane 0): stage copies, g.nst ahead of the consumer
  Cursor pc{lo / N, lo - (lo / N) * N, 0};
  int p_v = 0;
  auto issue_next = [&]() {
    if (done(pc)) return;
    const int n = rows_in_stage(pc);
    const int e = s_list[pc.si];
    const size_t row = (size_t)e * N + pc.r;
    const uint8_t* q = kGateUp ? (pc.half ? a.wu_q : a.wg_q) : a.wd_q;
    const uint8_t* sp = kGateUp ? (pc.half ? a.wu_s : a.wg_s) : a.wd_s;
    const size_t s0 = row * srow, s1 = (row + n) * srow;
    const size_t a0 = s0 & ~(size_t)15, a1 = min((s1 + 15) & ~(size_t)15, s_total);
    const int slot = p_v % g.nst;
    uint8_t* dst = ring + (size_t)slot * g.stage_bytes;
    const uint32_t cb = (uint32_t)(n * qrow);
    fence_proxy_async_smem();            // earlier generic reads of the slot come first
    mbar_expect_tx(&bars[slot], cb + (uint32_t)(a1 - a0));
    bulk_g2s(dst, q + row * qrow, cb, &bars[slot]);
    bulk_g2s(dst + g.sbuf_off, sp + a0, (uint32_t)(a1 - a0), &bars[slot]);
    ++p_v;
    advance(pc, n);
  };
  if (lane == 0)
    for (int i = 0; i < g.nst; ++i) issue_next();

  bool dead = false;
  int v = 0, slot = 0, phase = 0;
  int cur_si = -1, r0 = 0;
  uint32_t xr[BPL][16];
  float xs = 1.0f, gsum = 0.0f;
  Cursor c{lo / N, lo - (lo / N) * N, 0};
  while (!done(c)) {
    if (c.si != cur_si) {                 // new expert: load its activation row
      cur_si = c.si;
      const int e = s_list[c.si];
      r0 = __ldg(a.offsets + e);
      if (kGateUp) {
        const int tok = __ldg(a.row_token + r0);
        const __half* xrow = a.x16 + (size_t)tok * a.W;
#pragma unroll
        for (int j = 0; j < BPL; ++j) {
          const int b = lane + 32 * j;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            uint4 t = make_uint4(0u, 0u, 0u, 0u);
            if (b < KB) t = ldg16(xrow + b * 32 + 8 * q);
            xr[j][4 * q] = t.x; xr[j][4 * q + 1] = t.y; xr[j][4 * q + 2] = t.z; xr[j][4 * q + 3] = t.w;
          }
        }
        xs = __ldg(a.xscale + tok);
      } else {
        // h32 row -> f16 with one power-of-two scale for the row
        const float* hrow = a.h32 + (size_t)r0 * a.I;
        float m = 0.0f;
#pragma unroll
        for (int j = 0; j < BPL; ++j) {
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
        for (int j = 0; j < BPL; ++j) {
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
    const int n = rows_in_stage(c);
    if (!dead && !mbar_wait(&bars[slot], (uint32_t)phase)) {
      dead = true;
      if (lane == 0) atomicOr(a.status, kStatusWaitTimeout);
    }
    const uint8_t* stg = ring + (size_t)slot * g.stage_bytes;
    const int e = s_list[c.si];
    const uint32_t soff = (uint32_t)((((size_t)e * N + c.r) * srow) & 15);
    const uint8_t* ssc = stg + g.sbuf_off + soff;
    // the span copied with the stage is scanned once: codes 0 / 255 are rare
    const bool special = span_has_special(stg + g.sbuf_off, (int)((soff + n * srow + 15) & ~15u), lane);
    for (int rr = 0; rr < n; ++rr) {
      float acc = 0.0f;
#pragma unroll
      for (int j = 0; j < BPL; ++j) {
        const int b = lane + 32 * j;
        if (b < KB) {
          const uint4 w = *reinterpret_cast<const uint4*>(stg + rr * qrow + b * 16);
          const uint32_t code = ssc[rr * srow + b];
          acc = fmaf(dot_block(w, xr[j]), special ? e8m0_to_f32(code) : e8m0_fast(code), acc);
        }
      }
      const float sum = warp_sum(acc);
      if (kGateUp) {
        if (!c.half) gsum = sum;
        else if (lane == 0) a.h32[(size_t)r0 * a.I + c.r] = silu_f32(gsum * xs) * (sum * xs);
      } else if (lane == 0) {
        a.y_perm[(size_t)r0 * a.W + c.r + rr] = sum * xs;
      }
    }
    __syncwarp();
    ++v;
    if (++slot == g.nst) { slot = 0; phase ^= 1; }
    if (lane == 0 && !dead) issue_next();  // refill the slot just consumed
    advance(c, n);
  }
}

// Geometry for reduction length K (host side): rows per down stage rps (a
// power of two with about stage_target bytes of codes), stage buffer size
// (codes, then the E8M0 span with 32 bytes of alignment slack), ring depth
// nst from the shared-memory budget per CTA.
FmaGeometry fma_geometry(int K, bool gate_up, size_t smem_budget, size_t stage_target) {
  FmaGeometry g{};
  const size_t qrow = K / 2, srow = K / 32;
  int rps = 1;
  if (!gate_up)
    while (rps < 32 && (size_t)(2 * rps) * qrow <= stage_target) rps *= 2;
  g.rps = rps;
  g.sbuf_off = (uint32_t)((rps * qrow + 15) / 16 * 16);
  g.stage_bytes = (uint32_t)((g.sbuf_off + rps * srow + 32 + 127) / 128 * 128);
  const size_t per_warp = smem_budget / kFmaWarps;
  int nst = (int)(per_warp / (g.stage_bytes + 8));
  if (nst < 2) return g;
  g.nst = nst > 8 ? 8 : nst;
  g.smem_bytes = (uint32_t)(kFmaWarps * g.nst * (g.stage_bytes + 8));
  g.ok = 1;
  return g;
}

#define MOE_FMA_INST(BPL)                                                   \
  template __global__ void k_fma_gemv<BPL, true>(FmaArgs, FmaGeometry);    \
  template __global__ void k_fma_gemv<BPL, false>(FmaArgs, FmaGeometry);
MOE_FMA_INST(1)
MOE_FMA_INST(2)
MOE_FMA_INST(4)
MOE_FMA_INST(8)
#undef MOE_FMA_INST

}  // namespace moe
