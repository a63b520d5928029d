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
// dynamic shared memory = g.smem_bytes (the ring, then the activation buffer
// at g.act_off).
// gate/up: waits for the previous kernel (griddepcontrol.wait) before it
// reads anything (for one token the previous kernel is the top-k launch,
// which writes the dispatch this kernel starts from: expert list, offsets,
// row maps) and only then lets its dependants launch, so that when the down
// projection starts, the dispatch is complete.
// down: reads the dispatch and streams its first weight stages at once (they
// land while the gate/up grid's last CTAs finish); it waits for the previous
// kernel only before it copies the expert's h row, the gate/up output.
// ---------------------------------------------------------------------------
template <int BPL, bool kGateUp, int RPS>
__global__ void __launch_bounds__(32 * (kFmaConsumers + 1), 1) k_fma_gemv(FmaArgs a, FmaGeometry g) {
  if (kGateUp) pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int16_t s_list[1024];      // single-token experts, ascending (E <= 1024)
  __shared__ int s_wsum[kFmaConsumers + 1];
  __shared__ uint64_t s_bars[2 * kFmaMaxStages];
  __shared__ uint64_t s_act[3];         // activation buffer: [0] full, [1] empty, [2] down: h converted
  __shared__ int s_abort;
  __shared__ float2 s_part[2][kFmaConsumers / 2][2];   // gate/up partial sums [stage&1][pair][half]
  constexpr int kWarps = kFmaConsumers + 1;
  // gate/up with K > 2048: two warps per row pair, each over half of K; with
  // shorter rows one warp per pair (twice the pairs per stage, no exchange)
  constexpr bool kSplit = kGateUp && BPL > 2;
  constexpr int P = kGateUp ? (kSplit ? kFmaConsumers / 2 : kFmaConsumers) : kFmaConsumers * RPS;   // units per stage
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = kGateUp ? a.W : a.I;
  const int KB = K >> 5;
  const uint32_t qrow = (uint32_t)K / 2, srow = (uint32_t)K / 32;
  const int N = kGateUp ? a.I : a.W;                      // rows of one matrix
  const size_t s_total = (size_t)a.E * N * srow;          // bytes of a stacked E8M0 array
  uint8_t* act = smem + g.act_off;

  // 1) the single-token experts, in the order of the expert list (the
  //    dispatch's output, complete once the wait above returned; read through L2)
  const int n_act = __ldcg(a.expert_list);
  int n_single = 0;
  for (int base = 0; base < n_act; base += 32 * kWarps) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < n_act) {
      e = __ldcg(a.expert_list + 1 + i);
      if (__ldcg(a.offsets + e + 1) - __ldcg(a.offsets + e) != 1) e = -1;
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
  if (lo >= hi) {                                         // uniform across the CTA
    // no work; the grid must still not complete before the previous one (the
    // next kernel's wait covers this grid only)
    if (!kGateUp) pdl_wait();
    return;
  }
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kFmaMaxStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < g.nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kFmaConsumers);
    }
    mbar_init(&s_act[0], 1);
    mbar_init(&s_act[1], kFmaConsumers);
    mbar_init(&s_act[2], 1);
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
  // the activation row of expert slot si: gate/up -> its token's f16 row
  // (key = token), down -> the expert's h row (key = slot)
  auto act_key = [&](int si) -> int {
    return kGateUp ? __ldcg(a.row_token + __ldcg(a.offsets + s_list[si])) : si;
  };

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      uint32_t last_ph[kFmaMaxStages];
      bool filled[kFmaMaxStages];
#pragma unroll
      for (int s = 0; s < kFmaMaxStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      int si = si0, r = r_lo, slot = 0, k = 0;
      uint32_t ph = 0;
      // activation rows: the slots whose row is still to be copied, in order
      // (at most 4 deferred)
      int pend[4], n_pend = 0, n_loaded = 0, cur_key = -1, cur_si = -1;
      bool fenced = false, ok = true, waited = kGateUp;
      auto load_acts = [&]() -> bool {        // copy the pending rows
        if (!fenced) {
          if (!waited) {
            pdl_wait();                       // down: the gate/up grid's h rows
            waited = true;
          }
          asm volatile("fence.proxy.async;\n" ::: "memory");   // the previous grid's writes, then bulk reads
          fenced = true;
        }
        for (int i = 0; i < n_pend; ++i) {
          if (n_loaded > 0 && !tc::wait_or_abort(&s_act[1], (uint32_t)((n_loaded - 1) & 1), abort))
            return false;
          const int sp = pend[i];
          const int r0 = __ldcg(a.offsets + s_list[sp]);
          const uint32_t bytes = kGateUp ? (uint32_t)a.W * 2 : (uint32_t)a.I * 4;
          const void* src = kGateUp ? static_cast<const void*>(a.x16 + (size_t)__ldcg(a.row_token + r0) * a.W)
                                    : static_cast<const void*>(a.h32 + (size_t)r0 * a.I);
          fence_proxy_async_smem();
          mbar_expect_tx(&s_act[0], bytes);
          bulk_g2s(act, src, bytes, &s_act[0]);
          ++n_loaded;
        }
        n_pend = 0;
        return true;
      };
      for (long u = lo; u < hi && ok; ++k) {
        const int n = stage_units(u, r);
        if (si != cur_si) {                   // a new expert: a new activation row?
          cur_si = si;
          const int key = act_key(si);
          if (key != cur_key) {
            cur_key = key;
            pend[n_pend++] = si;
          }
        }
        // a new activation row goes out ahead of the stage's weights (it is
        // small, and the consumers need it before the stage); the down
        // kernel's first h row waits until the ring is full (the weights of
        // its first stages do not depend on the previous grid)
        if (n_pend > 0 && (waited || filled[slot] || n_pend == 4) && !load_acts()) { ok = false; break; }
        if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) { ok = false; break; }
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
      if (ok && n_pend > 0 && !load_acts()) ok = false;
      if (!waited) pdl_wait();                // the grid must not complete before the previous one
      if (*abort) {     // let every issued copy land before the CTA can exit
        for (int s = 0; s < g.nst; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
        if (n_loaded > 0) mbar_wait(&s_act[0], (uint32_t)((n_loaded - 1) & 1));
      }
    }
  } else {
    // ---------------- consumers ----------------
    // gate/up, K > 2048: warps 2p and 2p+1 share row pair p of a stage, each
    // over one half of K (half the activation registers), and combine their
    // partial sums through shared memory; K <= 2048: warp w takes row pair w;
    // down: warp w takes rows RPS*w ... of a stage
    const int w = warp - 1;
    constexpr int BW = kSplit ? (BPL + 1) / 2 : BPL;     // blocks per lane of this warp
    const int half = kSplit ? (w & 1) : 0;
    const int KBw = kSplit ? KB / 2 : KB;                 // blocks of this warp's K range
    const int kb0 = half * KBw;                           // its first block
    uint32_t xr[BW][16];
    float bsc[BW];                                        // down: per-block scale of h
#pragma unroll
    for (int j = 0; j < BW; ++j) bsc[j] = 1.0f;
    float xs = 1.0f;
    int cur_key = -1, cur_si = -1, r0 = 0;
    int si = si0, r = r_lo, slot = 0, k = 0;
    uint32_t ph = 0, act_seen = 0;
    for (long u = lo; u < hi; ++k) {
      const int n = stage_units(u, r);
      const int e = s_list[si];
      bool new_act = false;
      if (si != cur_si) {                     // a new expert: its row, and maybe a new activation row
        cur_si = si;
        r0 = __ldcg(a.offsets + e);
        const int key = act_key(si);
        new_act = key != cur_key;
        cur_key = key;
      }
      if (new_act) {                          // the new activation row: into registers
        if (kGateUp) xs = __ldg(a.xscale + __ldcg(a.row_token + r0));   // while the row is in flight
        if (!tc::wait_or_abort(&s_act[0], act_seen & 1u, abort)) break;
        const uint32_t ab = smem_u32(act);
        // a lane's block is 64 contiguous bytes of f16 (gate/up: the token
        // row; down: the converted h row); the lanes visit its 16-byte chunks
        // in a rotated order so that each access spreads over all banks
        uint32_t xb = ab;
        if (!kGateUp) {
          // warp 0 converts the fp32 h row once: block b -> f16 with the
          // block's own power-of-two scale (its largest |h| into [2^14, 2^15))
          const uint32_t h16 = ab + (uint32_t)K * 4u, hsc = h16 + (uint32_t)K * 2u;
          if (w == 0) {
            for (int b = lane; b < KB; b += 32) {
              const uint32_t hb = ab + (uint32_t)b * 128u;
              float m = 0.0f;
#pragma unroll
              for (int q = 0; q < 8; ++q) {
                const uint4 v = lds16(hb + 16u * ((q + lane) & 7));
                m = fmaxf(m, fmaxf(fmaxf(fabsf(__uint_as_float(v.x)), fabsf(__uint_as_float(v.y))),
                                   fmaxf(fabsf(__uint_as_float(v.z)), fabsf(__uint_as_float(v.w)))));
              }
              float inv = 1.0f, sc = 1.0f;
              if (m > 0.0f && isfinite(m)) {
                const int ex = max(-100, min(127, frexp_exponent(m)));
                sc = pow2_f32(ex - 15);
                inv = pow2_f32(15 - ex);
              }
              sts32(hsc + 4u * b, __float_as_uint(sc));
#pragma unroll
              for (int q = 0; q < 4; ++q) {          // 16 bytes of f16 from 32 bytes of fp32
                const int qq = (q + (lane >> 1)) & 3;
                const uint4 v0 = lds16(hb + 32u * qq), v1 = lds16(hb + 32u * qq + 16u);
                const __half2 p0 = __floats2half2_rn(__uint_as_float(v0.x) * inv, __uint_as_float(v0.y) * inv);
                const __half2 p1 = __floats2half2_rn(__uint_as_float(v0.z) * inv, __uint_as_float(v0.w) * inv);
                const __half2 p2 = __floats2half2_rn(__uint_as_float(v1.x) * inv, __uint_as_float(v1.y) * inv);
                const __half2 p3 = __floats2half2_rn(__uint_as_float(v1.z) * inv, __uint_as_float(v1.w) * inv);
                sts16(h16 + (uint32_t)b * 64u + 16u * qq,
                      make_uint4(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1),
                                 *reinterpret_cast<const uint32_t*>(&p2), *reinterpret_cast<const uint32_t*>(&p3)));
              }
            }
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&s_act[2]);
          }
          if (!tc::wait_or_abort(&s_act[2], act_seen & 1u, abort)) break;
          xb = h16;
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            const int b = lane + 32 * j;
            bsc[j] = b < KB ? __uint_as_float(lds32(hsc + 4u * b)) : 1.0f;
          }
        }
        ++act_seen;
        const int kbx = kGateUp ? kb0 : 0;
#pragma unroll
        for (int j = 0; j < BW; ++j) {
          const int b = lane + 32 * j;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int qq = (q + (lane >> 1)) & 3;
            uint4 t = make_uint4(0u, 0u, 0u, 0u);
            if (b < KBw) t = lds16(xb + (uint32_t)(kbx + b) * 64u + 16u * qq);
#pragma unroll
            for (int s = 0; s < 4; ++s)
              if (qq == s) { xr[j][4 * s] = t.x; xr[j][4 * s + 1] = t.y; xr[j][4 * s + 2] = t.z; xr[j][4 * s + 3] = t.w; }
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&s_act[1]);   // this warp is done with the buffer
      }
      if (!tc::wait_or_abort(&full[slot], ph, abort)) break;
      const uint32_t st = smem_u32(smem + (size_t)slot * g.stage_bytes);
      const uint32_t soff = (uint32_t)((((size_t)e * N + r) * srow) & 15u);
      // rows of this warp: gate/up -> row 0 = gate, row 1 = up of pair w/2;
      // down -> rows RPS*w ... (codes qrow apart, scales srow apart)
      constexpr int NR = kGateUp ? 2 : RPS;
      const int u0 = kGateUp ? (kSplit ? (w >> 1) : w) : RPS * w;
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
                const float sc = kGateUp ? e8m0_exact(code) : e8m0_exact(code) * bsc[j];
                acc[rr] = fmaf(dot_block(wv, xr[j]), sc, acc[rr]);
              }
            }
          }
        }
        if (kSplit) {
          const float gs = warp_sum(acc[0]), us = warp_sum(acc[1]);
          float2* part = s_part[k & 1][u0];
          if (lane == 0) part[half] = make_float2(gs, us);
          asm volatile("bar.sync %0, 64;\n" ::"r"(1 + u0) : "memory");   // the two warps of the pair
          if (half == 0 && lane == 0) {
            const float2 o = part[1];
            a.h32[(size_t)r0 * a.I + r + u0] = silu_f32((gs + o.x) * xs) * ((us + o.y) * xs);
          }
        } else if (kGateUp) {
          const float gs = warp_sum(acc[0]), us = warp_sum(acc[1]);
          if (lane == 0) a.h32[(size_t)r0 * a.I + r + u0] = silu_f32(gs * xs) * (us * xs);
        } else {
#pragma unroll
          for (int rr = 0; rr < NR; ++rr) {
            if (u0 + rr < n) {
              const float sum = warp_sum(acc[rr]);
              if (lane == 0) a.y_perm[(size_t)r0 * a.W + r + u0 + rr] = sum;
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
// (kFmaConsumers for K <= 2048; gate/up: the gate rows, then the up rows, then
// the two E8M0 spans) or
// kFmaConsumers * rps rows (down: codes, then their span); every span with 32
// bytes of alignment slack; after the ring the activation buffer (gate/up: an
// f16 token row of K; down: an fp32 h row of K, its f16 copy and K/32 fp32
// block scales); ring depth nst from the shared-memory budget.
FmaGeometry fma_geometry(int K, bool gate_up, size_t smem_budget) {
  FmaGeometry g{};
  const size_t qrow = K / 2, srow = K / 32;
  const int bpl = (K + 1023) / 1024;
  if (bpl > 8) return g;
  const int rps = gate_up ? 1 : (bpl > 4 ? 1 : bpl > 2 ? 2 : bpl > 1 ? 4 : 8);
  const int units = gate_up ? (bpl > 2 ? kFmaConsumers / 2 : kFmaConsumers) : kFmaConsumers * rps;
  g.rps = rps;
  g.units = units;
  g.code_bytes = (uint32_t)((units * qrow + 127) / 128 * 128);
  const uint32_t code_all = gate_up ? 2 * g.code_bytes : g.code_bytes;
  const uint32_t span = (uint32_t)((units * srow + 32 + 127) / 128 * 128);
  g.sbuf_off = code_all;
  g.sbuf2_off = code_all + span;
  g.stage_bytes = code_all + (gate_up ? 2 : 1) * span;
  // gate/up: the f16 token row; down: the fp32 h row, its f16 copy, the block scales
  const uint32_t act_bytes = (uint32_t)(((size_t)K * (gate_up ? 2 : 6) + (gate_up ? 0 : K / 8) + 127) / 128 * 128);
  if (smem_budget < act_bytes + 2 * (size_t)g.stage_bytes) return g;
  const int nst = (int)((smem_budget - act_bytes) / g.stage_bytes);
  g.nst = nst > kFmaMaxStages ? kFmaMaxStages : nst;
  g.act_off = (uint32_t)g.nst * g.stage_bytes;
  g.smem_bytes = g.act_off + act_bytes;
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
