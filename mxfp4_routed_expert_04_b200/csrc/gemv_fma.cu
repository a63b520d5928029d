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
//   a row's sum is a 5-step warp shuffle reduction (the one-token launch's
//   down warps sum their rows in one reduce-scatter, warp_sum_rows).
//
// One token (every expert single-token): k_fma_routed1 runs both projections
// in one launch whose CTAs take chunks from device counters (below); more
// tokens: k_fma_gemv<gate/up> then k_fma_gemv<down> over static shares.
//
// gate/up writes h = silu(g) * u in fp32 to h32; down reads h32 of the
// expert's token and converts it to f16 with one power-of-two scale per
// 32-element block (the block's largest |h| maps into [2^14, 2^15): relative
// rounding <= 2^-11). The token rows come the same way, one scale per row.
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
              float sc, inv;
              f16_block_scale(m, sc, inv, kF16OpTop);
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

// ---------------------------------------------------------------------------
// One token: gate/up and down of all its experts in ONE launch.
//
// With one token every active expert is a single-token expert. Two launches
// (gate/up, then down) over equal static shares end with the slowest CTA of
// each grid. Here every CTA takes chunks of work from two device counters as
// it frees a ring slot: first the gate/up chunks of all experts (chunk j =
// row pairs [P j', P j' + P) of expert slot j / cpe, experts in list order),
// then the down chunks (two at a time, so that most consecutive chunks of a
// CTA share an expert). A stage carries one chunk; its descriptor (job) sits
// beside the stage in shared memory, so the consumers, the producer and the
// signal warp walk the same sequence.
//
// Hand-over of h, per expert slot s: the gate/up consumers write their h
// values and arrive on the stage's hdone barrier; the signal warp then hands
// the slot back to the producer, fences (the h values become visible device-
// wide) and adds the stage's row pairs to sync[1 + s]. Before the first down
// chunk of an expert, the producer warp (after issuing that chunk's weight
// copies) waits until sync[1 + s] holds all I row pairs, reads the fp32 h
// row from L2 and converts it to f16 with one power-of-two scale per
// 32-element block into one of two buffers; the consumers load it into
// registers when they reach the chunk.
//
// Progress: a chunk is taken only by a running CTA, gate/up chunks depend on
// nothing, and a CTA takes down chunks only after the gate/up chunks are all
// taken, so every h row a down chunk waits for is being produced by running
// CTAs whatever the residency. Every wait is bounded (a timeout raises the
// abort flag and kStatusWaitTimeout).
// When a CTA finds no chunk left, it prefetches its share of the next
// kernel's weights (FmaArgs::l2_next) into L2: the HBM is otherwise idle
// while the last stages are computed.
// Counters: sync[0] finished CTAs, sync[1 + s] h row pairs of expert slot s,
// sync[kSyncGateUp] / sync[kSyncDown] the next chunk of each kind; the last
// CTA to finish puts them all back to zero (the workspace clear zeroes them
// first).
// ---------------------------------------------------------------------------
namespace {

constexpr int kSyncGateUp = 1 + kRouted1MaxK, kSyncDown = 2 + kRouted1MaxK;
constexpr int kDownGrab = 2;                 // down chunks taken at a time
enum : int { kJobGateUp = 0, kJobDown = 1, kJobDone = 2 };

// bounded wait of a whole warp with one decision (lane 0's), so that the
// warp leaves a loop together
MOE_DEV bool warp_wait(uint64_t* bar, uint32_t parity, volatile int* abort) {
  const int ok = tc::wait_or_abort(bar, parity, abort) ? 1 : 0;
  return __shfl_sync(0xFFFFFFFFu, ok, 0) != 0;
}

MOE_DEV int ld_acquire_gpu(const int32_t* p) {
  int v;
  asm volatile("ld.acquire.gpu.global.s32 %0, [%1];\n" : "=r"(v) : "l"(p) : "memory");
  return v;
}

// Sums over the warp of R per-lane values (R = 1, 2, 4, 8) in reduce-scatter
// form: log2 R halving steps (each lane keeps half of its values and adds the
// partner's copy of that half: R - 1 shuffles in all), then a butterfly over
// the remaining 32 / R lanes; returns the sum of value `row` = lane / (32 / R),
// the same in all 32 / R lanes of the group.
template <int R>
MOE_DEV float warp_sum_rows(const float (&v)[R], int lane, int& row) {
  constexpr int kSteps = R == 8 ? 3 : R == 4 ? 2 : R == 2 ? 1 : 0;
  static_assert(R == (1 << kSteps), "R must be 1, 2, 4 or 8");
  float c[R];
#pragma unroll
  for (int i = 0; i < R; ++i) c[i] = v[i];
#pragma unroll
  for (int s = 0; s < kSteps; ++s) {
    const int n = R >> s, off = 16 >> s;
    const bool up = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < n / 2; ++i) {
      const float keep = up ? c[n / 2 + i] : c[i];
      const float send = up ? c[i] : c[n / 2 + i];
      c[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
    }
  }
#pragma unroll
  for (int off = 16 >> kSteps; off >= 1; off >>= 1) c[0] += __shfl_xor_sync(0xFFFFFFFFu, c[0], off);
  row = lane >> (5 - kSteps);
  return c[0];
}

// place 16 bytes read in rotated order qq into x[4 qq .. 4 qq + 3] without
// dynamic register indexing
MOE_DEV void put16(uint32_t (&x)[16], int qq, uint4 t) {
#pragma unroll
  for (int s = 0; s < 4; ++s)
    if (qq == s) { x[4 * s] = t.x; x[4 * s + 1] = t.y; x[4 * s + 2] = t.z; x[4 * s + 3] = t.w; }
}

// the f16 copy of the expert's h row (K fp32 values) with one power-of-two
// scale per 32-element block, by one warp: block b -> 64 bytes at hb + 64 b,
// its scale at hsc + 4 b
MOE_DEV void convert_h_row(const float* hrow, int K, uint32_t hb, uint32_t hsc) {
  const int lane = threadIdx.x & 31;
  for (int blk = lane; blk < (K >> 5); blk += 32) {
    float v[32];
    const float4* src = reinterpret_cast<const float4*>(hrow + (size_t)blk * 32);
#pragma unroll
    for (int q = 0; q < 8; ++q) {
      const float4 t = __ldcg(src + q);
      v[4 * q] = t.x; v[4 * q + 1] = t.y; v[4 * q + 2] = t.z; v[4 * q + 3] = t.w;
    }
    float m = 0.0f;
#pragma unroll
    for (int i = 0; i < 32; ++i) m = fmaxf(m, fabsf(v[i]));
    float sc, inv;
    f16_block_scale(m, sc, inv, kF16OpTop);
    sts32(hsc + 4u * blk, __float_as_uint(sc));
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint32_t wv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        const __half2 p2 = __floats2half2_rn(v[8 * q + 2 * i] * inv, v[8 * q + 2 * i + 1] * inv);
        wv[i] = *reinterpret_cast<const uint32_t*>(&p2);
      }
      sts16(hb + (uint32_t)blk * 64u + 16u * q, make_uint4(wv[0], wv[1], wv[2], wv[3]));
    }
  }
}

struct Routed1Smem {
  uint64_t* full;       // [nst] stage landed (count 1: the producer's expect_tx or the done marker)
  uint64_t* empty;      // [nst] stage free (count 1: the signal warp)
  uint64_t* hdone;      // [nst] consumers done with the stage (count kFmaConsumers)
  uint64_t* act_full;   // the token row landed
  uint64_t* x_free;     // consumers have the token row in registers (count kFmaConsumers)
  uint64_t* hb_full;    // [2] f16 h buffer ready
  uint64_t* hb_empty;   // [2] consumers have the buffer in registers (count kFmaConsumers)
  int4* job;            // [nst] {kind, expert slot, first unit, units}
  float2 (*part)[kFmaConsumers / 2];     // gate/up: second-half sums per (slot, pair)
  uint64_t (*pbar)[kFmaConsumers / 2];
  const int16_t* list;
  volatile int* abort;
};

}  // namespace

template <int BG, int BD, int RPSD>
__global__ void __launch_bounds__(32 * kRouted1Warps, 1)
    k_fma_routed1(FmaArgs a, FmaGeometry gg, FmaGeometry gd) {
  pdl_wait();                          // the dispatch of the previous kernel
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ int16_t s_list[kRouted1MaxK];
  __shared__ uint64_t s_bars[3 * kFmaMaxStages + 6];
  __shared__ int4 s_job[kFmaMaxStages];
  __shared__ float2 s_part[kFmaMaxStages][kFmaConsumers / 2];
  __shared__ uint64_t s_pbar[kFmaMaxStages][kFmaConsumers / 2];
  __shared__ int s_abort;
  constexpr bool kSplit = BG > 2;      // gate/up: two warps per row pair, each over half of K
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int nst = gg.nst;              // the ring and the activation region are common to both kinds
  const uint32_t stride = gg.stage_bytes;
  const int n_slots = min(__ldcg(a.expert_list), kRouted1MaxK);
  if ((int)threadIdx.x < n_slots) s_list[threadIdx.x] = (int16_t)__ldcg(a.expert_list + 1 + threadIdx.x);
  Routed1Smem S;
  S.full = s_bars;
  S.empty = s_bars + kFmaMaxStages;
  S.hdone = s_bars + 2 * kFmaMaxStages;
  S.act_full = s_bars + 3 * kFmaMaxStages;
  S.x_free = S.act_full + 1;
  S.hb_full = S.act_full + 2;
  S.hb_empty = S.act_full + 4;
  S.job = s_job;
  S.part = s_part;
  S.pbar = s_pbar;
  S.list = s_list;
  S.abort = &s_abort;
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&S.full[s], 1);
      mbar_init(&S.empty[s], 1);
      mbar_init(&S.hdone[s], kFmaConsumers);
      for (int q = 0; q < kFmaConsumers / 2; ++q) mbar_init(&s_pbar[s][q], 1);
    }
    mbar_init(S.act_full, 1);
    mbar_init(S.x_free, kFmaConsumers);
    mbar_init(&S.hb_full[0], 1);
    mbar_init(&S.hb_full[1], 1);
    mbar_init(&S.hb_empty[0], kFmaConsumers);
    mbar_init(&S.hb_empty[1], kFmaConsumers);
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  // chunk counts: gate/up units are row pairs (N = I), down units rows (N = W)
  const int cpe_g = (a.I + gg.units - 1) / gg.units, cpe_d = (a.W + gd.units - 1) / gd.units;
  const int total_g = n_slots * cpe_g, total_d = n_slots * cpe_d;
  uint8_t* act = smem + gg.act_off;    // the token row (f16), later the two f16 h buffers
  const int Kg = a.W, Kd = a.I;

  if (warp == 0) {
    // ---------------- producer (lane 0 copies; the warp converts h rows) ----------------
    uint32_t last_ph[kFmaMaxStages];
    bool filled[kFmaMaxStages];
#pragma unroll
    for (int s = 0; s < kFmaMaxStages; ++s) { last_ph[s] = 0; filled[s] = false; }
    int slot = 0, cur_dsi = -1, nh = 0, kind = kJobGateUp;
    uint32_t ph = 0;
    bool x_waited = false;
    int tok = 0;
    if (n_slots > 0) tok = __ldcg(a.row_token + __ldcg(a.offsets + s_list[0]));   // the one token
    if (lane == 0 && n_slots > 0) {
      asm volatile("fence.proxy.async;\n" ::: "memory");   // the previous grid's writes, then bulk reads
      mbar_expect_tx(S.act_full, (uint32_t)Kg * 2);
      bulk_g2s(act, a.x16 + (size_t)tok * Kg, (uint32_t)Kg * 2, S.act_full);
    }
    int held = 0, held_j = 0;                // down chunks taken but not yet issued
    for (;;) {
      if (!warp_wait(&S.empty[slot], ph ^ 1u, abort)) break;
      // the next chunk
      int jk = kJobDone, j = 0;
      if (lane == 0) {
        if (kind == kJobGateUp) {
          j = atomicAdd(a.sync + kSyncGateUp, 1);
          if (j < total_g) jk = kJobGateUp;
          else kind = kJobDown;
        }
        if (kind == kJobDown) {
          if (held == 0) {
            held_j = atomicAdd(a.sync + kSyncDown, kDownGrab);
            held = kDownGrab;
          }
          j = held_j++;
          --held;
          if (j < total_d) jk = kJobDown;
          else held = 0;
        }
      }
      jk = __shfl_sync(0xFFFFFFFFu, jk, 0);
      j = __shfl_sync(0xFFFFFFFFu, j, 0);
      if (jk == kJobDone) {
        if (lane == 0) {
          s_job[slot] = make_int4(kJobDone, 0, 0, 0);
          tc::mbar_arrive(&S.full[slot]);
          // no chunks left: this CTA's share of what the next kernel reads
          // into L2, while the last stages of the launch are still computed
          if (a.l2_next) {
            const uint64_t per = ((a.l2_next_bytes + gridDim.x - 1) / gridDim.x + 15) & ~(uint64_t)15;
            const uint64_t lo = per * blockIdx.x;
            const uint64_t hi = min(lo + per, a.l2_next_bytes);
            for (uint64_t o = lo; o < hi; o += 32768)
              tc::prefetch_l2(static_cast<const uint8_t*>(a.l2_next) + o, (uint32_t)min((uint64_t)32768, hi - o));
          }
        }
        break;
      }
      const bool gu = jk == kJobGateUp;
      const FmaGeometry& g = gu ? gg : gd;
      const int cpe = gu ? cpe_g : cpe_d, N = gu ? a.I : a.W, K = gu ? Kg : Kd;
      const int si = j / cpe, r = (j - si * cpe) * g.units, n = min(g.units, N - r);
      if (lane == 0) {
        const uint32_t qrow = (uint32_t)K / 2, srow = (uint32_t)K / 32;
        const size_t s_total = (size_t)a.E * N * srow;
        const size_t row = (size_t)s_list[si] * N + r;
        const uint32_t cb = n * qrow;
        const size_t s0 = row * srow, s1 = (row + n) * srow;
        const size_t a0 = s0 & ~(size_t)15, a1 = min((s1 + 15) & ~(size_t)15, s_total);
        const uint32_t sb = (uint32_t)(a1 - a0);
        uint8_t* st = smem + (size_t)slot * stride;
        s_job[slot] = make_int4(jk, si, r, n);
        fence_proxy_async_smem();            // the consumers' reads of the slot come first
        if (gu) {
          mbar_expect_tx(&S.full[slot], 2 * cb + 2 * sb);
          bulk_g2s(st, a.wg_q + row * qrow, cb, &S.full[slot]);
          bulk_g2s(st + g.code_bytes, a.wu_q + row * qrow, cb, &S.full[slot]);
          bulk_g2s(st + g.sbuf_off, a.wg_s + a0, sb, &S.full[slot]);
          bulk_g2s(st + g.sbuf2_off, a.wu_s + a0, sb, &S.full[slot]);
        } else {
          mbar_expect_tx(&S.full[slot], cb + sb);
          bulk_g2s(st, a.wd_q + row * qrow, cb, &S.full[slot]);
          bulk_g2s(st + g.sbuf_off, a.wd_s + a0, sb, &S.full[slot]);
        }
        last_ph[slot] = ph;
        filled[slot] = true;
      }
      if (!gu && si != cur_dsi) {
        // the first down chunk of this expert here: its h row into the next buffer
        cur_dsi = si;
        const int b = nh & 1;
        if (!x_waited) {                    // the buffers overlay the token row
          if (!warp_wait(S.x_free, 0, abort)) break;
          x_waited = true;
        }
        if (nh >= 2 && !warp_wait(&S.hb_empty[b], (uint32_t)(((nh >> 1) - 1) & 1), abort)) break;
        int ok = 1;
        if (lane == 0) {
          uint32_t it = 0;
          while (ld_acquire_gpu(a.sync + 1 + si) < a.I) {
            if (*abort || ++it > (1u << 22)) { ok = 0; break; }
            __nanosleep(64);
          }
          if (!ok) *abort = 1;
        }
        if (!__shfl_sync(0xFFFFFFFFu, ok, 0)) break;
        __syncwarp();                       // lane 0's acquire orders the other lanes' reads
        const uint32_t hb = smem_u32(act) + (uint32_t)b * gd.act_stride;
        convert_h_row(a.h32 + (size_t)__ldcg(a.offsets + s_list[si]) * Kd, Kd, hb, hb + (uint32_t)Kd * 2u);
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.hb_full[b]);
        ++nh;
      }
      if (++slot == nst) { slot = 0; ph ^= 1u; }
    }
    if (lane == 0 && *abort) {     // let every issued copy land before the CTA can exit
      if (n_slots > 0) mbar_wait(S.act_full, 0);
      for (int s = 0; s < nst; ++s)
        if (filled[s]) mbar_wait(&S.full[s], last_ph[s]);
    }
  } else if (warp <= kFmaConsumers) {
    // ---------------- consumers ----------------
    const int w = warp - 1;
    int slot = 0;
    uint32_t ph = 0;
    int4 job = make_int4(kJobDone, 0, 0, 0);
    bool have = false;
    if (n_slots > 0) {
      // gate/up jobs: the token row in registers (gate/up K > 2048: warps 2p
      // and 2p+1 take row pair p of a stage, each over one half of K)
      constexpr int BW = kSplit ? (BG + 1) / 2 : BG;
      const int half = kSplit ? (w & 1) : 0;
      const int KB = Kg >> 5;
      const int KBw = kSplit ? KB / 2 : KB;
      const int kb0 = half * KBw;
      const uint32_t qrow = (uint32_t)Kg / 2, srow = (uint32_t)Kg / 32;
      uint32_t xr[BW][16];
      bool ok = warp_wait(S.act_full, 0, abort);
      if (ok) {
        const uint32_t ab = smem_u32(act);
#pragma unroll
        for (int j = 0; j < BW; ++j) {
          const int b = lane + 32 * j;
#pragma unroll
          for (int q = 0; q < 4; ++q) {
            const int qq = (q + (lane >> 1)) & 3;
            uint4 t = make_uint4(0u, 0u, 0u, 0u);
            if (b < KBw) t = lds16(ab + (uint32_t)(kb0 + b) * 64u + 16u * qq);
            put16(xr[j], qq, t);
          }
        }
      }
      __syncwarp();
      if (lane == 0) tc::mbar_arrive(S.x_free);    // the region may now hold h buffers
      const float xs = ok ? __ldg(a.xscale + __ldcg(a.row_token + __ldcg(a.offsets + s_list[0]))) : 0.0f;
      const int u0 = kSplit ? (w >> 1) : w;
      uint32_t pph = 0;          // per slot: phase parity of this pair's exchange barrier
      while (ok) {
        if (!warp_wait(&S.full[slot], ph, abort)) break;
        job = s_job[slot];
        if (job.x != kJobGateUp) { have = true; break; }   // this slot is the first of the down jobs
        const int si = job.y, r = job.z, n = job.w;
        const int e = s_list[si];
        const int r0 = __ldcg(a.offsets + e);
        const uint32_t st = smem_u32(smem + (size_t)slot * stride);
        const uint32_t soff = (uint32_t)((((size_t)e * a.I + r) * srow) & 15u);
        if (u0 < n) {
          float acc[2] = {0.0f, 0.0f};
          uint32_t cb[2], sbs[2];
#pragma unroll
          for (int rr = 0; rr < 2; ++rr) {
            cb[rr] = st + rr * gg.code_bytes + u0 * qrow + 16u * (kb0 + lane);
            sbs[rr] = st + (rr ? gg.sbuf2_off : gg.sbuf_off) + soff + u0 * srow + kb0 + lane;
          }
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            if (lane + 32 * j < KBw) {
#pragma unroll
              for (int rr = 0; rr < 2; ++rr) {
                const uint4 wv = lds16(cb[rr] + 512u * j);
                const uint32_t code = lds8(sbs[rr] + 32u * j);
                acc[rr] = fmaf(dot_block(wv, xr[j]), e8m0_exact(code), acc[rr]);
              }
            }
          }
          const float gs = warp_sum(acc[0]), us = warp_sum(acc[1]);
          if (kSplit) {
            // the second half's sums reach the first through shared memory and
            // a (slot, pair) barrier: bounded, and a slot is not refilled before
            // both warps are done with it, so the second warp cannot arrive
            // twice before the first has waited
            if (half == 1) {
              if (lane == 0) {
                s_part[slot][u0] = make_float2(gs, us);
                tc::mbar_arrive(&s_pbar[slot][u0]);
              }
              pph ^= 1u << slot;
            } else {
              if (!warp_wait(&s_pbar[slot][u0], (pph >> slot) & 1u, abort)) break;
              if (lane == 0) {
                const float2 o = s_part[slot][u0];
                a.h32[(size_t)r0 * a.I + r + u0] = silu_f32((gs + o.x) * xs) * ((us + o.y) * xs);
              }
              pph ^= 1u << slot;
            }
          } else if (lane == 0) {
            a.h32[(size_t)r0 * a.I + r + u0] = silu_f32(gs * xs) * (us * xs);
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.hdone[slot]);    // this warp's h values are written
        if (++slot == nst) { slot = 0; ph ^= 1u; }
      }
    }
    if (have && job.x == kJobDown) {
      // down jobs: warp w takes rows RPSD*w ... of a stage; the expert's f16 h
      // row in registers, loaded at each new expert
      constexpr int BW = BD;
      const int KB = Kd >> 5;
      const uint32_t qrow = (uint32_t)Kd / 2, srow = (uint32_t)Kd / 32;
      uint32_t xr[BW][16];
      float bsc[BW];
      int cur_si = -1, r0 = 0, nh = 0;
      const int u0 = RPSD * w;
      for (;;) {
        const int si = job.y, r = job.z, n = job.w;
        const int e = s_list[si];
        if (si != cur_si) {                   // a new expert: its f16 h row into registers
          cur_si = si;
          r0 = __ldcg(a.offsets + e);
          const int b = nh & 1;
          if (!warp_wait(&S.hb_full[b], (uint32_t)((nh >> 1) & 1), abort)) break;
          const uint32_t hb = smem_u32(act) + (uint32_t)b * gd.act_stride;
          const uint32_t hsc = hb + (uint32_t)Kd * 2u;
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            const int blk = lane + 32 * j;
            bsc[j] = blk < KB ? __uint_as_float(lds32(hsc + 4u * blk)) : 1.0f;
#pragma unroll
            for (int q = 0; q < 4; ++q) {
              const int qq = (q + (lane >> 1)) & 3;
              uint4 t = make_uint4(0u, 0u, 0u, 0u);
              if (blk < KB) t = lds16(hb + (uint32_t)blk * 64u + 16u * qq);
              put16(xr[j], qq, t);
            }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&S.hb_empty[b]);   // this warp is done with the buffer
          ++nh;
        }
        const uint32_t st = smem_u32(smem + (size_t)slot * stride);
        const uint32_t soff = (uint32_t)((((size_t)e * a.W + r) * srow) & 15u);
        if (u0 < n) {
          float acc[RPSD];
          uint32_t cb[RPSD], sbs[RPSD];
#pragma unroll
          for (int rr = 0; rr < RPSD; ++rr) {
            acc[rr] = 0.0f;
            cb[rr] = st + (u0 + rr) * qrow + 16u * lane;
            sbs[rr] = st + gd.sbuf_off + soff + (u0 + rr) * srow + lane;
          }
#pragma unroll
          for (int j = 0; j < BW; ++j) {
            if (lane + 32 * j < KB) {
#pragma unroll
              for (int rr = 0; rr < RPSD; ++rr) {
                if (u0 + rr < n) {
                  const uint4 wv = lds16(cb[rr] + 512u * j);
                  const uint32_t code = lds8(sbs[rr] + 32u * j);
                  acc[rr] = fmaf(dot_block(wv, xr[j]), e8m0_exact(code) * bsc[j], acc[rr]);
                }
              }
            }
          }
          // the RPSD row sums in one reduce-scatter; lane row * 32 / RPSD
          // writes row `row`
          int row;
          const float sum = warp_sum_rows<RPSD>(acc, lane, row);
          if ((lane & (32 / RPSD - 1)) == 0 && u0 + row < n) a.y_perm[(size_t)r0 * a.W + r + u0 + row] = sum;
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&S.hdone[slot]);   // this warp is done with the slot
        if (++slot == nst) { slot = 0; ph ^= 1u; }
        if (!warp_wait(&S.full[slot], ph, abort)) break;
        job = s_job[slot];
        if (job.x != kJobDown) break;
      }
    }
  } else {
    // ---------------- signal warp ----------------
    // each stage: consumers done -> slot back to the producer; a gate/up
    // stage's h values then become visible device-wide before its count is added
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      for (;;) {
        if (!tc::wait_or_abort(&S.full[slot], ph, abort)) break;
        const int4 job = s_job[slot];
        if (job.x == kJobDone) break;
        if (!tc::wait_or_abort(&S.hdone[slot], ph, abort)) break;
        tc::mbar_arrive(&S.empty[slot]);
        if (job.x == kJobGateUp) {
          __threadfence();
          atomicAdd(a.sync + 1 + job.y, job.w);
        }
        if (++slot == nst) { slot = 0; ph ^= 1u; }
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0) {
    if (*abort) atomicOr(a.status, kStatusWaitTimeout);
    // the last CTA to finish clears the counters for the next launch
    __threadfence();
    if (atomicAdd(a.sync, 1) == (int)gridDim.x - 1) {
      for (int s = 1; s <= kSyncDown; ++s) a.sync[s] = 0;
      __threadfence();
      a.sync[0] = 0;
    }
  }
}

// Geometry for reduction length K (host side): rows per consumer warp in a
// down stage rps = max(1, 8 / BPL); a stage holds kFmaConsumers / 2 row pairs
// (kFmaConsumers for K <= 2048; gate/up: the gate rows, then the up rows, then
// the two E8M0 spans) or
// kFmaConsumers * rps rows (down: codes, then their span); every span with 32
// bytes of alignment slack; after the ring the activation buffer (gate/up: an
// f16 token row of K; down: an fp32 h row of K, its f16 copy and K/32 fp32
// block scales; the one-token launch instead: two buffers of the f16 row and
// its block scales); ring depth nst from the shared-memory budget.
FmaGeometry fma_geometry(int K, bool gate_up, size_t smem_budget, bool routed1) {
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
  g.act_stride = (uint32_t)(((size_t)K * 2 + K / 8 + 127) / 128 * 128);
  uint32_t act_bytes = (uint32_t)(((size_t)K * (gate_up ? 2 : 6) + (gate_up ? 0 : K / 8) + 127) / 128 * 128);
  if (routed1 && !gate_up) act_bytes = 2 * g.act_stride;
  if (smem_budget < act_bytes + 2 * (size_t)g.stage_bytes) return g;
  const int nst = (int)((smem_budget - act_bytes) / g.stage_bytes);
  g.nst = nst > kFmaMaxStages ? kFmaMaxStages : nst;
  g.act_off = (uint32_t)g.nst * g.stage_bytes;
  g.smem_bytes = g.act_off + act_bytes;
  g.ok = 1;
  return g;
}

void routed1_geometry(int W, int I, size_t smem_budget, FmaGeometry& gg, FmaGeometry& gd) {
  gg = fma_geometry(W, true, smem_budget);
  gd = fma_geometry(I, false, smem_budget, true);
  if (!gg.ok || !gd.ok) { gg.ok = gd.ok = 0; return; }
  const uint32_t stride = gg.stage_bytes > gd.stage_bytes ? gg.stage_bytes : gd.stage_bytes;
  const uint32_t xrow = (uint32_t)(((size_t)W * 2 + 127) / 128 * 128);
  const uint32_t act = xrow > 2 * gd.act_stride ? xrow : 2 * gd.act_stride;
  if (smem_budget < act + 2 * (size_t)stride) { gg.ok = gd.ok = 0; return; }
  int nst = (int)((smem_budget - act) / stride);
  if (nst > kFmaMaxStages) nst = kFmaMaxStages;
  for (FmaGeometry* g : {&gg, &gd}) {
    g->stage_bytes = stride;
    g->nst = nst;
    g->act_off = (uint32_t)nst * stride;
    g->smem_bytes = g->act_off + act;
  }
}

#define MOE_FMA_INST(BPL, RPS)                                                 \
  template __global__ void k_fma_gemv<BPL, true, 1>(FmaArgs, FmaGeometry);    \
  template __global__ void k_fma_gemv<BPL, false, RPS>(FmaArgs, FmaGeometry);
MOE_FMA_INST(1, 8)
MOE_FMA_INST(2, 4)
MOE_FMA_INST(4, 2)
MOE_FMA_INST(8, 1)
#undef MOE_FMA_INST

#define MOE_ROUTED1_INST(BG)                                                            \
  template __global__ void k_fma_routed1<BG, 1, 8>(FmaArgs, FmaGeometry, FmaGeometry); \
  template __global__ void k_fma_routed1<BG, 2, 4>(FmaArgs, FmaGeometry, FmaGeometry); \
  template __global__ void k_fma_routed1<BG, 4, 2>(FmaArgs, FmaGeometry, FmaGeometry); \
  template __global__ void k_fma_routed1<BG, 8, 1>(FmaArgs, FmaGeometry, FmaGeometry);
MOE_ROUTED1_INST(1)
MOE_ROUTED1_INST(2)
MOE_ROUTED1_INST(4)
MOE_ROUTED1_INST(8)
#undef MOE_ROUTED1_INST

}  // namespace moe
