// MXFP4 GEMV on the CUDA cores for experts that received exactly one token
// (every expert of a 1-token decode step; most experts of small batches).
//
// With one token a tensor-core MMA would use 1 of its 8 columns, and the
// legacy mma.sync rate of sm_100 then caps the kernel near half the HBM
// bandwidth. Here every warp works alone on whole weight rows:
//
// * lane l owns the 32-element K blocks l, l+32, l+64, ... of the activation
//   row (BPL of them), kept in registers as f16 for the whole work item;
// * the warp streams its rows through a private ring of shared-memory stages
//   (RPS rows of packed codes plus their E8M0 codes per stage) filled by bulk
//   TMA copies (cp.async.bulk) that lane 0 issues NST stages ahead, across
//   work-item boundaries, completing on one mbarrier per stage;
// * per 32 weights a lane spends 16 cvt.rn.f16x2.e2m1x2 (exact decode) and
//   32 fma.rn.f32.f16 (exact f16 x f16 products, fp32 sums) and one fp32 FMA
//   for the block scale; a row's sum is a 5-step warp shuffle reduction;
// * no barrier couples the warps of a CTA.
//
// Work items: gate/up = (active expert, RT rows of I): its RT gate rows and
// the RT matching up rows, then h = silu(g) * u written in fp32 to h32;
// down = (active expert, RT rows of W), reading h32 of the expert's token and
// converting it to f16 with one power-of-two scale per row (the largest |h|
// maps into [2^14, 2^15); relative rounding <= 2^-11 for |h| >= 2^-14 max|h|).
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
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4];
    e2m1x8_to_f16x8(words[q], h);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a[2 * (j & 1)] = fma_f16lo(h[j], x[4 * q + j], a[2 * (j & 1)]);
      a[2 * (j & 1) + 1] = fma_f16hi(h[j], x[4 * q + j], a[2 * (j & 1) + 1]);
    }
  }
  return (a[0] + a[1]) + (a[2] + a[3]);
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

// next work item of this warp whose expert received exactly one token
MOE_DEV int next_single_item(const int32_t* __restrict__ list, const int32_t* __restrict__ offsets,
                             int it, int items, int tiles, int stride) {
  for (; it < items; it += stride) {
    const int e = __ldg(list + 1 + it / tiles);
    if (__ldg(offsets + e + 1) - __ldg(offsets + e) == 1) break;
  }
  return it;
}

}  // namespace

// ---------------------------------------------------------------------------
// block = kFmaWarps independent warps; persistent grid; dynamic shared memory
// = kFmaWarps * g.nst * (g.stage_bytes + 8): the warps' rings, then one
// mbarrier per stage
// ---------------------------------------------------------------------------
template <int BPL, bool kGateUp>
__global__ void __launch_bounds__(32 * kFmaWarps) k_fma_gemv(FmaArgs a, FmaGeometry g) {
  extern __shared__ __align__(128) uint8_t smem[];
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = kGateUp ? a.W : a.I;
  const int KB = K >> 5;
  const size_t qrow = (size_t)K / 2, srow = (size_t)K / 32;
  const int RT = g.rt;
  const int item_rows = kGateUp ? 2 * RT : RT;
  const int spi = item_rows / g.rps;                        // stages per item
  const int tiles = kGateUp ? a.I / RT : a.W / RT;
  const int items = __ldg(a.expert_list) * tiles;
  const int gw = blockIdx.x * kFmaWarps + warp, nwarps = gridDim.x * kFmaWarps;
  uint8_t* ring = smem + (size_t)warp * g.nst * g.stage_bytes;
  uint64_t* bars = reinterpret_cast<uint64_t*>(smem + (size_t)kFmaWarps * g.nst * g.stage_bytes) +
                   warp * g.nst;
  const uint32_t cb = (uint32_t)(g.rps * qrow), sb = (uint32_t)(g.rps * srow);

  if (lane == 0) {
    for (int i = 0; i < g.nst; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncwarp();

  // producer cursor (used by lane 0 only): item and stage of the next copy
  int p_item = next_single_item(a.expert_list, a.offsets, gw, items, tiles, nwarps), p_st = 0;
  int p_v = 0;
  auto issue_next = [&]() {
    if (p_item >= items) return;
    const int ai = p_item / tiles, tile = p_item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const int r = p_st * g.rps;                               // row inside the item
    size_t row;
    const uint8_t *q, *s;
    if (kGateUp) {
      row = (size_t)e * a.I + tile * RT + (r < RT ? r : r - RT);
      q = r < RT ? a.wg_q : a.wu_q;
      s = r < RT ? a.wg_s : a.wu_s;
    } else {
      row = (size_t)e * a.W + tile * RT + r;
      q = a.wd_q;
      s = a.wd_s;
    }
    const int slot = p_v % g.nst;
    uint8_t* dst = ring + (size_t)slot * g.stage_bytes;
    fence_proxy_async_smem();           // earlier generic reads of the slot come first
    mbar_expect_tx(&bars[slot], cb + sb);
    bulk_g2s(dst, q + row * qrow, cb, &bars[slot]);
    bulk_g2s(dst + cb, s + row * srow, sb, &bars[slot]);
    ++p_v;
    if (++p_st == spi) {
      p_st = 0;
      p_item = next_single_item(a.expert_list, a.offsets, p_item + nwarps, items, tiles, nwarps);
    }
  };
  if (lane == 0)
    for (int i = 0; i < g.nst; ++i) issue_next();

  bool dead = false;                                          // a wait timed out
  int v = 0;
  for (int item = next_single_item(a.expert_list, a.offsets, gw, items, tiles, nwarps); item < items;
       item = next_single_item(a.expert_list, a.offsets, item + nwarps, items, tiles, nwarps)) {
    const int ai = item / tiles, tile = item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const int r0 = __ldg(a.offsets + e);
    // activation blocks of this lane, f16
    uint32_t xr[BPL][16];
    float xs = 1.0f;
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
          const __half2 lo = __floats2half2_rn(t.x * inv, t.y * inv);
          const __half2 hi = __floats2half2_rn(t.z * inv, t.w * inv);
          xr[j][2 * q] = *reinterpret_cast<const uint32_t*>(&lo);
          xr[j][2 * q + 1] = *reinterpret_cast<const uint32_t*>(&hi);
        }
      }
    }

    float res = 0.0f;                         // lane r keeps the sum of item row r
    for (int st = 0; st < spi; ++st, ++v) {
      const int slot = v % g.nst;
      if (!dead && !mbar_wait(&bars[slot], (uint32_t)(v / g.nst) & 1u)) {
        dead = true;
        if (lane == 0) atomicOr(a.status, kStatusWaitTimeout);
      }
      const uint8_t* stg = ring + (size_t)slot * g.stage_bytes;
      for (int rr = 0; rr < g.rps; ++rr) {
        float acc = 0.0f;
#pragma unroll
        for (int j = 0; j < BPL; ++j) {
          const int b = lane + 32 * j;
          if (b < KB) {
            const uint4 w = *reinterpret_cast<const uint4*>(stg + rr * qrow + b * 16);
            acc = fmaf(dot_block(w, xr[j]), e8m0_to_f32(stg[cb + rr * srow + b]), acc);
          }
        }
        const float sum = warp_sum(acc);
        if (lane == st * g.rps + rr) res = sum;
      }
      __syncwarp();
      if (lane == 0 && !dead) issue_next();   // refill the slot just consumed
    }

    if (kGateUp) {
      // lanes 0..RT-1: gate row tile*RT + lane; lanes RT..2RT-1: the up rows
      const float u = __shfl_down_sync(0xFFFFFFFFu, res, RT);
      const float h = silu_f32(res * xs) * (u * xs);
      if (lane < RT) a.h32[(size_t)r0 * a.I + tile * RT + lane] = h;
    } else {
      if (lane < RT) a.y_perm[(size_t)r0 * a.W + tile * RT + lane] = res * xs;
    }
  }
}

// Geometry for reduction length K (host side): rows per item side RT, rows per
// ring stage rps (a power of two dividing RT with codes about stage_target
// bytes and E8M0 bytes a multiple of 16), ring depth nst from the smem budget.
FmaGeometry fma_geometry(int K, int rt, size_t smem_budget, size_t stage_target) {
  FmaGeometry g{};
  const size_t qrow = K / 2, srow = K / 32;
  int rps = 0;
  for (int r = 1; r <= rt; r *= 2) {
    if (rt % r || (r * srow) % 16) continue;
    rps = r;
    if ((size_t)r * qrow >= stage_target) break;
  }
  if (!rps) return g;
  g.rt = rt;
  g.rps = rps;
  g.stage_bytes = (uint32_t)((rps * (qrow + srow) + 127) / 128 * 128);
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
