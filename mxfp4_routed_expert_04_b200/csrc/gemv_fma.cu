// MXFP4 GEMV on the CUDA cores for experts that received exactly one token
// (every expert of a 1-token decode step; most experts of small batches).
//
// With one token a tensor-core MMA would use 1 of its 8 columns, and the
// legacy mma.sync rate of sm_100 then caps the kernel near half the HBM
// bandwidth. Design, per persistent CTA:
//
// * weights stream through a 4-slot shared-memory ring filled by bulk TMA
//   copies (cp.async.bulk, one per stage for the packed codes of RPS
//   consecutive rows and one for their E8M0 codes) completing on mbarriers;
//   the producer thread runs 3 stages ahead, across work-item boundaries, so
//   HBM stays busy while the CTA reduces and writes an item;
// * every thread owns BPT fixed 32-element K blocks of the activation row,
//   kept in registers as f16, and reads the matching 16-byte code slices of
//   each staged row (consecutive threads, consecutive 16 bytes);
// * per 32 weights a thread spends 16 cvt.rn.f16x2.e2m1x2 (exact decode) and
//   32 fma.rn.f32.f16 (exact f16 x f16 product, fp32 accumulation), then one
//   fp32 FMA applies the E8M0 block scale;
// * row sums are reduced across the CTA by a warp reduce-scatter and one
//   shared-memory pass at the end of each item.
//
// Work items: gate/up = (active expert, 16-row tile of I) over the 16 gate
// rows then the 16 up rows; down = (active expert, 32-row tile of W).
// The h produced here is f16 with one power-of-two scale per group of 16
// CONSECUTIVE intermediate rows (the tensor-core path uses interleaved groups;
// an expert's gate/up and down always take the same path).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kRing = 4;              // ring slots
constexpr int kItemRows = 32;         // weight rows per work item

// Dot products of the two 16-element halves of one MXFP4 block with 32 f16
// activations (block scale not applied).
MOE_DEV void dot_block_halves(uint4 w, const uint32_t (&x)[16], float& p0, float& p1) {
  const uint32_t words[4] = {w.x, w.y, w.z, w.w};
  float a[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
  for (int q = 0; q < 4; ++q) {
    uint32_t h[4];
    e2m1x8_to_f16x8(words[q], h);
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      a[(q >> 1) * 2] = fma_f16lo(h[j], x[4 * q + j], a[(q >> 1) * 2]);
      a[(q >> 1) * 2 + 1] = fma_f16hi(h[j], x[4 * q + j], a[(q >> 1) * 2 + 1]);
    }
  }
  p0 = a[0] + a[1];
  p1 = a[2] + a[3];
}

template <int BPT>
MOE_DEV void load_act_blocks(uint32_t (&xr)[BPT][16], const __half* row, int KB) {
#pragma unroll
  for (int j = 0; j < BPT; ++j) {
    const int b = threadIdx.x + j * blockDim.x;
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      uint4 v = make_uint4(0u, 0u, 0u, 0u);
      if (b < KB) v = ldg16(row + b * 32 + 8 * q);
      xr[j][4 * q] = v.x; xr[j][4 * q + 1] = v.y; xr[j][4 * q + 2] = v.z; xr[j][4 * q + 3] = v.w;
    }
  }
}

// CTA-wide sum of acc[32] (one value per row): returns row `lane`'s total in
// every lane of warp 0. `red` holds 32 x 33 floats.
MOE_DEV float cta_row_sums(float (&acc)[32], float (*red)[33]) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5, nw = blockDim.x >> 5;
  const float v = warp_reduce_scatter32(acc, lane);
  red[warp][lane] = v;
  __syncthreads();
  float s = 0.f;
  if (warp == 0)
    for (int w = 0; w < nw; ++w) s += red[w][lane];
  return s;
}

// The CTA's work items, in order, restricted to experts with exactly one
// token. Every thread walks the same sequence.
struct ItemCursor {
  int item;    // current item (>= items: done)
  int stage;   // stage inside the item
};

MOE_DEV int next_single_item(const int32_t* __restrict__ list, const int32_t* __restrict__ offsets,
                             int it, int items, int tiles) {
  for (; it < items; it += gridDim.x) {
    const int e = __ldg(list + 1 + it / tiles);
    if (__ldg(offsets + e + 1) - __ldg(offsets + e) == 1) break;
  }
  return it;
}

}  // namespace

// ---------------------------------------------------------------------------
// grid: persistent; block: KB/BPT threads rounded up to a warp (<= 256);
// dynamic smem: kRing stages of RPS rows (codes, then E8M0 codes)
// ---------------------------------------------------------------------------
template <int BPT, int RPS, bool kGateUp>
__global__ void __launch_bounds__(kFmaMaxThreads) k_fma_gemv(FmaArgs a) {
  constexpr int SPI = kItemRows / RPS;          // stages per item
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[32][33];
  __shared__ __align__(8) uint64_t bars[kRing];
  const int K = kGateUp ? a.W : a.I;            // reduction length
  const int KB = K >> 5;
  const size_t qrow = (size_t)K / 2, srow = (size_t)K / 32;
  const uint32_t cbytes = (uint32_t)(RPS * qrow), sbytes = (uint32_t)(RPS * srow);
  const uint32_t stage_bytes = (cbytes + sbytes + 127u) & ~127u;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int tiles = kGateUp ? (a.I >> 4) : (a.W >> 5);
  const int items = __ldg(a.expert_list) * tiles;

  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing; ++i) mbar_init(&bars[i], 1);
    fence_mbar_init();
  }
  __syncthreads();

  // producer: issue stage `st` of `item` into ring slot `slot`
  auto issue = [&](int item, int st, int slot) {
    const int ai = item / tiles, tile = item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const uint8_t *q, *s;
    size_t row;
    if (kGateUp) {
      const int r = st * RPS;                   // 0..31: gate rows then up rows
      row = (size_t)e * a.I + tile * 16 + (r & 15);
      q = (r < 16 ? a.wg_q : a.wu_q);
      s = (r < 16 ? a.wg_s : a.wu_s);
    } else {
      row = (size_t)e * a.W + tile * 32 + st * RPS;
      q = a.wd_q;
      s = a.wd_s;
    }
    uint8_t* dst = smem + (size_t)slot * stage_bytes;
    mbar_expect_tx(&bars[slot], cbytes + sbytes);
    bulk_g2s(dst, q + row * qrow, cbytes, &bars[slot]);
    bulk_g2s(dst + cbytes, s + row * srow, sbytes, &bars[slot]);
  };

  ItemCursor prod{next_single_item(a.expert_list, a.offsets, blockIdx.x, items, tiles), 0};
  int prod_v = 0;                               // stages issued so far
  auto advance = [&](ItemCursor& c) {
    if (++c.stage == SPI) {
      c.stage = 0;
      c.item = next_single_item(a.expert_list, a.offsets, c.item + gridDim.x, items, tiles);
    }
  };
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRing && prod.item < items; ++i) {
      issue(prod.item, prod.stage, prod_v % kRing);
      ++prod_v;
      advance(prod);
    }
  }

  int cons_v = 0;                               // stages consumed so far
  for (int item = next_single_item(a.expert_list, a.offsets, blockIdx.x, items, tiles); item < items;
       item = next_single_item(a.expert_list, a.offsets, item + gridDim.x, items, tiles)) {
    const int ai = item / tiles, tile = item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const int r0 = __ldg(a.offsets + e);
    uint32_t xr[BPT][16];
    float hs[BPT][2];
    int tok = 0;
    if (kGateUp) {
      tok = __ldg(a.row_token + r0);
      load_act_blocks<BPT>(xr, a.x16 + (size_t)tok * a.W, KB);
    } else {
      load_act_blocks<BPT>(xr, a.h16 + (size_t)r0 * a.I, KB);
#pragma unroll
      for (int j = 0; j < BPT; ++j) {
        const int b = threadIdx.x + j * blockDim.x;
        hs[j][0] = hs[j][1] = 0.0f;
        if (b < KB) {
          hs[j][0] = __ldg(a.hscale + (size_t)(2 * b) * a.R + r0);
          hs[j][1] = __ldg(a.hscale + (size_t)(2 * b + 1) * a.R + r0);
        }
      }
    }
    float acc[32];
#pragma unroll
    for (int st = 0; st < SPI; ++st) {
      const int slot = cons_v % kRing;
      if (!mbar_wait(&bars[slot], (uint32_t)(cons_v / kRing) & 1u)) {
        if (threadIdx.x == 0) atomicOr(a.status, kStatusWaitTimeout);
        return;
      }
      const uint8_t* stg = smem + (size_t)slot * stage_bytes;
#pragma unroll
      for (int rr = 0; rr < RPS; ++rr) {
        float v = 0.f;
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          const int b = threadIdx.x + j * blockDim.x;
          if (b < KB) {
            const uint4 w = *reinterpret_cast<const uint4*>(stg + rr * qrow + b * 16);
            const float sc = e8m0_to_f32(stg[cbytes + rr * srow + b]);
            float p0, p1;
            dot_block_halves(w, xr[j], p0, p1);
            if (kGateUp) v = fmaf(p0 + p1, sc, v);
            else v = fmaf(fmaf(p1, hs[j][1], p0 * hs[j][0]), sc, v);
          }
        }
        acc[st * RPS + rr] = v;
      }
      ++cons_v;
      __syncthreads();                          // every thread is done with this slot
      if (threadIdx.x == 0 && prod.item < items) {
        fence_proxy_async_smem();
        issue(prod.item, prod.stage, prod_v % kRing);
        ++prod_v;
        advance(prod);
      }
    }
    const float s = cta_row_sums(acc, red);
    if (warp == 0) {
      if (kGateUp) {
        // lanes 0..15: gate row tile*16+lane; lanes 16..31: up row
        const float xs = __ldg(a.xscale + tok);
        const float u = __shfl_down_sync(0xFFFFFFFFu, s, 16);
        const float h = silu_f32(s * xs) * (u * xs);
        float m = (lane < 16) ? fabsf(h) : 0.0f;
#pragma unroll
        for (int off = 8; off >= 1; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
        float scale = 1.0f, inv = 1.0f;
        if (m > 0.0f && isfinite(m)) {
          int ex;
          frexpf(m, &ex);
          ex = max(-100, min(127, ex));
          scale = ldexpf(1.0f, ex - 15);
          inv = ldexpf(1.0f, 15 - ex);
        }
        if (lane < 16) a.h16_out[(size_t)r0 * a.I + tile * 16 + lane] = __float2half_rn(h * inv);
        if (lane == 0) a.hscale_out[(size_t)tile * a.R + r0] = scale;
      } else {
        a.y_perm[(size_t)r0 * a.W + tile * 32 + lane] = s;
      }
    }
    __syncthreads();
  }
}

size_t fma_stage_bytes(int K, int rps) {
  const size_t c = (size_t)rps * (K / 2), s = (size_t)rps * (K / 32);
  return (c + s + 127) / 128 * 128;
}
size_t fma_smem_bytes(int K, int rps) { return kRing * fma_stage_bytes(K, rps); }

#define MOE_FMA_INST(BPT, RPS)                                    \
  template __global__ void k_fma_gemv<BPT, RPS, true>(FmaArgs);  \
  template __global__ void k_fma_gemv<BPT, RPS, false>(FmaArgs);
MOE_FMA_INST(1, 1) MOE_FMA_INST(1, 2) MOE_FMA_INST(1, 4) MOE_FMA_INST(1, 8) MOE_FMA_INST(1, 16)
MOE_FMA_INST(2, 1) MOE_FMA_INST(2, 2) MOE_FMA_INST(2, 4) MOE_FMA_INST(2, 8) MOE_FMA_INST(2, 16)
#undef MOE_FMA_INST

}  // namespace moe
