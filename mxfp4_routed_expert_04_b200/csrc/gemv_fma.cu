// MXFP4 GEMV on the CUDA cores for experts that received exactly one token
// (every expert of a 1-token decode step; most experts of small batches).
//
// With one token a tensor-core MMA would use 1 of its 8 columns, and the
// legacy mma.sync rate of sm_100 then caps the kernel near half the HBM
// bandwidth. Design (one persistent, warp-specialised CTA per SM slot):
//
// * a producer warp streams the weights with bulk TMA copies
//   (cp.async.bulk: the packed codes of RPS consecutive rows plus their E8M0
//   codes per stage) into a ring of shared-memory slots guarded by full/empty
//   mbarriers, and the activation row of each work item (f16; for the down
//   projection also its per-16 scales) into a double buffer;
// * NT consumer threads: thread (rp, bt) owns BPT fixed 32-element K blocks
//   (kept in registers as f16) of row rp of every group of RP rows in a stage,
//   reads the matching 16-byte code slices (consecutive threads, consecutive
//   16 bytes), decodes with cvt.rn.f16x2.e2m1x2 (exact) and accumulates with
//   fma.rn.f32.f16 (exact f16 x f16 products, fp32 sums), applies the E8M0
//   block scale with one fp32 FMA, and writes one partial per row to shared
//   memory; consumers never wait on each other inside an item;
// * at the end of an item the consumers sum the partials of its 32 rows and
//   warp 0 runs the epilogue (SwiGLU + h quantisation, or the y_perm store).
//
// Every wait is bounded: on timeout the status word gets kStatusWaitTimeout,
// the CTA stops issuing copies and runs to its end without waiting again.
//
// Work items: gate/up = (active expert, 16-row tile of I): its 16 gate rows
// then its 16 up rows; down = (active expert, 32-row tile of W). The h made
// here is f16 with one power-of-two scale per group of 16 CONSECUTIVE
// intermediate rows (the tensor-core path uses interleaved groups; an
// expert's gate/up and down always take the same path).
#include "common.cuh"
#include "kernels.h"

namespace moe {

namespace {

constexpr int kItemRows = 32;         // weight rows per work item

// Dot product of one 32-element MXFP4 block with 32 f16 activations (block
// scale not applied); p0 / p1 = the two 16-element halves.
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

MOE_DEV void named_bar(int id, int nthreads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(nthreads) : "memory");
}

MOE_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

// next work item of this CTA whose expert received exactly one token
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
// block = NT consumer threads + 1 producer warp; persistent grid;
// dynamic shared memory laid out by FmaGeometry (see fma_geometry()).
// ---------------------------------------------------------------------------
template <int NT, int BPT, bool kGateUp>
__global__ void __launch_bounds__(NT + 32) k_fma_gemv(FmaArgs a, FmaGeometry g) {
  extern __shared__ __align__(128) uint8_t smem[];
  constexpr int NW = NT / 32;
  const int K = kGateUp ? a.W : a.I;
  const int KB = K >> 5;
  const size_t qrow = (size_t)K / 2, srow = (size_t)K / 32;
  const int tiles = kGateUp ? (a.I >> 4) : (a.W >> 5);
  const int items = __ldg(a.expert_list) * tiles;
  const int SPI = kItemRows / g.rps;

  uint8_t* ring = smem;
  uint8_t* xbuf = smem + g.off_x;
  float* part = reinterpret_cast<float*>(smem + g.off_part);     // [32][tpr]
  float* rsum = reinterpret_cast<float*>(smem + g.off_rsum);     // [32]
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + g.off_bar);
  uint64_t* empty = full + g.nslot;
  uint64_t* xfull = empty + g.nslot;
  uint64_t* xempty = xfull + 2;
  volatile int* abort_flag = reinterpret_cast<volatile int*>(xempty + 2);

  if (threadIdx.x == 0) {
    for (int i = 0; i < g.nslot; ++i) { mbar_init(&full[i], 1); mbar_init(&empty[i], NW); }
    for (int i = 0; i < 2; ++i) { mbar_init(&xfull[i], 1); mbar_init(&xempty[i], NW); }
    *abort_flag = 0;
    fence_mbar_init();
  }
  __syncthreads();

  auto timed_out = [&]() {
    *abort_flag = 1;
    atomicOr(a.status, kStatusWaitTimeout);
  };

  if (threadIdx.x >= NT) {
    // ------------------------------ producer ------------------------------
    if (threadIdx.x != NT) return;
    int v = 0, xi = 0;
    for (int item = next_single_item(a.expert_list, a.offsets, blockIdx.x, items, tiles); item < items;
         item = next_single_item(a.expert_list, a.offsets, item + gridDim.x, items, tiles), ++xi) {
      const int ai = item / tiles, tile = item - ai * tiles;
      const int e = __ldg(a.expert_list + 1 + ai);
      const int r0 = __ldg(a.offsets + e);
      const int p = xi & 1;
      if (xi >= 2 && (*abort_flag || !mbar_wait(&xempty[p], (uint32_t)((xi >> 1) - 1) & 1u))) {
        if (!*abort_flag) timed_out();
        return;
      }
      // the consumers' generic-proxy reads of this buffer (ordered by the
      // mbarrier) must precede the bulk copy's async-proxy writes
      fence_proxy_async_smem();
      uint8_t* xb = xbuf + p * g.x_bytes;
      if (kGateUp) {
        const int tok = __ldg(a.row_token + r0);
        mbar_expect_tx(&xfull[p], (uint32_t)(K * 2));
        bulk_g2s(xb, a.x16 + (size_t)tok * a.W, (uint32_t)(K * 2), &xfull[p]);
      } else {
        const uint32_t hb = (uint32_t)(K * 2), sb = (uint32_t)(K / 16 * 4);
        mbar_expect_tx(&xfull[p], hb + sb);
        bulk_g2s(xb, a.h16 + (size_t)r0 * a.I, hb, &xfull[p]);
        bulk_g2s(xb + hb, a.hscale + (size_t)r0 * (a.I >> 4), sb, &xfull[p]);
      }
      for (int st = 0; st < SPI; ++st, ++v) {
        const int slot = v % g.nslot;
        if (v >= g.nslot &&
            (*abort_flag || !mbar_wait(&empty[slot], (uint32_t)(v / g.nslot - 1) & 1u))) {
          if (!*abort_flag) timed_out();
          return;
        }
        fence_proxy_async_smem();
        size_t row;
        const uint8_t *q, *s;
        if (kGateUp) {
          const int r = st * g.rps;               // 0..31: gate rows then up rows
          row = (size_t)e * a.I + tile * 16 + (r & 15);
          q = (r < 16 ? a.wg_q : a.wu_q);
          s = (r < 16 ? a.wg_s : a.wu_s);
        } else {
          row = (size_t)e * a.W + tile * 32 + st * g.rps;
          q = a.wd_q;
          s = a.wd_s;
        }
        uint8_t* dst = ring + (size_t)slot * g.stage_bytes;
        const uint32_t cb = (uint32_t)(g.rps * qrow), sb = (uint32_t)(g.rps * srow);
        mbar_expect_tx(&full[slot], cb + sb);
        bulk_g2s(dst, q + row * qrow, cb, &full[slot]);
        bulk_g2s(dst + cb, s + row * srow, sb, &full[slot]);
      }
    }
    return;
  }

  // -------------------------------- consumers --------------------------------
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int rp = tid / g.tpr, bt = tid - rp * g.tpr;   // row slot, block slot
  const int RP = NT / g.tpr;                           // rows processed side by side
  const uint32_t cb = (uint32_t)(g.rps * qrow);
  int v = 0, xi = 0;
  for (int item = next_single_item(a.expert_list, a.offsets, blockIdx.x, items, tiles); item < items;
       item = next_single_item(a.expert_list, a.offsets, item + gridDim.x, items, tiles), ++xi) {
    const int ai = item / tiles, tile = item - ai * tiles;
    const int e = __ldg(a.expert_list + 1 + ai);
    const int r0 = __ldg(a.offsets + e);
    const int p = xi & 1;
    if (!*abort_flag && !mbar_wait(&xfull[p], (uint32_t)(xi >> 1) & 1u)) timed_out();
    const uint8_t* xb = xbuf + p * g.x_bytes;
    uint32_t xr[BPT][16];
    float hs[BPT][2];
#pragma unroll
    for (int j = 0; j < BPT; ++j) {
      const int b = bt + j * g.tpr;
      const bool ok = b < KB;
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        uint4 t = make_uint4(0u, 0u, 0u, 0u);
        if (ok) t = *reinterpret_cast<const uint4*>(xb + b * 64 + 16 * q);
        xr[j][4 * q] = t.x; xr[j][4 * q + 1] = t.y; xr[j][4 * q + 2] = t.z; xr[j][4 * q + 3] = t.w;
      }
      hs[j][0] = hs[j][1] = 0.0f;
      if (!kGateUp && ok) {
        const float* hsc = reinterpret_cast<const float*>(xb + K * 2);
        hs[j][0] = hsc[2 * b];
        hs[j][1] = hsc[2 * b + 1];
      }
    }
    __syncwarp();
    if (lane == 0) mbar_arrive(&xempty[p]);

    for (int st = 0; st < SPI; ++st, ++v) {
      const int slot = v % g.nslot;
      if (!*abort_flag && !mbar_wait(&full[slot], (uint32_t)(v / g.nslot) & 1u)) timed_out();
      const uint8_t* stg = ring + (size_t)slot * g.stage_bytes;
      for (int rr = rp; rr < g.rps; rr += RP) {
        float acc = 0.f;
#pragma unroll
        for (int j = 0; j < BPT; ++j) {
          const int b = bt + j * g.tpr;
          if (b < KB) {
            const uint4 w = *reinterpret_cast<const uint4*>(stg + rr * qrow + b * 16);
            const float sc = e8m0_to_f32(stg[cb + rr * srow + b]);
            float p0, p1;
            dot_block_halves(w, xr[j], p0, p1);
            if (kGateUp) acc = fmaf(p0 + p1, sc, acc);
            else acc = fmaf(fmaf(p1, hs[j][1], p0 * hs[j][0]), sc, acc);
          }
        }
        part[(st * g.rps + rr) * g.tpr + bt] = acc;
      }
      __syncwarp();
      if (lane == 0) mbar_arrive(&empty[slot]);
    }

    named_bar(1, NT);                                  // all partials of the item are in
    for (int row = warp; row < kItemRows; row += NW) {
      float s = 0.f;
      for (int i = lane; i < g.tpr; i += 32) s += part[row * g.tpr + i];
#pragma unroll
      for (int off = 16; off >= 1; off >>= 1) s += __shfl_xor_sync(0xFFFFFFFFu, s, off);
      if (lane == 0) rsum[row] = s;
    }
    named_bar(1, NT);
    if (warp == 0) {
      const float s = rsum[lane];
      if (kGateUp) {
        // lanes 0..15: gate row tile*16+lane; lanes 16..31: up row
        const float xs = __ldg(a.xscale + __ldg(a.row_token + r0));
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
        if (lane == 0) a.hscale_out[(size_t)r0 * (a.I >> 4) + tile] = scale;
      } else {
        a.y_perm[(size_t)r0 * a.W + tile * 32 + lane] = s;
      }
    }
    named_bar(1, NT);                                  // part / rsum free for the next item
  }
}

// Geometry of one launch for reduction length K (host side). A gate/up
// stage never spans the gate and up rows (at most 16 rows).
FmaGeometry fma_geometry(int K, bool gate_up, int nt, int bpt, size_t smem_budget,
                         size_t stage_target) {
  FmaGeometry g{};
  const int kb = K / 32;
  const int need = (kb + bpt - 1) / bpt;               // threads per row
  int tpr = 1;
  while (tpr < need) tpr *= 2;
  if (tpr > nt) return g;                              // ok == 0
  g.tpr = tpr;
  const int rp = nt / tpr;
  const size_t qrow = K / 2, srow = K / 32;
  // rows per stage: a power of two, multiple of rp, <= 32, codes >= stage_target,
  // E8M0 bytes a multiple of 16 (bulk-copy size rule)
  int rps = 0;
  for (int r = 1; r <= (gate_up ? 16 : kItemRows); r *= 2) {
    if (r % rp) continue;
    if ((r * srow) % 16) continue;
    rps = r;
    if ((size_t)r * qrow >= stage_target) break;
  }
  if (!rps) return g;
  g.rps = rps;
  g.stage_bytes = (uint32_t)((rps * (qrow + srow) + 127) / 128 * 128);
  g.x_bytes = (uint32_t)((K * 2 + (gate_up ? 0 : K / 16 * 4) + 127) / 128 * 128);
  const size_t fixed = 2 * (size_t)g.x_bytes + (size_t)kItemRows * tpr * 4 + kItemRows * 4 + 1024;
  int nslot = (int)((smem_budget - fixed) / g.stage_bytes);
  if (nslot < 2) return g;
  g.nslot = nslot > 32 ? 32 : nslot;
  g.off_x = (uint32_t)g.nslot * g.stage_bytes;
  g.off_part = g.off_x + 2 * g.x_bytes;
  g.off_rsum = g.off_part + (uint32_t)(kItemRows * tpr * 4);
  g.off_bar = (g.off_rsum + kItemRows * 4 + 15) / 16 * 16;
  g.smem_bytes = g.off_bar + (uint32_t)((2 * g.nslot + 4) * 8 + 16);
  g.ok = 1;
  return g;
}

#define MOE_FMA_INST(NT, BPT)                                                  \
  template __global__ void k_fma_gemv<NT, BPT, true>(FmaArgs, FmaGeometry);   \
  template __global__ void k_fma_gemv<NT, BPT, false>(FmaArgs, FmaGeometry);
MOE_FMA_INST(64, 1)
MOE_FMA_INST(256, 1)
MOE_FMA_INST(256, 2)
#undef MOE_FMA_INST

}  // namespace moe
