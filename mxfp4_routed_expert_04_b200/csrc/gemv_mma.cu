// Grouped MXFP4 GEMV for the routed experts that received 2 or more tokens
// (small decode batches) when W and I are multiples of 512: the "expert
// matmul" of the rabbit README phase breakdown, gate/up with the SwiGLU
// epilogue, then the down projection, every weight byte read once from HBM.
//
// Design (B200, memory-bound):
// * one CTA per SM, a producer warp and 16 consumer warps around a ring of
//   shared-memory stages; every stage is one 512-element K slice of a weight
//   row group: codes by 2-D tensor maps (128-byte swizzle, the layout
//   ldmatrix reads without bank conflicts), their E8M0 scales by 2-D tensor
//   maps, and the slice of every token's activation row by bulk copies;
// * ldmatrix.x4 hands every lane 8 E2M1 codes of one 32-element block for
//   rows g and g+8 of a 16-row tile, the A-fragment shape of mma.m16n8k16
//   with K permuted inside the block (the activation fragment takes the same
//   permutation), so one MMA pair covers one scale block and the E8M0 scale
//   is applied once per block to the fp32 MMA result;
// * activations are f16 with one power-of-two scale per row: x as the
//   dispatch writes it (exact for bf16 x), h converted from the fp32 rows of
//   the gate/up kernel by k_h_rowscale; the row scale is applied once, in the
//   epilogue;
// * work items (expert, row group) are numbered group-major, so that every
//   CTA's contiguous share mixes experts with many and few tokens (the MMA
//   work grows with the token count, the bytes do not).
#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

constexpr int kMgRows = 64;                          // weight rows per gate/up item and matrix
constexpr int kMgBox = kMgRows * 128;                // one code box (256 K elements)
constexpr int kMgCodes = 2 * kMgBox;                 // one matrix's codes of a stage (512 K)
constexpr int kMgScales = kMgRows * 16;              // one matrix's scales of a stage
constexpr int kXStride = 1088;                       // token row stride in a stage: 68 x 16 bytes, so the
                                                     // fragment loads of two tokens hit disjoint banks
constexpr int kMgXOff = 2 * kMgCodes + 2 * kMgScales;
constexpr int kTok = 16;                             // tokens per pass over the weights
constexpr int kNG = kTok / 8;                        // 8-token MMA column groups
constexpr int kMgStage = (kMgXOff + kTok * kXStride + 1023) / 1024 * 1024;
constexpr int kMgRed = 4 * 3 * 32 * (8 * kNG) * 4;   // K-quarter partial sums [tile][quarter-1][lane][16]

constexpr int kMdRows = 128;                         // weight rows per down item
constexpr int kMdBox = kMdRows * 128;
constexpr int kMdCodes = 2 * kMdBox;
constexpr int kMdScales = kMdRows * 16;
constexpr int kMdHOff = kMdCodes + kMdScales;
constexpr int kMdStage = (kMdHOff + kTok * kXStride + 1023) / 1024 * 1024;
constexpr int kMdRed = 8 * 32 * (4 * kNG) * 4;       // K-half partial sums [tile][lane][8]

static_assert(kMmaConsumers == 16, "the tile / K-split layout below assumes 16 consumer warps");

// The experts of the expert list with at least min_tokens tokens, in list
// order, into s_list; returns their count (every thread).
MOE_DEV int multi_token_experts(const int32_t* __restrict__ expert_list, const int32_t* __restrict__ offsets,
                                int min_tokens, int16_t* s_list, int* s_wsum) {
  constexpr int kWarps = kMmaConsumers + 1;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int n_act = __ldg(expert_list);
  int n_multi = 0;
  for (int base = 0; base < n_act; base += 32 * kWarps) {
    const int i = base + threadIdx.x;
    int e = -1;
    if (i < n_act) {
      e = __ldg(expert_list + 1 + i);
      if (__ldg(offsets + e + 1) - __ldg(offsets + e) < min_tokens) e = -1;
    }
    const unsigned m = __ballot_sync(0xFFFFFFFFu, e >= 0);
    if (lane == 0) s_wsum[warp] = __popc(m);
    __syncthreads();
    int before = n_multi;
    for (int w = 0; w < warp; ++w) before += s_wsum[w];
    if (e >= 0) s_list[before + __popc(m & ((1u << lane) - 1u))] = (int16_t)e;
    for (int w = 0; w < kWarps; ++w) n_multi += s_wsum[w];
    __syncthreads();
  }
  return n_multi;
}

// True when no byte of w is an E8M0 code 0 or 255 (the two codes whose
// value is not the plain power of two c << 23).
MOE_DEV bool e8m0_plain4(uint32_t w) { return (__vcmpeq4(w, 0u) | __vcmpeq4(w, 0xFFFFFFFFu)) == 0u; }

// Value of E8M0 code byte i of w: the exponent field alone on the plain path,
// else e8m0_to_f32 (2^-127 for code 0, NaN for 255).
template <int i>
MOE_DEV float e8m0_byte(uint32_t w, bool plain) {
  if (plain) return __uint_as_float((i < 3 ? (w << (23 - 8 * i)) : (w >> 1)) & 0x7F800000u);
  return e8m0_to_f32((w >> (8 * i)) & 0xFFu);
}

MOE_DEV void named_barrier(int id, int threads) {
  asm volatile("bar.sync %0, %1;\n" ::"r"(id), "r"(threads) : "memory");
}

}  // namespace

// ---------------------------------------------------------------------------
// gate/up + SwiGLU
// block 32 * (kMmaConsumers + 1), one CTA per SM, dynamic smem
// mma_gateup_smem_bytes(); item = (multi-token expert, 64-row group of I); a
// stage: gate and up codes (two 128-byte boxes x 64 rows each), their scales
// (16 bytes x 64 rows each), the slice of up to 16 token rows (f16).
// Consumer warp w takes the 16-row tile w % 4 over the K quarter w / 4 of
// every slice; the quarters are added through shared memory, in order, at
// the end of the item. Output: h = silu(Wg x) * (Wu x) as fp32 rows [R, I].
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * (kMmaConsumers + 1), 1) k_mma_gateup(const __grid_constant__ MmaGateUpArgs A) {
  pdl_wait();
  pdl_trigger();
  const GateUpArgs& a = A.g;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_red = reinterpret_cast<float*>(smem + kMmaStages * kMgStage);
  __shared__ int16_t s_list[1024];
  __shared__ int s_wsum[kMmaConsumers + 1];
  __shared__ uint64_t s_bars[2 * kMmaStages];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = a.W, I = a.I;

  const int n_multi = multi_token_experts(a.expert_list, a.offsets, a.min_tokens, s_list, s_wsum);
  const int groups = I / kMgRows;
  const long total = (long)n_multi * groups;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kMmaStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmaStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMmaConsumers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  const int nslice = W / 512;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      uint32_t last_ph[kMmaStages];
      bool filled[kMmaStages];
      for (int s = 0; s < kMmaStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      bool ok = true;
      for (long it = lo; it < hi && ok; ++it) {
        const int e = s_list[it % n_multi], rg = (int)(it / n_multi);
        const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
        const int wrow = e * I + rg * kMgRows;
        for (int c0 = 0; c0 < n_all && ok; c0 += kTok) {
          const int nt = min(kTok, n_all - c0);
          for (int s = 0; s < nslice; ++s) {
            if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) { ok = false; break; }
            uint8_t* st = smem + (size_t)slot * kMgStage;
            fence_proxy_async_smem();
            mbar_expect_tx(&full[slot], 2 * kMgCodes + 2 * kMgScales + nt * 1024);
            tc::tma_load_2d(st, &A.map_gq, s * 256, wrow, &full[slot]);
            tc::tma_load_2d(st + kMgBox, &A.map_gq, s * 256 + 128, wrow, &full[slot]);
            tc::tma_load_2d(st + kMgCodes, &A.map_uq, s * 256, wrow, &full[slot]);
            tc::tma_load_2d(st + kMgCodes + kMgBox, &A.map_uq, s * 256 + 128, wrow, &full[slot]);
            tc::tma_load_2d(st + 2 * kMgCodes, &A.map_gs, s * 16, wrow, &full[slot]);
            tc::tma_load_2d(st + 2 * kMgCodes + kMgScales, &A.map_us, s * 16, wrow, &full[slot]);
            for (int c = 0; c < nt; ++c)
              bulk_g2s(st + kMgXOff + c * kXStride, a.x16 + (size_t)__ldg(a.row_token + r0 + c0 + c) * W + s * 512,
                       1024u, &full[slot]);
            last_ph[slot] = ph;
            filled[slot] = true;
            if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
          }
        }
      }
      if (*abort) {
        for (int s = 0; s < kMmaStages; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int tt = w & 3, kq = w >> 2;                 // row tile, K quarter of the slice
    const int g = lane >> 2, t4 = lane & 3;
    const int lq = lane >> 3, lr = lane & 7;
    const int ldrow = 16 * tt + (lq & 1) * 8 + lr;     // smem row of this lane's ldmatrix address
    const int row_g = 16 * tt + g, row_g8 = row_g + 8;
    const uint32_t lda = (uint32_t)((kq >> 1) * kMgBox + ldrow * 128);
    int slot = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long it = lo; it < hi && ok; ++it) {
      const int e = s_list[it % n_multi], rg = (int)(it / n_multi);
      const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
      for (int c0 = 0; c0 < n_all; c0 += kTok) {
        const int n = min(kTok, n_all - c0);
        const int ng = (n + 7) >> 3;
        float accG[kNG][4], accU[kNG][4];
#pragma unroll
        for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
          for (int j = 0; j < 4; ++j) accG[gi][j] = accU[gi][j] = 0.0f;
        for (int s = 0; s < nslice; ++s) {
          if (!tc::wait_or_abort(&full[slot], ph, abort)) { ok = false; break; }
          const uint8_t* st = smem + (size_t)slot * kMgStage;
          const uint32_t gq = smem_u32(st) + lda, uq = gq + kMgCodes;
          // the scales of this warp's four blocks: bytes 4 kq .. 4 kq + 3 of rows g, g + 8
          const uint8_t* gsc = st + 2 * kMgCodes + 4 * kq;
          const uint8_t* usc = gsc + kMgScales;
          const uint32_t xs0 = smem_u32(st + kMgXOff);
#pragma unroll 1
          for (int bp = 0; bp < 2; ++bp) {
            const int b0 = 4 * kq + 2 * bp;                    // first block of the pair in the slice
            const int ch = (b0 & 7) + (lq >> 1);               // its 16-byte chunk in the box row
            const uint32_t sw = (uint32_t)((ch ^ (ldrow & 7)) << 4);
            uint32_t Rg[4], Ru[4];
            ldmatrix_x4(Rg, gq + sw);
            ldmatrix_x4(Ru, uq + sw);
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
              const int b = b0 + hb;
              const int sb = 2 * bp + hb;                      // scale byte of the block
              const float sc[4] = {e8m0_to_f32(gsc[row_g * 16 + sb]), e8m0_to_f32(gsc[row_g8 * 16 + sb]),
                                   e8m0_to_f32(usc[row_g * 16 + sb]), e8m0_to_f32(usc[row_g8 * 16 + sb])};
              uint32_t ag0[4], ag1[4], au0[4], au1[4];
              decode_block(Rg[2 * hb], Rg[2 * hb + 1], ag0, ag1);
              decode_block(Ru[2 * hb], Ru[2 * hb + 1], au0, au1);
#pragma unroll
              for (int gi = 0; gi < kNG; ++gi) {
                if (gi < ng) {
                  // columns past n read stale rows of the stage: they only
                  // reach accumulator columns that are never stored
                  const uint4 xv = lds16(xs0 + (gi * 8 + g) * kXStride + (32 * b + 8 * t4) * 2);
                  float cg[4] = {0.f, 0.f, 0.f, 0.f}, cu[4] = {0.f, 0.f, 0.f, 0.f};
                  mma_f16(cg, ag0, xv.x, xv.y);
                  mma_f16(cu, au0, xv.x, xv.y);
                  mma_f16(cg, ag1, xv.z, xv.w);
                  mma_f16(cu, au1, xv.z, xv.w);
                  accG[gi][0] = fmaf(cg[0], sc[0], accG[gi][0]);
                  accG[gi][1] = fmaf(cg[1], sc[0], accG[gi][1]);
                  accG[gi][2] = fmaf(cg[2], sc[1], accG[gi][2]);
                  accG[gi][3] = fmaf(cg[3], sc[1], accG[gi][3]);
                  accU[gi][0] = fmaf(cu[0], sc[2], accU[gi][0]);
                  accU[gi][1] = fmaf(cu[1], sc[2], accU[gi][1]);
                  accU[gi][2] = fmaf(cu[2], sc[3], accU[gi][2]);
                  accU[gi][3] = fmaf(cu[3], sc[3], accU[gi][3]);
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&empty[slot]);
          if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        // the K quarters of tile tt: quarters 1..3 hand their sums to quarter 0
        float* red = s_red + (size_t)(tt * 3) * 32 * (8 * kNG) + lane * (8 * kNG);
        if (kq > 0) {
          float* mine = red + (size_t)(kq - 1) * 32 * (8 * kNG);
#pragma unroll
          for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
            for (int j = 0; j < 4; ++j) { mine[gi * 4 + j] = accG[gi][j]; mine[4 * kNG + gi * 4 + j] = accU[gi][j]; }
        }
        named_barrier(1 + tt, 128);
        if (kq == 0) {
#pragma unroll
          for (int q = 0; q < 3; ++q) {
            const float* o = red + (size_t)q * 32 * (8 * kNG);
#pragma unroll
            for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
              for (int j = 0; j < 4; ++j) { accG[gi][j] += o[gi * 4 + j]; accU[gi][j] += o[4 * kNG + gi * 4 + j]; }
          }
          // epilogue: h = silu(G) * U with the token's row scale, fp32 rows
#pragma unroll
          for (int gi = 0; gi < kNG; ++gi) {
            if (gi < ng) {
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int col = gi * 8 + 2 * t4 + c;
                if (col < n) {
                  const float xs = __ldg(a.xscale + __ldg(a.row_token + r0 + c0 + col));
                  float* hrow = A.h32 + (size_t)(r0 + c0 + col) * I + rg * kMgRows + 16 * tt + g;
                  hrow[0] = silu_f32(accG[gi][c] * xs) * (accU[gi][c] * xs);
                  hrow[8] = silu_f32(accG[gi][2 + c] * xs) * (accU[gi][2 + c] * xs);
                }
              }
            }
          }
        }
        named_barrier(1 + tt, 128);                     // red free again
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(A.status, kStatusWaitTimeout);
}

size_t mma_gateup_smem_bytes() { return 1024 + (size_t)kMmaStages * kMgStage + kMgRed; }

// ---------------------------------------------------------------------------
// h rows of the experts with >= min_tokens tokens: fp32 -> f16 with one
// power-of-two scale per row (the row's largest magnitude mapped into
// [2^14, 2^15), so every f16 carries 11 significant bits); the scale goes to
// hrs[row]. block 256 (a warp per row), grid-stride over the R rows.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(256) k_h_rowscale(const float* __restrict__ h32,
                                                    const int32_t* __restrict__ offsets, int E, int R,
                                                    int I, int min_tokens, __half* __restrict__ h16,
                                                    float* __restrict__ hrs) {
  pdl_wait();
  pdl_trigger();
  __shared__ int s_off[1025];                             // offsets[0..E], E <= 1024
  for (int i = threadIdx.x; i <= E; i += blockDim.x) s_off[i] = __ldg(offsets + i);
  __syncthreads();
  const int lane = threadIdx.x & 31;
  for (int r = blockIdx.x * 8 + (threadIdx.x >> 5); r < R; r += gridDim.x * 8) {
    // the expert of row r: offsets[e] <= r < offsets[e + 1]
    int lo = 0, hi = E;
    while (hi - lo > 1) {
      const int mid = (lo + hi) >> 1;
      if (s_off[mid] <= r) lo = mid; else hi = mid;
    }
    if (s_off[lo + 1] - s_off[lo] < min_tokens) continue;
    const float4* src = reinterpret_cast<const float4*>(h32 + (size_t)r * I);
    float m = 0.0f;
    for (int i = lane; i < I / 4; i += 32) {
      const float4 v = __ldcg(src + i);
      m = fmaxf(m, fmaxf(fmaxf(fabsf(v.x), fabsf(v.y)), fmaxf(fabsf(v.z), fabsf(v.w))));
    }
#pragma unroll
    for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
    float sc, inv;
    f16_block_scale(m, sc, inv);
    uint2* dst = reinterpret_cast<uint2*>(h16 + (size_t)r * I);
    for (int i = lane; i < I / 4; i += 32) {
      const float4 v = __ldcg(src + i);
      const __half2 p0 = __floats2half2_rn(v.x * inv, v.y * inv);
      const __half2 p1 = __floats2half2_rn(v.z * inv, v.w * inv);
      dst[i] = make_uint2(*reinterpret_cast<const uint32_t*>(&p0), *reinterpret_cast<const uint32_t*>(&p1));
    }
    if (lane == 0) hrs[r] = sc;
  }
}

// ---------------------------------------------------------------------------
// down projection
// block 32 * (kMmaConsumers + 1), one CTA per SM; item = (multi-token expert,
// 128-row group of W); a stage: the down codes (two 128-byte boxes x 128
// rows), their scales (16 bytes x 128 rows), the slice of up to 16 token h
// rows (f16). Consumer warp w takes the 16-row tile w % 8 over the K half
// w / 8 of every slice (one code box); the halves are added through shared
// memory at the end of the item, then scaled by the h row scale.
// ---------------------------------------------------------------------------
__global__ void __launch_bounds__(32 * (kMmaConsumers + 1), 1) k_mma_down(const __grid_constant__ MmaDownArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* s_red = reinterpret_cast<float*>(smem + kMmaStages * kMdStage);
  __shared__ int16_t s_list[1024];
  __shared__ int s_wsum[kMmaConsumers + 1];
  __shared__ uint64_t s_bars[2 * kMmaStages];
  __shared__ int s_abort;
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int W = a.W, I = a.I;

  const int n_multi = multi_token_experts(a.expert_list, a.offsets, a.min_tokens, s_list, s_wsum);
  const int groups = W / kMdRows;
  const long total = (long)n_multi * groups;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;
  uint64_t* full = s_bars;
  uint64_t* empty = s_bars + kMmaStages;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kMmaStages; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], kMmaConsumers);
    }
    s_abort = 0;
    fence_mbar_init();
  }
  __syncthreads();
  volatile int* abort = &s_abort;
  const int nslice = I / 512;

  if (warp == 0) {
    // ---------------- producer ----------------
    if (lane == 0) {
      int slot = 0;
      uint32_t ph = 0;
      uint32_t last_ph[kMmaStages];
      bool filled[kMmaStages];
      for (int s = 0; s < kMmaStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      bool ok = true;
      for (long it = lo; it < hi && ok; ++it) {
        const int e = s_list[it % n_multi], rg = (int)(it / n_multi);
        const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
        const int wrow = e * W + rg * kMdRows;
        for (int c0 = 0; c0 < n_all && ok; c0 += kTok) {
          const int nt = min(kTok, n_all - c0);
          for (int s = 0; s < nslice; ++s) {
            if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) { ok = false; break; }
            uint8_t* st = smem + (size_t)slot * kMdStage;
            fence_proxy_async_smem();
            mbar_expect_tx(&full[slot], kMdCodes + kMdScales + nt * 1024);
            tc::tma_load_2d(st, &a.map_dq, s * 256, wrow, &full[slot]);
            tc::tma_load_2d(st + kMdBox, &a.map_dq, s * 256 + 128, wrow, &full[slot]);
            tc::tma_load_2d(st + kMdCodes, &a.map_ds, s * 16, wrow, &full[slot]);
            for (int c = 0; c < nt; ++c)
              bulk_g2s(st + kMdHOff + c * kXStride, a.h16 + (size_t)(r0 + c0 + c) * I + s * 512, 1024u,
                       &full[slot]);
            last_ph[slot] = ph;
            filled[slot] = true;
            if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
          }
        }
      }
      if (*abort) {
        for (int s = 0; s < kMmaStages; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int tt = w & 7, kh = w >> 3;                  // row tile, K half (code box) of the slice
    const int g = lane >> 2, t4 = lane & 3;
    const int lq = lane >> 3, lr = lane & 7;
    const int ldrow = 16 * tt + (lq & 1) * 8 + lr;
    const int row_g = 16 * tt + g, row_g8 = row_g + 8;
    const uint32_t lda = (uint32_t)(kh * kMdBox + ldrow * 128);
    int slot = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long it = lo; it < hi && ok; ++it) {
      const int e = s_list[it % n_multi], rg = (int)(it / n_multi);
      const int r0 = __ldg(a.offsets + e), n_all = __ldg(a.offsets + e + 1) - r0;
      for (int c0 = 0; c0 < n_all; c0 += kTok) {
        const int n = min(kTok, n_all - c0);
        const int ng = (n + 7) >> 3;
        float acc[kNG][4];
#pragma unroll
        for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
          for (int j = 0; j < 4; ++j) acc[gi][j] = 0.0f;
        for (int s = 0; s < nslice; ++s) {
          if (!tc::wait_or_abort(&full[slot], ph, abort)) { ok = false; break; }
          const uint8_t* st = smem + (size_t)slot * kMdStage;
          const uint32_t cq = smem_u32(st) + lda;
          // the scales of this warp's eight blocks: bytes 8 kh .. 8 kh + 7 of rows g, g + 8
          const uint8_t* wsc = st + kMdCodes + 8 * kh;
          const uint2 w0 = *reinterpret_cast<const uint2*>(wsc + row_g * 16);
          const uint2 w8 = *reinterpret_cast<const uint2*>(wsc + row_g8 * 16);
          const bool plain = __all_sync(0xFFFFFFFFu, e8m0_plain4(w0.x) && e8m0_plain4(w0.y) &&
                                                         e8m0_plain4(w8.x) && e8m0_plain4(w8.y));
          const uint32_t hs0 = smem_u32(st + kMdHOff);
#pragma unroll 2
          for (int bp = 0; bp < 4; ++bp) {
            uint32_t R[4];
            const int ch = 2 * bp + (lq >> 1);
            ldmatrix_x4(R, cq + ((ch ^ (ldrow & 7)) << 4));
            const uint32_t s0 = (bp < 2) ? w0.x : w0.y, s8 = (bp < 2) ? w8.x : w8.y;
            float sc[2][2];                                   // [block][row g, row g+8]
            if (bp & 1) {
              sc[0][0] = e8m0_byte<2>(s0, plain); sc[0][1] = e8m0_byte<2>(s8, plain);
              sc[1][0] = e8m0_byte<3>(s0, plain); sc[1][1] = e8m0_byte<3>(s8, plain);
            } else {
              sc[0][0] = e8m0_byte<0>(s0, plain); sc[0][1] = e8m0_byte<0>(s8, plain);
              sc[1][0] = e8m0_byte<1>(s0, plain); sc[1][1] = e8m0_byte<1>(s8, plain);
            }
#pragma unroll
            for (int hb = 0; hb < 2; ++hb) {
              const int b = 8 * kh + 2 * bp + hb;                 // block in the slice
              uint32_t a0[4], a1[4];
              decode_block(R[2 * hb], R[2 * hb + 1], a0, a1);
#pragma unroll
              for (int gi = 0; gi < kNG; ++gi) {
                if (gi < ng) {
                  // columns past n read stale rows of the stage (never stored)
                  const uint4 hv = lds16(hs0 + (gi * 8 + g) * kXStride + (32 * b + 8 * t4) * 2);
                  float c[4] = {0.f, 0.f, 0.f, 0.f};
                  mma_f16(c, a0, hv.x, hv.y);
                  mma_f16(c, a1, hv.z, hv.w);
                  acc[gi][0] = fmaf(c[0], sc[hb][0], acc[gi][0]);
                  acc[gi][1] = fmaf(c[1], sc[hb][0], acc[gi][1]);
                  acc[gi][2] = fmaf(c[2], sc[hb][1], acc[gi][2]);
                  acc[gi][3] = fmaf(c[3], sc[hb][1], acc[gi][3]);
                }
              }
            }
          }
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&empty[slot]);
          if (++slot == kMmaStages) { slot = 0; ph ^= 1u; }
        }
        if (!ok) break;
        // K half 1 hands its sums to half 0, which scales by the h row scale
        float* red = s_red + (size_t)(tt * 32 + lane) * (4 * kNG);
        if (kh == 1) {
#pragma unroll
          for (int gi = 0; gi < kNG; ++gi)
#pragma unroll
            for (int j = 0; j < 4; ++j) red[gi * 4 + j] = acc[gi][j];
        }
        named_barrier(1 + tt, 64);
        if (kh == 0) {
          const int n0 = rg * kMdRows + 16 * tt + g;      // output column (row of Wd) of fragment row g
#pragma unroll
          for (int gi = 0; gi < kNG; ++gi) {
            if (gi < ng) {
#pragma unroll
              for (int c = 0; c < 2; ++c) {
                const int col = gi * 8 + 2 * t4 + c;
                if (col < n) {
                  const size_t r = (size_t)(r0 + c0 + col);
                  const float hs = __ldg(a.hrs + r);
                  float* yrow = a.y_perm + r * W + n0;
                  yrow[0] = (acc[gi][c] + red[gi * 4 + c]) * hs;
                  yrow[8] = (acc[gi][2 + c] + red[gi * 4 + 2 + c]) * hs;
                }
              }
            }
          }
        }
        named_barrier(1 + tt, 64);                      // red free again
      }
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
}

size_t mma_down_smem_bytes() { return 1024 + (size_t)kMmaStages * kMdStage + kMdRed; }

}  // namespace moe
