// bf16 GEMV for a single token: the router logits and the sigmoid-gate logit
// (rabbit README, model table row "MoE routing", with its gated shared expert),
// the latent down-projection rows, and the shared expert's SwiGLU and down
// projection.
//
// One CTA per SM streams a contiguous range of weight rows, so no partial sums
// leave the CTA (no split-K across SMs):
//
// * rows go in groups of one stage's slots (1..16, from the rows per CTA;
//   plain: consecutive rows of one segment, up to three matrices stacked
//   along the output; SwiGLU: gate rows i.. in the first half of the slots,
//   up rows i.. in the second, read as MMA rows 0.. and 8..); a ring stage
//   holds one K chunk of the group's rows (about 64 KB, so few rows per CTA
//   come in one stage), each row by its own bulk copy into a slot 16 bytes
//   longer than the chunk, which makes the ldmatrix reads conflict-free; MMA
//   rows beyond the slots read a slot again and are never stored;
// * the dot products run on the tensor cores (mma.m16n8k16, bf16 x bf16 ->
//   fp32): A = 16 weight rows from ldmatrix, B = the activation in every
//   column (only column 0 is kept), 16 consumer warps each over 1/16 of the
//   chunk; the activation sits in shared memory as bf16 (x), or as a bf16
//   hi/lo pair (fp32 x: two MMAs, about 16 significant bits);
// * at the end of a group every warp leaves its 16 row sums in shared memory
//   and, behind one barrier of the consumer warps, warp w adds the 16 parts of
//   output row w in warp order (fixed, so the sums are reproducible) and
//   writes it: plain -> out[s][row]; SwiGLU -> h[i] = silu(g_i) * u_i; for the
//   shared down projection of one token the plain mode can instead finish the
//   layer's combine for the row (k <= 32 routed slots gathered by lanes,
//   summed in slot order, then the gated shared term, as in k_combine).
// Every wait is bounded as in the other streaming kernels.
#include "common.cuh"
#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

MOE_DEV void consumer_barrier() { asm volatile("bar.sync 1, %0;\n" ::"n"(32 * kRowsConsumers) : "memory"); }

}  // namespace

// block = 32 * (kRowsConsumers + 1) threads (warp 0: producer), one CTA per
// SM; dynamic shared memory = nst * rows_stage_bytes(K) + rows_act_bytes(K, kXF32)
template <bool kSwiGLU, bool kXF32>
__global__ void __launch_bounds__(32 * (kRowsConsumers + 1), 1) k_rows_bf16(RowsArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ uint64_t s_bars[2 * kRowsMaxStages];
  __shared__ int s_abort;
  __shared__ float s_red[2][kRowsConsumers][16];          // [group parity][warp][row of the group]
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const int K = a.K, SL = a.slots;
  const int KC = rows_chunk(K, SL);                       // K elements of a stage
  const int nkc = K / KC;                                 // stages of a group
  const uint32_t slot_bytes = (uint32_t)KC * 2 + 16;
  const uint32_t stage_bytes = (uint32_t)rows_stage_bytes(K, SL);
  const int nst = a.nst;
  uint8_t* act = smem + (size_t)nst * stage_bytes;
  // units: plain -> rows of the stacked segments; SwiGLU -> row pairs (gate i, up i)
  const int G = kSwiGLU ? SL / 2 : SL;                    // units of a group
  const int U0 = a.rows[0], U1 = kSwiGLU ? 0 : a.rows[1], U2 = kSwiGLU ? 0 : a.rows[2];
  const long total = (long)U0 + U1 + U2;
  const long lo = total * blockIdx.x / gridDim.x, hi = total * (blockIdx.x + 1) / gridDim.x;
  if (lo >= hi) return;                                   // uniform across the CTA
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
  // the cursor (segment, row in it) of unit lo; a group takes at most G
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
      bool ok = true;
      for (long u = lo; u < hi && ok;) {
        const int n = (int)min((long)min(G, seg_units(seg) - r), hi - u);
        for (int kc = 0; kc < nkc; ++kc) {
          if (!tc::wait_or_abort(&empty[slot], ph ^ 1u, abort)) { ok = false; break; }
          uint8_t* st = smem + (size_t)slot * stage_bytes;
          const uint32_t cb = (uint32_t)KC * 2;
          fence_proxy_async_smem();          // the consumers' reads of the slot come first
          mbar_expect_tx(&full[slot], (kSwiGLU ? 2u : 1u) * (uint32_t)n * cb);
          for (int i = 0; i < n; ++i) {
            if (kSwiGLU) {
              bulk_g2s(st + i * slot_bytes, a.w[0] + (size_t)(r + i) * K + kc * KC, cb, &full[slot]);
              bulk_g2s(st + (G + i) * slot_bytes, a.w[1] + (size_t)(r + i) * K + kc * KC, cb, &full[slot]);
            } else {
              bulk_g2s(st + i * slot_bytes, a.w[seg] + (size_t)(r + i) * K + kc * KC, cb, &full[slot]);
            }
          }
          last_ph[slot] = ph;
          filled[slot] = true;
          if (++slot == nst) { slot = 0; ph ^= 1u; }
        }
        u += n;
        r += n;
        while (seg < 2 && r == seg_units(seg)) { r = 0; ++seg; }   // skips empty segments
      }
      if (*abort) {     // let every issued copy land before the CTA can exit
        for (int s = 0; s < nst; ++s)
          if (filled[s]) mbar_wait(&full[s], last_ph[s]);
      }
    }
  } else {
    // ---------------- consumers ----------------
    const int w = warp - 1;
    const int g = lane >> 2, t4 = lane & 3;
    // the activation into shared memory, 8 elements per thread and step:
    // bf16 x as is; fp32 x as hi = bf16(x), lo = bf16(x - hi)
    {
      const int tid = threadIdx.x - 32;
      for (int i = tid; i < K / 8; i += 32 * kRowsConsumers) {
        if (kXF32) {
          const float4* xp = reinterpret_cast<const float4*>(static_cast<const float*>(a.x)) + 2 * i;
          const float4 v0 = __ldg(xp), v1 = __ldg(xp + 1);
          const float v[8] = {v0.x, v0.y, v0.z, v0.w, v1.x, v1.y, v1.z, v1.w};
          uint32_t hi2[4], lo2[4];
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const uint32_t h0 = f32_to_bf16_rne(v[2 * j]), h1 = f32_to_bf16_rne(v[2 * j + 1]);
            const uint32_t l0 = f32_to_bf16_rne(v[2 * j] - bf16_to_f32(h0));
            const uint32_t l1 = f32_to_bf16_rne(v[2 * j + 1] - bf16_to_f32(h1));
            hi2[j] = h0 | (h1 << 16);
            lo2[j] = l0 | (l1 << 16);
          }
          sts16(smem_u32(act) + 16u * i, make_uint4(hi2[0], hi2[1], hi2[2], hi2[3]));
          sts16(smem_u32(act) + (uint32_t)K * 2u + 16u * i, make_uint4(lo2[0], lo2[1], lo2[2], lo2[3]));
        } else {
          const uint4 v = __ldg(reinterpret_cast<const uint4*>(static_cast<const uint16_t*>(a.x)) + i);
          sts16(smem_u32(act) + 16u * i, v);
        }
      }
      consumer_barrier();
    }
    const int steps = KC / 16 / kRowsConsumers;          // k16 steps of a warp in a stage
    const int kw0 = w * (KC / kRowsConsumers);           // first element of the warp's part of a chunk
    // ldmatrix row / column of this lane: matrices (rows 0-7 | 8-15) x (k 0-7 | 8-15);
    // the slot holding MMA row m (rows past the group's slots read one again)
    const int mrow = (lane & 7) + 8 * ((lane >> 3) & 1), lcol = 8 * (lane >> 4);
    const int lrow = kSwiGLU ? (mrow < 8 ? mrow % G : G + (mrow - 8) % G) : mrow % SL;
    const uint32_t xa = smem_u32(act);
    // the combine's per-slot operands (lanes below k), the same for every row
    int sr = 0;
    float wj = 0.0f, gsig = 0.0f;
    if (!kSwiGLU && a.y) {
      if (lane < a.k) {
        sr = __ldg(a.slot_row + lane);
        wj = __ldg(a.topk_w + lane);
      }
      gsig = sigmoid_f32(__ldg(a.gate_logit));
    }
    int seg = seg0, slot = 0, gp = 0;
    int r = (int)r_lo;
    uint32_t ph = 0;
    bool ok = true;
    for (long u = lo; u < hi && ok;) {
      const int n = (int)min((long)min(G, seg_units(seg) - r), hi - u);
      // the routed values of output row w for the combine, loaded ahead of the group
      float v = 0.0f;
      if (!kSwiGLU && a.y && w < n && lane < a.k) v = __ldg(a.y_perm + (size_t)sr * a.rows[0] + r + w);
      // two accumulators (even and odd k16 steps; fp32 x: the hi and the lo
      // halves) halve the chain of dependent MMAs; added at the group's end
      float d[4] = {0.f, 0.f, 0.f, 0.f}, d2[4] = {0.f, 0.f, 0.f, 0.f};
      for (int kc = 0; kc < nkc; ++kc) {
        if (!tc::wait_or_abort(&full[slot], ph, abort)) { ok = false; break; }
        const uint32_t ab = smem_u32(smem + (size_t)slot * stage_bytes) + lrow * slot_bytes + (kw0 + lcol) * 2;
        const uint32_t xb = xa + (uint32_t)(kc * KC + kw0 + 2 * t4) * 2u;
        if (kXF32) {
          for (int s = 0; s < steps; ++s) {
            uint32_t A[4];
            ldmatrix_x4(A, ab + 32u * s);
            mma_bf16(d, A, lds32(xb + 32u * s), lds32(xb + 32u * s + 16u));
            mma_bf16(d2, A, lds32(xb + (uint32_t)K * 2u + 32u * s), lds32(xb + (uint32_t)K * 2u + 32u * s + 16u));
          }
        } else {
          for (int s = 0; s < steps; s += 2) {       // steps is even (KC >= 512)
            uint32_t A[4], B[4];
            ldmatrix_x4(A, ab + 32u * s);
            ldmatrix_x4(B, ab + 32u * s + 32u);
            mma_bf16(d, A, lds32(xb + 32u * s), lds32(xb + 32u * s + 16u));
            mma_bf16(d2, B, lds32(xb + 32u * s + 32u), lds32(xb + 32u * s + 48u));
          }
        }
        __syncwarp();
        if (lane == 0) tc::mbar_arrive(&empty[slot]);   // this warp is done with the slot
        if (++slot == nst) { slot = 0; ph ^= 1u; }
      }
      if (!ok) break;
      // every column of the fragment holds the same sums: rows g ([0]) and g + 8 ([2])
      if (t4 == 0) {
        s_red[gp][w][g] = d[0] + d2[0];
        s_red[gp][w][g + 8] = d[2] + d2[2];
      }
      consumer_barrier();
      if (w < n) {
        // output row w of the group: its 16 warp parts in warp order
        float sum = 0.0f, su = 0.0f;
#pragma unroll
        for (int j = 0; j < kRowsConsumers; ++j) {
          sum += s_red[gp][j][w];
          if (kSwiGLU) su += s_red[gp][j][w + 8];
        }
        const int row = r + w;
        if (kSwiGLU) {
          if (lane == 0) a.out[0][row] = silu_f32(sum) * su;
        } else if (a.y) {
          // the layer's combine for this output row, in the combine's own
          // order: routed slots j = 0.. (fma), then the gated shared term
          float acc = 0.0f;
          for (int j = 0; j < a.k; ++j)
            acc = fmaf(__shfl_sync(0xFFFFFFFFu, wj, j), __shfl_sync(0xFFFFFFFFu, v, j), acc);
          acc = fmaf(gsig, sum, acc);
          if (lane == 0) a.y[row] = acc;
        } else if (lane == 0) {
          a.out[seg][row] = sum;
        }
      }
      gp ^= 1;
      u += n;
      r += n;
      while (seg < 2 && r == seg_units(seg)) { r = 0; ++seg; }
    }
    if (!kSwiGLU && !kXF32 && a.x16 && blockIdx.x == 0) {
      // the activation operand from the row in shared memory: every warp
      // takes the largest |x| over the whole row (no barrier), then converts
      // its sixteenth of the row
      const uint32_t xs = smem_u32(act);
      float m = 0.0f;
      for (int i = lane; i < K / 8; i += 32) {
        const uint4 v = lds16(xs + 16u * i);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
        for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16_to_f32(wv[j] & 0xFFFFu)), fabsf(bf16_to_f32(wv[j] >> 16))));
      }
#pragma unroll
      for (int off = 16; off > 0; off >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, off));
      float scale, inv;
      f16_block_scale(m, scale, inv, kF16OpTop);
      for (int i = w * 32 + lane; i < K / 8; i += 32 * kRowsConsumers) {
        const uint4 v = lds16(xs + 16u * i);
        const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
        uint32_t o[4];
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const __half2 h = __floats2half2_rn(bf16_to_f32(wv[j] & 0xFFFFu) * inv, bf16_to_f32(wv[j] >> 16) * inv);
          o[j] = *reinterpret_cast<const uint32_t*>(&h);
        }
        *reinterpret_cast<uint4*>(a.x16 + 8 * i) = make_uint4(o[0], o[1], o[2], o[3]);
      }
      if (w == 0 && lane == 0) *a.xscale = scale;
    }
  }
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
}

template __global__ void k_rows_bf16<false, false>(RowsArgs);
template __global__ void k_rows_bf16<true, false>(RowsArgs);
template __global__ void k_rows_bf16<false, true>(RowsArgs);

// stages of the ring for reduction length K within the shared-memory budget
int rows_stages(int K, int slots, bool x_f32, size_t smem_budget) {
  const size_t sb = rows_stage_bytes(K, slots), ab = rows_act_bytes(K, x_f32);
  if (smem_budget < ab + 2 * sb) return 0;
  const size_t n = (smem_budget - ab) / sb;
  return (int)(n > kRowsMaxStages ? kRowsMaxStages : n);
}

}  // namespace moe
