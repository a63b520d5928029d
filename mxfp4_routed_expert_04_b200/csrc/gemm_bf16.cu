// Dense bf16 GEMMs on tcgen05 (kind::f16, fp32 accumulation in tensor memory):
// the router logits (rabbit README, model table row "MoE routing") and the
// always-applied gated shared expert (rabbit README, the same row),
// for any number of tokens.
//
// Orientation as in the MXFP4 GEMM: the MMA's M side is 128 weight rows, its
// N side a tile of N tokens (16..128), K the reduction in stages of 64
// elements (rows of 128 bytes, 128-byte swizzle, loaded by TMA). Each stage
// carries two 128-row weight tiles that share the token tile, so two
// accumulation chains keep the tensor pipe busy; with one or two tokens the
// tensor pipe idles and the kernel is a TMA weight stream. Modes:
//   kPlain   C[s, t, col] = sum over split s of K of W[m, k] x[t, k] (fp32
//            out) for up to three weight matrices ("segments") stacked along
//            the output columns; with two passes the token operand is a hi/lo
//            bf16 pair of one fp32 operand, both halves sit in the same stage
//            and accumulate into the same chain, so the weights stream once
//   kSwiGLU  the two tiles are the same rows of Wg and Wu; the epilogue
//            writes h = silu(g) * u as a bf16 hi/lo pair (hi = bf16(h),
//            lo = bf16(h - hi)) for the shared down projection
// Roles and bounded waits as in the MXFP4 GEMM (warp 0 TMA, warp 1 MMA,
// warps 2-5 epilogue; double-buffered accumulators).
#include <math.h>

#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

constexpr int kTileBytes = 128 * 128;           // 128 rows x 64 bf16
constexpr int kMaxStages = 8;
constexpr int kThreads = 192;

// kind::f16 with bf16 A and B, fp32 D, M = 128, both K-major
MOE_DEV uint32_t idesc_bf16(int N) {
  return (1u << 4) | (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | ((128u >> 4) << 24);
}

MOE_DEV void mma_bf16_tc(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                         uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %4, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, {%5, %5, %5, %5}, p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate), "r"(0u)
      : "memory");
}

struct Work {
  int seg;      // weight segment
  int m0;       // first row of the first tile within the segment
  int rows;     // rows of the segment
  int col0;     // first output column of the segment
  int n0;       // first token
  int split;    // K split
  bool two;     // a second 128-row tile follows the first
};

// TMEM columns: two buffers x two chains x N, a power of two >= 32
MOE_DEV uint32_t tmem_cols_for(int N) {
  uint32_t c = 32;
  while (c < 4u * (uint32_t)N) c <<= 1;
  return c;
}

}  // namespace

__global__ void __launch_bounds__(kThreads, 1) k_bf16_gemm(const __grid_constant__ Bf16GemmArgs a) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  const int N = a.N;
  const int nst = bf16_stages(N, a.passes);
  const int stage_bytes = bf16_stage_bytes(N, a.passes);
  const int btile = N * 128;                  // one token tile of one pass
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + nst * stage_bytes);
  uint64_t* empty = full + kMaxStages;
  uint64_t* acc_full = empty + kMaxStages;    // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const bool swiglu = a.mode == kBf16SwiGLU;
  const uint32_t tmem_cols = tmem_cols_for(N);
  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(&acc_full[b], 1);
      mbar_init(&acc_empty[b], 4);
    }
    mbar_init(drain, 1);
    *abort = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    for (int i = 0; i < 3; ++i)
      if (a.seg_rows[i] > 0 || (swiglu && i == 1)) tc::prefetch_map(&a.map_a[i]);
    tc::prefetch_map(&a.map_b0);
    if (a.passes > 1) tc::prefetch_map(&a.map_b1);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, tmem_cols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;

  // weight units: SwiGLU one 128-row tile of Wg and Wu; plain up to two
  // consecutive 128-row tiles of one segment
  int U[3];
  for (int i = 0; i < 3; ++i)
    U[i] = swiglu ? (i == 0 ? a.seg_rows[0] / 128 : 0) : (a.seg_rows[i] + 255) / 256;
  const int NTt = (a.T + N - 1) / N;
  const long per_split = (long)(U[0] + U[1] + U[2]) * NTt;
  const long items = per_split * a.S;
  const int ks_stages = a.K / a.S / 64;                        // stages of one split
  auto work_of = [&](long q) {
    Work w;
    w.split = (int)(q / per_split);
    const long r = q - (long)w.split * per_split;
    int u = (int)(r / NTt);
    w.n0 = (int)(r - (long)u * NTt) * N;
    w.seg = 0;
    w.col0 = 0;
    while (w.seg < 2 && u >= U[w.seg]) {
      u -= U[w.seg];
      w.col0 += a.seg_rows[w.seg];
      ++w.seg;
    }
    w.rows = a.seg_rows[swiglu ? 0 : w.seg];
    w.m0 = u * (swiglu ? 128 : 256);
    w.two = swiglu || w.m0 + 128 < w.rows;
    return w;
  };

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t last_ph[kMaxStages];
      bool filled[kMaxStages];
#pragma unroll
      for (int s = 0; s < kMaxStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long q = blockIdx.x; q < items && ok; q += gridDim.x) {
        const Work w = work_of(q);
        const CUtensorMap* m0 = &a.map_a[w.seg];
        const CUtensorMap* m1 = swiglu ? &a.map_a[1] : m0;
        const int r1 = swiglu ? w.m0 : w.m0 + 128;
        for (int j = 0; j < ks_stages; ++j) {
          if (!tc::wait_or_abort(&empty[s], ph ^ 1u, abort)) { ok = false; break; }
          uint8_t* st = smem + s * stage_bytes;
          const int x = (w.split * ks_stages + j) * 64;
          mbar_expect_tx(&full[s], (w.two ? 2 : 1) * kTileBytes + a.passes * btile);
          tc::tma_load_2d(st, m0, x, w.m0, &full[s]);
          if (w.two) tc::tma_load_2d(st + kTileBytes, m1, x, r1, &full[s]);
          tc::tma_load_2d(st + 2 * kTileBytes, &a.map_b0, x, w.n0, &full[s]);
          if (a.passes > 1) tc::tma_load_2d(st + 2 * kTileBytes + btile, &a.map_b1, x, w.n0, &full[s]);
          last_ph[s] = ph;
          filled[s] = true;
          if (++s == nst) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort) {
        for (int s2 = 0; s2 < nst; ++s2)
          if (filled[s2]) mbar_wait(&full[s2], last_ph[s2]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    const uint32_t idesc = idesc_bf16(N);
    int s = 0;
    uint32_t ph = 0;
    int n_it = 0;
    bool ok = true;
    for (long q = blockIdx.x; q < items && ok; q += gridDim.x, ++n_it) {
      const Work w = work_of(q);
      const int buf = n_it & 1;
      const uint32_t acc_ph = (uint32_t)((n_it >> 1) & 1);
      if (!tc::wait_or_abort(&acc_empty[buf], acc_ph ^ 1u, abort)) break;
      tc::fence_after_sync();
      const uint32_t d0 = tbase + 2u * N * buf, d1 = d0 + N;
      for (int j = 0; j < ks_stages; ++j) {
        if (!tc::wait_or_abort(&full[s], ph, abort)) { ok = false; break; }
        tc::fence_after_sync();
        if (lane == 0) {
          const uint8_t* st = smem + s * stage_bytes;
          // descriptors of the stage's tiles, built once; a K block or the
          // second B tile only moves the 14-bit address field (16-byte units),
          // which cannot carry below 228 KB of shared memory
          const uint64_t da0 = tc::desc_sw128(smem_u32(st)), da1 = tc::desc_sw128(smem_u32(st + kTileBytes));
          const uint64_t db = tc::desc_sw128(smem_u32(st + 2 * kTileBytes));
          const uint32_t bstep = (uint32_t)btile >> 4;
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {                 // K = 16 per MMA: 32 bytes
            for (int p = 0; p < a.passes; ++p) {
              const uint32_t acc = (j > 0 || kb > 0 || p > 0) ? 1u : 0u;
              const uint64_t bdesc = db + p * bstep + 2u * kb;
              mma_bf16_tc(d0, da0 + 2u * kb, bdesc, idesc, acc);
              if (w.two) mma_bf16_tc(d1, da1 + 2u * kb, bdesc, idesc, acc);
            }
          }
          tc::commit(&empty[s]);
          if (j == ks_stages - 1) tc::commit(&acc_full[buf]);
        }
        __syncwarp();
        if (++s == nst) { s = 0; ph ^= 1u; }
      }
    }
    if (lane == 0) {
      tc::commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 2-5) ----------------
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    int n_it = 0;
    for (long q = blockIdx.x; q < items; q += gridDim.x, ++n_it) {
      const Work w = work_of(q);
      const int buf = n_it & 1;
      const uint32_t acc_ph = (uint32_t)((n_it >> 1) & 1);
      if (!tc::wait_or_abort(&acc_full[buf], acc_ph, abort)) break;
      tc::fence_after_sync();
      const uint32_t dcol = tbase + lane_off + 2u * N * buf;
      const int m = w.m0 + 32 * wq + lane;          // this lane's weight row (first tile)
      const int nmax = min(N, a.T - w.n0);
      for (int c0 = 0; c0 < N; c0 += 32) {
        uint32_t g[32], u[32];
        if (N - c0 >= 32) {
          tc::ld_32cols(dcol + c0, g);
          if (w.two) tc::ld_32cols(dcol + N + c0, u);
        } else {
          tc::ld_16cols(dcol + c0, g);
          if (w.two) tc::ld_16cols(dcol + N + c0, u);
        }
        tc::wait_ld();
        if (c0 + 32 >= N) {                         // accumulators read: the MMA may reuse them
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
        }
        const int nc = min(32, nmax - c0);
        if (swiglu) {
#pragma unroll
          for (int c = 0; c < 32; ++c) {
            if (c < nc) {
              const float h = silu_f32(__uint_as_float(g[c])) * __uint_as_float(u[c]);
              const uint32_t hi = f32_to_bf16_rne(h);
              const uint32_t lo = f32_to_bf16_rne(h - bf16_to_f32(hi));
              const size_t o = (size_t)(w.n0 + c0 + c) * w.rows + m;
              a.h_hi[o] = (uint16_t)hi;
              a.h_lo[o] = (uint16_t)lo;
            }
          }
        } else {
          // rows past the segment's end (a last tile of fewer than 128 rows) are not stored
          float* orow = a.out + ((size_t)w.split * a.T + w.n0 + c0) * a.ld + w.col0 + m;
          if (m < w.rows) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < nc) orow[(size_t)c * a.ld] = __uint_as_float(g[c]);
          }
          if (w.two && m + 128 < w.rows) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < nc) orow[(size_t)c * a.ld + 128] = __uint_as_float(u[c]);
          }
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
  if (warp == 1) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, tmem_cols);
  }
}

size_t bf16_gemm_smem_bytes(int N, int passes) {
  return 1024 + (size_t)bf16_stages(N, passes) * bf16_stage_bytes(N, passes) + 256;
}
int bf16_gemm_threads() { return kThreads; }

}  // namespace moe
