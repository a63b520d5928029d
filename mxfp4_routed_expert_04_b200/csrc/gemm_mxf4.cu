// Grouped block-scaled MXFP4 GEMM for experts with many tokens (prefill):
// 5th-generation tensor-core MMAs (tcgen05 kind::mxf4, E2M1 operands with one
// E8M0 scale per 32 elements of K) accumulating in tensor memory.
//
// The contraction is the routed expert of the rabbit README ("expert matmul"
// phase; model table row "MoE routing") with activations quantised to MXFP4
// like the weights (Kimi K3 page: "MXFP4 routed experts", read byte for byte).
//
// Orientation: the MMA's M side is 128 weight rows of one expert, its N side
// up to 128 of that expert's tokens, K the reduction. A "tile" is a run of at
// most 128 consecutive permuted rows of one expert (k_tile_list); an item is
// (m-tile, tile), and the persistent CTAs take items m-tile-major so that the
// several tiles of a hot expert read the same weight tile at about the same
// time (once from HBM, then from L2).
//
// Roles inside a CTA (256 threads, one CTA per SM):
//   warp 0     TMA producer: weight tiles, 128 rows x 128 bytes, 128-byte swizzle
//   warp 1     cp.async producer: the tokens' code rows (gathered through
//              row_token), written in the same swizzled layout
//   warp 2     allocates tensor memory; lane 0 copies the scale factors into
//              tensor memory (tcgen05.cp) and issues the MMAs
//   warp 3     cp.async producer: scale factors, repacked into the 512-byte
//              blocks tcgen05.cp expects (row m of 128 at byte 16*(m%32) + 4*(m/32),
//              four consecutive K-scales per row)
//   warps 4-7  epilogue: tensor memory -> registers; gate/up: h = silu(g) * u
//              quantised to MXFP4 along the intermediate dimension; down: fp32 rows
// Every wait is bounded; on a timeout the CTA raises an abort flag, drains
// what it has in flight, frees its tensor memory and reports kStatusWaitTimeout.
#include <math.h>

#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

constexpr int kTileBytes = 128 * 128;   // 128 rows x 128 bytes (256 E2M1 elements)
constexpr int kSfBytes = 1024;          // two 512-byte scale blocks (K = 256)
constexpr uint32_t kTmemCols = 512;

template <bool kGateUp>
struct Shape {
  static constexpr int kA = kGateUp ? 2 : 1;             // weight operands per stage
  static constexpr int kStages = kGateUp ? 4 : 6;
  static constexpr int kOffB = kA * kTileBytes;
  static constexpr int kOffSfa = (kA + 1) * kTileBytes;
  static constexpr int kOffSfb = kOffSfa + kA * kSfBytes;
  static constexpr int kStageBytes = kOffSfb + kSfBytes;
  static constexpr int kStagesBytes = kStages * kStageBytes;
  static constexpr int kStagingBytes = kGateUp ? 4 * 32 * 33 * 4 : 0;   // epilogue transposes
  static constexpr int kRowTabOff = kStagesBytes + kStagingBytes;
  static constexpr int kBarOff = kRowTabOff + 2 * 128 * 4;
  static constexpr int kSmem = 1024 + kBarOff + 256;     // + alignment slack of the base
  // tensor-memory columns: accumulators, then scale factors
  static constexpr uint32_t kColUp = 128;                // gate/up: up accumulator
  static constexpr uint32_t kColSfa = 256;               // kA x 8 columns
  static constexpr uint32_t kColSfb = 256 + 8 * kA;      // 8 columns
};
static_assert(Shape<true>::kSmem <= 232448, "gate/up shared memory");
static_assert(Shape<false>::kSmem <= 232448, "down shared memory");
static_assert(Shape<true>::kStageBytes % 1024 == 0 && Shape<false>::kStageBytes % 1024 == 0,
              "stages must keep the 1024-byte alignment of the swizzled tiles");

// MXFP4 encoding of 32 fp32 values (one block): 16 bytes of codes (element
// 2j in the low nibble of byte j) and the E8M0 scale code. Same rule as the
// activation quantiser: scale 2^(floor(log2 amax) - 2), nearest E2M1 with
// ties to even, sign kept (also for values that round to zero).
MOE_DEV uint4 quantize_block32(const float (&v)[32], uint32_t& code_s) {
  float amax = 0.0f;
#pragma unroll
  for (int j = 0; j < 32; ++j) amax = fmaxf(amax, fabsf(v[j]));
  // floor(log2 amax) + 127 is the biased exponent; zero and subnormal amax give code 0
  const int eb = (int)((__float_as_uint(amax) >> 23) & 0xFFu);
  const int cs = max(eb - 2, 0);
  code_s = (uint32_t)cs;
  const float inv = __uint_as_float((uint32_t)(254 - cs) << 23);   // 2^(127 - cs), exact
  uint32_t w[4] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int j = 0; j < 32; ++j) {
    const uint32_t c = e2m1_magnitude_code(fabsf(v[j]) * inv) | ((__float_as_uint(v[j]) >> 31) << 3);
    w[j >> 3] |= c << (4 * (j & 7));
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

}  // namespace

// One CTA of 1024 threads: the tiles of every active expert, in expert_list
// order; tiles[t] = {expert, first permuted row, rows (1..128), 0}.
__global__ void __launch_bounds__(1024) k_tile_list(const int32_t* __restrict__ offsets,
                                                    const int32_t* __restrict__ expert_list,
                                                    int4* __restrict__ tiles,
                                                    int32_t* __restrict__ n_tiles) {
  __shared__ int32_t warp_sum[32];
  const int n_act = __ldg(expert_list);
  const int a = threadIdx.x;
  int e = 0, first = 0, cnt = 0;
  if (a < n_act) {
    e = __ldg(expert_list + 1 + a);
    first = __ldg(offsets + e);
    cnt = __ldg(offsets + e + 1) - first;
  }
  const int nt = (cnt + 127) / 128;
  // exclusive scan of nt over the CTA (warp shuffles, then warp totals)
  const int lane = a & 31, warp = a >> 5;
  int incl = nt;
#pragma unroll
  for (int off = 1; off < 32; off <<= 1) {
    const int o = __shfl_up_sync(0xFFFFFFFFu, incl, off);
    if (lane >= off) incl += o;
  }
  if (lane == 31) warp_sum[warp] = incl;
  __syncthreads();
  if (warp == 0) {
    int v = warp_sum[lane];
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int o = __shfl_up_sync(0xFFFFFFFFu, v, off);
      if (lane >= off) v += o;
    }
    warp_sum[lane] = v;     // inclusive totals of warps 0..lane
  }
  __syncthreads();
  const int base = (warp ? warp_sum[warp - 1] : 0) + incl - nt;
  for (int j = 0; j < nt; ++j)
    tiles[base + j] = make_int4(e, first + 128 * j, min(128, cnt - 128 * j), 0);
  if (a == 1023) *n_tiles = warp_sum[31];
}

template <bool kGateUp>
__global__ void __launch_bounds__(256, 1) k_mxf4_gemm(const __grid_constant__ Mxf4GemmArgs a) {
  using S = Shape<kGateUp>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* staging = reinterpret_cast<float*>(smem + S::kStagesBytes);
  int32_t* rowtab_b = reinterpret_cast<int32_t*>(smem + S::kRowTabOff);
  int32_t* rowtab_s = rowtab_b + 128;
  uint64_t* full_tma = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* full_cp = full_tma + kStages;
  uint64_t* empty = full_cp + kStages;
  uint64_t* acc_full = empty + kStages;       // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
      mbar_init(&full_tma[s], 1);
      mbar_init(&full_cp[s], 64);
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
    tc::prefetch_map(&a.map_a0);
    if (kGateUp) tc::prefetch_map(&a.map_a1);
  }
  if (warp == 2) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;

  const int NT = __ldg(a.n_tiles);
  const int MT = a.M / 128;
  const int KT = (a.K + 255) / 256;
  const int kb_last = (a.K - (KT - 1) * 256) / 64;     // MMAs in the last stage: 2 or 4
  const long items = (long)NT * MT;
  const int ks = a.K / 32;                              // scale bytes per row

  if (warp == 0) {
    // ---------------- TMA producer: weight tiles ----------------
    uint32_t last_ph[kStages];
    bool filled[kStages];
#pragma unroll
    for (int s = 0; s < kStages; ++s) { last_ph[s] = 0; filled[s] = false; }
    if (lane == 0) {
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long q = blockIdx.x; q < items && ok; q += gridDim.x) {
        const int mt = (int)(q / NT);
        const int4 tile = __ldg(&a.tiles[q - (long)mt * NT]);
        const int y = tile.x * a.M + mt * 128;
        for (int kt = 0; kt < KT; ++kt) {
          if (!tc::wait_or_abort(&empty[s], ph ^ 1u, abort)) { ok = false; break; }
          uint8_t* st = smem + s * S::kStageBytes;
          mbar_expect_tx(&full_tma[s], S::kA * kTileBytes);
          tc::tma_load_2d(st, &a.map_a0, kt * 128, y, &full_tma[s]);
          if (kGateUp) tc::tma_load_2d(st + kTileBytes, &a.map_a1, kt * 128, y, &full_tma[s]);
          last_ph[s] = ph;
          filled[s] = true;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort) {     // let every issued load land before the CTA can exit
#pragma unroll
        for (int s2 = 0; s2 < kStages; ++s2)
          if (filled[s2]) mbar_wait(&full_tma[s2], last_ph[s2]);
      }
    }
  } else if (warp == 1 || warp == 3) {
    // ---------------- cp.async producers: token rows / scale factors ----------------
    const bool rows_role = (warp == 1);
    int32_t* rowtab = rows_role ? rowtab_b : rowtab_s;
    int s = 0;
    uint32_t ph = 0;
    bool ok = true;
    for (long q = blockIdx.x; q < items && ok; q += gridDim.x) {
      const int mt = (int)(q / NT);
      const int4 tile = __ldg(&a.tiles[q - (long)mt * NT]);
      const int nrows = tile.z, npad = (tile.z + 15) & ~15;
      __syncwarp();
#pragma unroll
      for (int j = 0; j < 4; ++j) {
        const int n = lane + 32 * j;
        int src = -1;
        if (n < nrows) src = a.row_token ? __ldg(a.row_token + tile.y + n) : tile.y + n;
        rowtab[n] = src;
      }
      __syncwarp();
      const long arow = (long)tile.x * a.M + mt * 128;
      for (int kt = 0; kt < KT; ++kt) {
        if (!tc::wait_or_abort(&empty[s], ph ^ 1u, abort)) { ok = false; break; }
        uint8_t* st = smem + s * S::kStageBytes;
        const int kbytes = min(128, a.K / 2 - kt * 128);     // 64 or 128
        if (rows_role) {
          const uint32_t bsm = smem_u32(st + S::kOffB);
          const int c = lane & 7;
          if (c * 16 < kbytes) {
            for (int n = lane >> 3; n < npad; n += 4) {
              const int src = rowtab[n];
              const uint8_t* g = src >= 0 ? a.bq + (size_t)src * (a.K / 2) + kt * 128 + c * 16 : a.bq;
              tc::cp16_zfill(bsm + n * 128 + ((c ^ (n & 7)) << 4), g, src >= 0 ? 16u : 0u);
            }
          }
        } else {
          const int nblk = kbytes / 64;
#pragma unroll
          for (int op = 0; op < S::kA; ++op) {
            const uint8_t* sa = op ? a.sa1 : a.sa0;
            const uint32_t dst = smem_u32(st + S::kOffSfa + op * kSfBytes);
#pragma unroll
            for (int j = 0; j < 4; ++j) {
              const uint8_t* g = sa + (size_t)(arow + lane + 32 * j) * ks + kt * 8;
              for (int b = 0; b < nblk; ++b) tc::cp4_zfill(dst + b * 512 + 16 * lane + 4 * j, g + 4 * b, 4u);
            }
          }
          const uint32_t dst = smem_u32(st + S::kOffSfb);
#pragma unroll
          for (int j = 0; j < 4; ++j) {
            const int src = rowtab[lane + 32 * j];
            const uint8_t* g = src >= 0 ? a.bs + (size_t)src * ks + kt * 8 : a.bs;
            for (int b = 0; b < nblk; ++b)
              tc::cp4_zfill(dst + b * 512 + 16 * lane + 4 * j, src >= 0 ? g + 4 * b : g, src >= 0 ? 4u : 0u);
          }
        }
        tc::cp_async_arrive(&full_cp[s]);
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
    }
    tc::cp_async_wait_all();
  } else if (warp == 2) {
    // ---------------- MMA issuer ----------------
    int s = 0;
    uint32_t ph = 0;
    int it = 0;
    bool ok = true;
    for (long q = blockIdx.x; q < items && ok; q += gridDim.x, ++it) {
      const int mt = (int)(q / NT);
      const int4 tile = __ldg(&a.tiles[q - (long)mt * NT]);
      const int npad = (tile.z + 15) & ~15;
      const uint32_t idesc = tc::idesc_mxf4(npad);
      const int buf = kGateUp ? 0 : (it & 1);
      const uint32_t acc_ph = kGateUp ? (uint32_t)(it & 1) : (uint32_t)((it >> 1) & 1);
      if (!tc::wait_or_abort(&acc_empty[buf], acc_ph ^ 1u, abort)) break;
      tc::fence_after_sync();
      const uint32_t d0 = tbase + (kGateUp ? 0u : 128u * buf);
      const uint32_t d1 = tbase + S::kColUp;
      const uint32_t sfa0 = tbase + S::kColSfa, sfa1 = tbase + S::kColSfa + 8, sfb = tbase + S::kColSfb;
      for (int kt = 0; kt < KT; ++kt) {
        if (!tc::wait_or_abort(&full_tma[s], ph, abort) || !tc::wait_or_abort(&full_cp[s], ph, abort)) {
          ok = false;
          break;
        }
        tc::fence_after_sync();
        fence_proxy_async_smem();       // cp.async data (generic proxy) -> tensor-core reads
        if (lane == 0) {
          const uint8_t* st = smem + s * S::kStageBytes;
          const int nkb = (kt == KT - 1) ? kb_last : 4;
          for (int b = 0; b < nkb / 2; ++b) {
            tc::cp_sf_block(sfa0 + 4 * b, tc::desc_sf(smem_u32(st + S::kOffSfa + b * 512)));
            if (kGateUp)
              tc::cp_sf_block(sfa1 + 4 * b, tc::desc_sf(smem_u32(st + S::kOffSfa + kSfBytes + b * 512)));
            tc::cp_sf_block(sfb + 4 * b, tc::desc_sf(smem_u32(st + S::kOffSfb + b * 512)));
          }
          const uint32_t a0 = smem_u32(st), a1 = smem_u32(st + kTileBytes), bb = smem_u32(st + S::kOffB);
          for (int kb = 0; kb < nkb; ++kb) {
            const uint32_t id = (kb & 1) ? 2u : 0u;            // byte of the 32-bit scale column
            const uint32_t col = 4u * (uint32_t)(kb >> 1);
            const uint32_t idk = tc::idesc_sf_id(idesc, id);
            const uint32_t acc = (kt > 0 || kb > 0) ? 1u : 0u;
            const uint64_t bdesc = tc::desc_sw128(bb + 32 * kb);
            tc::mma_mxf4(d0, tc::desc_sw128(a0 + 32 * kb), bdesc, idk, (sfa0 + col) | (id << 30),
                         (sfb + col) | (id << 30), acc);
            if (kGateUp)
              tc::mma_mxf4(d1, tc::desc_sw128(a1 + 32 * kb), bdesc, idk, (sfa1 + col) | (id << 30),
                           (sfb + col) | (id << 30), acc);
          }
          tc::commit(&empty[s]);
          if (kt == KT - 1) tc::commit(&acc_full[buf]);
        }
        __syncwarp();
        if (++s == kStages) { s = 0; ph ^= 1u; }
      }
    }
    if (lane == 0) {      // everything issued has completed before tensor memory is freed
      tc::commit(drain);
      mbar_wait(drain, 0);
    }
    __syncwarp();
  } else {
    // ---------------- epilogue (warps 4-7: tensor-memory lanes 32*(warp%4) ...) ----------------
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    int it = 0;
    for (long q = blockIdx.x; q < items; q += gridDim.x, ++it) {
      const int mt = (int)(q / NT);
      const int4 tile = __ldg(&a.tiles[q - (long)mt * NT]);
      const int row0 = tile.y, nrows = tile.z;
      const int buf = kGateUp ? 0 : (it & 1);
      const uint32_t acc_ph = kGateUp ? (uint32_t)(it & 1) : (uint32_t)((it >> 1) & 1);
      if (!tc::wait_or_abort(&acc_full[buf], acc_ph, abort)) break;
      tc::fence_after_sync();
      const int m0 = mt * 128 + 32 * wq;          // first weight row of this warp
      if (kGateUp) {
        float* stg = staging + wq * 32 * 33;
        for (int c0 = 0; c0 < nrows; c0 += 32) {
          uint32_t g[32], u[32];
          tc::ld_32cols(tbase + lane_off + c0, g);
          tc::ld_32cols(tbase + lane_off + S::kColUp + c0, u);
          tc::wait_ld();
          if (c0 + 32 >= nrows) {        // accumulators read: the next item may start
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&acc_empty[0]);
          }
#pragma unroll
          for (int c = 0; c < 32; ++c)
            stg[lane * 33 + c] = silu_f32(__uint_as_float(g[c])) * __uint_as_float(u[c]);
          __syncwarp();
          const int n = c0 + lane;       // this lane now owns token column n
          if (n < nrows) {
            float v[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) v[r] = stg[r * 33 + lane];
            uint32_t cs;
            const uint4 qv = quantize_block32(v, cs);
            const size_t row = (size_t)(row0 + n);
            *reinterpret_cast<uint4*>(a.hq + row * (a.M / 2) + m0 / 2) = qv;
            a.hs[row * (a.M / 32) + m0 / 32] = (uint8_t)cs;
          }
          __syncwarp();
        }
      } else {
        const uint32_t dcol = 128u * buf;
        for (int c0 = 0; c0 < nrows; c0 += 32) {
          uint32_t v[32];
          tc::ld_32cols(tbase + lane_off + dcol + c0, v);
          tc::wait_ld();
          if (c0 + 32 >= nrows) {
            tc::fence_before_sync();
            __syncwarp();
            if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
          }
          float* yrow = a.y + (size_t)(row0 + c0) * a.M + m0 + lane;
          const int nc = min(32, nrows - c0);
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < nc) yrow[(size_t)c * a.M] = __uint_as_float(v[c]);
        }
      }
    }
  }

  tc::fence_before_sync();
  __syncthreads();
  if (threadIdx.x == 0 && *abort) atomicOr(a.status, kStatusWaitTimeout);
  if (warp == 2) {
    tc::fence_after_sync();
    tc::tmem_dealloc(tbase, kTmemCols);
  }
}

size_t mxf4_gemm_smem_bytes(bool gate_up) {
  return gate_up ? (size_t)Shape<true>::kSmem : (size_t)Shape<false>::kSmem;
}

template __global__ void k_mxf4_gemm<true>(const __grid_constant__ Mxf4GemmArgs);
template __global__ void k_mxf4_gemm<false>(const __grid_constant__ Mxf4GemmArgs);

}  // namespace moe
