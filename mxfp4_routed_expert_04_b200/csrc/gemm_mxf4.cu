// Grouped block-scaled MXFP4 GEMM for experts with many tokens (prefill):
// 5th-generation tensor-core MMAs (tcgen05 kind::mxf4, E2M1 operands with one
// E8M0 scale per 32 elements of K) accumulating in tensor memory.
//
// The contraction is the routed expert of the rabbit README ("expert matmul"
// phase; model table row "MoE routing") with activations quantised to MXFP4
// like the weights (Kimi K3 page: its routed experts are MXFP4, read byte for
// byte).
//
// Orientation: the MMA's M side is 128 weight rows of one expert, its N side
// one tile of at most kTileRows of that expert's permuted rows, K the
// reduction. An item is (m-tile, tile); persistent CTAs take items
// m-tile-major, so that the tiles of a hot expert read the same weight tile at
// about the same time (once from HBM, then from L2).
//
// Every operand arrives by TMA on one mbarrier per stage (no generic-proxy
// copies on the data path): weight codes and token codes as 2-D tensor tiles
// with the 128-byte swizzle (rows of 128 bytes = 256 elements of K), the
// weight and token scales as contiguous 512-byte blocks of the tiled scale
// layout (sf_tiled_offset), which tcgen05.cp moves into tensor memory.
//
// Each stage carries two 128-row weight tiles that share the token tile (gate
// and up rows for gate/up, two consecutive row tiles of Wd for down): two
// independent accumulation chains keep the tensor pipe busy, where one chain
// would wait on the latency of each MMA.
//
// Roles (192 threads, one CTA per SM):
//   warp 0     TMA producer
//   warp 1     allocates tensor memory; lane 0 issues scale copies and MMAs
//   warps 2-5  epilogue (tensor-memory lane quarter = warp % 4):
//              gate/up: h = silu(g) * u, quantised to MXFP4 along the
//              intermediate dimension (codes row-major, scales tiled);
//              down: fp32 rows of y_perm
// Accumulators are double-buffered, so the epilogue of one item overlaps the
// main loop of the next. Every wait is bounded; on a timeout the CTA raises an
// abort flag, drains what it has in flight, frees its tensor memory and
// reports kStatusWaitTimeout.
#include <math.h>

#include "kernels.h"
#include "tc05.cuh"

namespace moe {

namespace {

constexpr int kATileBytes = 128 * 128;          // 128 weight rows x 128 bytes
constexpr int kBTileBytes = kTileRows * 128;    // kTileRows token rows x 128 bytes
constexpr int kSfBytes = 1024;                  // two 512-byte scale blocks (K = 256)
constexpr uint32_t kTmemCols = 512;
constexpr int kThreads = 192;

template <bool kGateUp>
struct Shape {
  static constexpr int kA = 2;                           // weight tiles per stage
  static constexpr int kStages = 4;
  static constexpr int kOffB = kA * kATileBytes;
  static constexpr int kOffSfa = kOffB + kBTileBytes;
  static constexpr int kOffSfb = kOffSfa + kA * kSfBytes;
  static constexpr int kStageBytes = kOffSfb + kSfBytes;
  static constexpr int kStagesBytes = kStages * kStageBytes;
  static constexpr int kStagingBytes = kGateUp ? 4 * 32 * 33 * 4 : 0;   // epilogue transposes
  static constexpr int kBarOff = kStagesBytes + kStagingBytes;
  static constexpr int kSmem = 1024 + kBarOff + 256;     // + alignment slack of the base
  // tensor-memory columns: two accumulator buffers, then the scale factors
  static constexpr uint32_t kAccCols = 2 * kTileRows;
  static constexpr uint32_t kColUp = kTileRows;          // second accumulator of a buffer
  static constexpr uint32_t kColSfa = 2 * kAccCols;      // kA x 8 columns
  static constexpr uint32_t kColSfb = kColSfa + 8 * kA;  // 8 columns
};
static_assert(Shape<true>::kSmem <= 232448 && Shape<false>::kSmem <= 232448, "shared memory");
static_assert(Shape<true>::kStageBytes % 1024 == 0 && Shape<false>::kStageBytes % 1024 == 0 &&
                  kBTileBytes % 1024 == 0,
              "stages must keep the 1024-byte alignment of the swizzled tiles");
static_assert(Shape<true>::kColSfb + 8 <= kTmemCols && Shape<false>::kColSfb + 8 <= kTmemCols,
              "tensor memory columns");
static_assert(kTileRows % 16 == 0 && kTileRows <= 128, "tile rows");

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

// silu(g) * u with the hardware exponential and divide; h is rounded to
// MXFP4 right after, far coarser than their few-ulp error.
MOE_DEV float swiglu_fast(float g, float u) { return __fdividef(g, 1.0f + __expf(-g)) * u; }

// item q -> (m-tile, tile)
struct Item {
  int mt;
  long t;
  int4 tile;
};
MOE_DEV Item item_of(long q, int NT, const int4* tiles) {
  Item it;
  it.mt = (int)(q / NT);
  it.t = q - (long)it.mt * NT;
  it.tile = __ldg(tiles + it.t);
  return it;
}

}  // namespace

// One CTA of 1024 threads: the tiles of every active expert, in expert_list
// order; tiles[t] = {expert, first permuted row, rows (1..kTileRows), 0},
// tile_base[e] = index of expert e's first tile, n_tiles[0] = tile count.
__global__ void __launch_bounds__(1024) k_tile_list(const int32_t* __restrict__ offsets,
                                                    const int32_t* __restrict__ expert_list,
                                                    int4* __restrict__ tiles,
                                                    int32_t* __restrict__ tile_base,
                                                    int32_t* __restrict__ n_tiles) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t warp_sum[32];
  const int n_act = __ldg(expert_list);
  const int a = threadIdx.x;
  int e = 0, first = 0, cnt = 0;
  if (a < n_act) {
    e = __ldg(expert_list + 1 + a);
    first = __ldg(offsets + e);
    cnt = __ldg(offsets + e + 1) - first;
  }
  const int nt = (cnt + kTileRows - 1) / kTileRows;
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
  if (a < n_act) tile_base[e] = base;
  for (int j = 0; j < nt; ++j)
    tiles[base + j] = make_int4(e, first + kTileRows * j, min(kTileRows, cnt - kTileRows * j), 0);
  if (a == 1023) *n_tiles = warp_sum[31];
}

// Row-major E8M0 scales [rows, K/32] -> the tiled layout with 128-row tiles
// (row m in tile m/128 at position m%128). rows % 128 == 0, K % 128 == 0.
__global__ void k_tile_scales(const uint8_t* __restrict__ src, long rows, int K,
                              uint8_t* __restrict__ dst) {
  pdl_wait();
  pdl_trigger();
  const int groups = K / 128;                    // 512-byte blocks per tile along K
  const long n = rows * (K / 128);
  for (long i = (long)blockIdx.x * blockDim.x + threadIdx.x; i < n; i += (long)gridDim.x * blockDim.x) {
    const long m = i / groups;
    const int g = (int)(i - m * groups);
    const uint32_t v = __ldg(reinterpret_cast<const uint32_t*>(src + m * (K / 32)) + g);
    *reinterpret_cast<uint32_t*>(dst + sf_tiled_offset(m / 128, groups, (int)(m % 128), 4 * g)) = v;
  }
}

template <bool kGateUp>
__global__ void __launch_bounds__(kThreads, 1) k_mxf4_gemm(const __grid_constant__ Mxf4GemmArgs a) {
  pdl_wait();
  pdl_trigger();
  using S = Shape<kGateUp>;
  constexpr int kStages = S::kStages;
  extern __shared__ uint8_t smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(smem_raw) + 1023) &
                                             ~static_cast<uintptr_t>(1023));
  float* staging = reinterpret_cast<float*>(smem + S::kStagesBytes);
  uint64_t* full = reinterpret_cast<uint64_t*>(smem + S::kBarOff);
  uint64_t* empty = full + kStages;
  uint64_t* acc_full = empty + kStages;       // [2]
  uint64_t* acc_empty = acc_full + 2;         // [2]
  uint64_t* drain = acc_empty + 2;
  uint32_t* tmem_slot = reinterpret_cast<uint32_t*>(drain + 1);
  volatile int* abort = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  if (threadIdx.x == 0) {
    for (int s = 0; s < kStages; ++s) {
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
    tc::prefetch_map(&a.map_a0);
    if (kGateUp) tc::prefetch_map(&a.map_a1);
    tc::prefetch_map(&a.map_b);
  }
  if (warp == 1) {
    tc::tmem_alloc(tmem_slot, kTmemCols);
    tc::tmem_relinquish();
  }
  tc::fence_before_sync();
  __syncthreads();
  tc::fence_after_sync();
  const uint32_t tbase = *tmem_slot;

  const int NT = __ldg(a.n_tiles);
  // gate/up: an m-tile is 128 rows of Wg and the same rows of Wu; down: 256
  // rows of Wd as two 128-row tiles (the second absent past the last row)
  const int MT = kGateUp ? a.M / 128 : (a.M + 255) / 256;
  const int KT = (a.K + 255) / 256;
  const int k128 = a.K / 128;                     // 512-byte scale blocks per tile row of K
  const int kb_last = (a.K - (KT - 1) * 256) / 64;     // MMAs in the last stage: 2 or 4
  const long items = (long)NT * MT;

  if (warp == 0) {
    // ---------------- TMA producer ----------------
    if (lane == 0) {
      uint32_t last_ph[kStages];
      bool filled[kStages];
#pragma unroll
      for (int s = 0; s < kStages; ++s) { last_ph[s] = 0; filled[s] = false; }
      int s = 0;
      uint32_t ph = 0;
      bool ok = true;
      for (long q = blockIdx.x; q < items && ok; q += gridDim.x) {
        const Item it = item_of(q, NT, a.tiles);
        const int ya = it.tile.x * a.M + it.mt * (kGateUp ? 128 : 256);
        const bool two = kGateUp || it.mt * 256 + 128 < a.M;
        const uint8_t* sfa0 = a.sa0 + ((size_t)(ya / 128) * k128) * 512;
        const uint8_t* sfa1 = kGateUp ? a.sa1 + ((size_t)(ya / 128) * k128) * 512
                                      : sfa0 + (size_t)k128 * 512;
        const uint8_t* sfb = a.bs + ((size_t)it.t * k128) * 512;
        for (int kt = 0; kt < KT; ++kt) {
          if (!tc::wait_or_abort(&empty[s], ph ^ 1u, abort)) { ok = false; break; }
          uint8_t* st = smem + s * S::kStageBytes;
          const uint32_t sf_bytes = (kt == KT - 1 && kb_last == 2) ? 512u : 1024u;
          const int na = two ? 2 : 1;
          mbar_expect_tx(&full[s], na * kATileBytes + kBTileBytes + (na + 1) * sf_bytes);
          tc::tma_load_2d(st, &a.map_a0, kt * 128, ya, &full[s]);
          if (kGateUp) tc::tma_load_2d(st + kATileBytes, &a.map_a1, kt * 128, ya, &full[s]);
          else if (two) tc::tma_load_2d(st + kATileBytes, &a.map_a0, kt * 128, ya + 128, &full[s]);
          tc::tma_load_2d(st + S::kOffB, &a.map_b, kt * 128, it.tile.y, &full[s]);
          bulk_g2s(st + S::kOffSfa, sfa0 + kt * 1024, sf_bytes, &full[s]);
          if (two) bulk_g2s(st + S::kOffSfa + kSfBytes, sfa1 + kt * 1024, sf_bytes, &full[s]);
          bulk_g2s(st + S::kOffSfb, sfb + kt * 1024, sf_bytes, &full[s]);
          last_ph[s] = ph;
          filled[s] = true;
          if (++s == kStages) { s = 0; ph ^= 1u; }
        }
      }
      if (*abort) {     // let every issued copy land before the CTA can exit
#pragma unroll
        for (int s2 = 0; s2 < kStages; ++s2)
          if (filled[s2]) mbar_wait(&full[s2], last_ph[s2]);
      }
    }
  } else if (warp == 1) {
    // ---------------- MMA issuer ----------------
    int s = 0;
    uint32_t ph = 0;
    int n_it = 0;
    bool ok = true;
    for (long q = blockIdx.x; q < items && ok; q += gridDim.x, ++n_it) {
      const Item it = item_of(q, NT, a.tiles);
      const int npad = (it.tile.z + 15) & ~15;
      const uint32_t idesc = tc::idesc_mxf4(npad);
      const bool two = kGateUp || it.mt * 256 + 128 < a.M;
      const int buf = n_it & 1;
      const uint32_t acc_ph = (uint32_t)((n_it >> 1) & 1);
      if (!tc::wait_or_abort(&acc_empty[buf], acc_ph ^ 1u, abort)) break;
      tc::fence_after_sync();
      const uint32_t d0 = tbase + S::kAccCols * buf;
      const uint32_t d1 = d0 + S::kColUp;
      const uint32_t sfa0 = tbase + S::kColSfa, sfa1 = sfa0 + 8, sfb = tbase + S::kColSfb;
      for (int kt = 0; kt < KT; ++kt) {
        if (!tc::wait_or_abort(&full[s], ph, abort)) { ok = false; break; }
        tc::fence_after_sync();
        if (lane == 0) {
          const uint8_t* st = smem + s * S::kStageBytes;
          const int nkb = (kt == KT - 1) ? kb_last : 4;
          // descriptors of the stage's first blocks; a later block only moves
          // the 14-bit address field (16-byte units: +2 per 32 bytes of a
          // swizzled row, +32 per 512-byte scale block), which cannot carry:
          // the stages are 1024-byte aligned below 228 KB
          const uint64_t dsa0 = tc::desc_sf(smem_u32(st + S::kOffSfa));
          const uint64_t dsa1 = tc::desc_sf(smem_u32(st + S::kOffSfa + kSfBytes));
          const uint64_t dsb = tc::desc_sf(smem_u32(st + S::kOffSfb));
#pragma unroll
          for (int b = 0; b < 2; ++b) {
            if (b < nkb / 2) {
              tc::cp_sf_block(sfa0 + 4 * b, dsa0 + 32u * b);
              if (two) tc::cp_sf_block(sfa1 + 4 * b, dsa1 + 32u * b);
              tc::cp_sf_block(sfb + 4 * b, dsb + 32u * b);
            }
          }
          const uint64_t da0 = tc::desc_sw128(smem_u32(st)), da1 = tc::desc_sw128(smem_u32(st + kATileBytes));
          const uint64_t db = tc::desc_sw128(smem_u32(st + S::kOffB));
          const uint32_t idk0 = tc::idesc_sf_id(idesc, 0u), idk2 = tc::idesc_sf_id(idesc, 2u);
#pragma unroll
          for (int kb = 0; kb < 4; ++kb) {
            if (kb < nkb) {
              const uint32_t id = (kb & 1) ? 2u : 0u;          // byte of the 32-bit scale column
              const uint32_t col = 4u * (uint32_t)(kb >> 1);
              const uint32_t idk = (kb & 1) ? idk2 : idk0;
              const uint32_t acc = (kt > 0 || kb > 0) ? 1u : 0u;
              const uint64_t bdesc = db + 2u * kb;
              tc::mma_mxf4(d0, da0 + 2u * kb, bdesc, idk, (sfa0 + col) | (id << 30), (sfb + col) | (id << 30),
                           acc);
              if (two)
                tc::mma_mxf4(d1, da1 + 2u * kb, bdesc, idk, (sfa1 + col) | (id << 30),
                             (sfb + col) | (id << 30), acc);
            }
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
    // ---------------- epilogue (warps 2-5: tensor-memory lanes 32*(warp%4) ...) ----------------
    const int wq = warp & 3;
    const uint32_t lane_off = (uint32_t)(32 * wq) << 16;
    int n_it = 0;
    for (long q = blockIdx.x; q < items; q += gridDim.x, ++n_it) {
      const Item it = item_of(q, NT, a.tiles);
      const int row0 = it.tile.y, nrows = it.tile.z;
      const int buf = n_it & 1;
      const uint32_t acc_ph = (uint32_t)((n_it >> 1) & 1);
      if (!tc::wait_or_abort(&acc_full[buf], acc_ph, abort)) break;
      tc::fence_after_sync();
      const uint32_t dcol = tbase + lane_off + S::kAccCols * buf;
      const bool two = kGateUp || it.mt * 256 + 128 < a.M;
      // first weight row of this warp (down: of its lanes in the first 128-row tile)
      const int m0 = it.mt * (kGateUp ? 128 : 256) + 32 * wq;
      for (int c0 = 0; c0 < nrows; c0 += 32) {
        const bool last = c0 + 32 >= nrows;
        uint32_t g[32], u[32];
        if (c0 + 32 <= kTileRows) {
          tc::ld_32cols(dcol + c0, g);
          if (two) tc::ld_32cols(dcol + S::kColUp + c0, u);
        } else {                                     // the last 16 columns of a tile
          tc::ld_16cols(dcol + c0, g);
          if (two) tc::ld_16cols(dcol + S::kColUp + c0, u);
        }
        tc::wait_ld();
        if (last) {                                  // accumulators read: the MMA may reuse them
          tc::fence_before_sync();
          __syncwarp();
          if (lane == 0) tc::mbar_arrive(&acc_empty[buf]);
        }
        const int nc = min(32, nrows - c0);
        if (kGateUp) {
          float* stg = staging + wq * 32 * 33;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            stg[lane * 33 + c] = swiglu_fast(__uint_as_float(g[c]), __uint_as_float(u[c]));
          __syncwarp();
          if (lane < nc) {                             // this lane now owns token column c0 + lane
            const int n = c0 + lane;
            float v[32];
#pragma unroll
            for (int r = 0; r < 32; ++r) v[r] = stg[r * 33 + lane];
            uint32_t cs;
            const uint4 qv = quantize_block32(v, cs);
            *reinterpret_cast<uint4*>(a.hq + (size_t)(row0 + n) * (a.M / 2) + m0 / 2) = qv;
            a.hs[sf_tiled_offset(it.t, a.M / 128, n, m0 / 32)] = (uint8_t)cs;
          }
          __syncwarp();
        } else {
          float* yrow = a.y + (size_t)(row0 + c0) * a.M + m0 + lane;
#pragma unroll
          for (int c = 0; c < 32; ++c)
            if (c < nc) yrow[(size_t)c * a.M] = __uint_as_float(g[c]);
          if (two) {
#pragma unroll
            for (int c = 0; c < 32; ++c)
              if (c < nc) yrow[(size_t)c * a.M + 128] = __uint_as_float(u[c]);
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
    tc::tmem_dealloc(tbase, kTmemCols);
  }
}

size_t mxf4_gemm_smem_bytes(bool gate_up) {
  return gate_up ? (size_t)Shape<true>::kSmem : (size_t)Shape<false>::kSmem;
}
int mxf4_gemm_threads() { return kThreads; }

template __global__ void k_mxf4_gemm<true>(const __grid_constant__ Mxf4GemmArgs);
template __global__ void k_mxf4_gemm<false>(const __grid_constant__ Mxf4GemmArgs);

}  // namespace moe
