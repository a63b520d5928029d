// Token -> expert dispatch and the activation operands of the expert kernels.
//
// k_permute: per-expert histogram, exclusive scan and a stable placement of
// the T*k (token, slot) pairs: rows grouped by expert, ascending token inside
// an expert. One CTA of 1024 threads walks the pairs in chunks of 8192 in
// (token, slot) order, each warp over 256 consecutive pairs in 8 rounds;
// a pair's rank among equal experts comes from __match_any_sync within its
// round, its warp's count from the earlier rounds, and a per-(warp, expert)
// exclusive scan over the 32 warps, so the placement is deterministic.
//
// k_act_to_f16: bf16 activation rows -> f16 rows with one power-of-two scale
// per row (the largest magnitude maps into [2^14, 2^15); bf16 values keep all
// their bits down to 2^-29 of the row maximum).
//
// k_act_to_mxfp4_perm: bf16 activation rows -> OCP MXFP4 (the OCP MX v1.0
// conversion: shared exponent floor(log2 amax) - 2, elements rounded to the
// nearest E2M1 value with ties to the even code, saturating at 6), written to
// every permuted row of the token (the operand of the tensor-core path).
#include <math.h>

#include "common.cuh"
#include "kernels.h"

namespace moe {

constexpr int kPermThreads = 1024;
constexpr int kPermWarps = kPermThreads / 32;
constexpr int kPermSub = 8;            // rounds of 32 pairs per warp and chunk

// cursors [E], a flag word, and (more than one warp of pairs) the per-warp
// counts [32][E]
size_t permute_smem_bytes(int E, int R) {
  return ((size_t)E + 4 + (R > 32 ? (size_t)kPermWarps * E : 0)) * sizeof(int32_t);
}

// grid 1, block 1024, dynamic smem permute_smem_bytes(E, T * k)
__global__ void __launch_bounds__(kPermThreads) k_permute(const int32_t* __restrict__ idx, int T, int k,
                                                        int E, int32_t* __restrict__ counts,
                                                        int32_t* __restrict__ offsets,
                                                        int32_t* __restrict__ expert_list,
                                                        int32_t* __restrict__ row_token,
                                                        int32_t* __restrict__ row_slot,
                                                        int32_t* __restrict__ slot_row,
                                                        int32_t* __restrict__ status) {
  pdl_wait();
  pdl_trigger();
  extern __shared__ int32_t sm[];
  int32_t* cnt = sm;                   // [E]  running cursor per expert
  int32_t* flag = sm + E;
  int32_t* whist = sm + E + 4;         // [32][E] per-warp counts -> exclusive bases
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int R = T * k;

  for (int e = tid; e < E; e += kPermThreads) cnt[e] = 0;
  if (tid == 0) flag[0] = 0;
  __syncthreads();

  // validate and count
  for (int p = tid; p < R; p += kPermThreads) {
    const int e = idx[p];
    if (e < 0 || e >= E) {
      atomicOr(&flag[0], kStatusBadExpertIndex);
      continue;
    }
    const int t = p / k, j = p - t * k;
    for (int jj = 0; jj < j; ++jj)
      if (idx[t * k + jj] == e) atomicOr(&flag[0], kStatusRepeatedExpert);
    atomicAdd(&cnt[e], 1);
  }
  __syncthreads();
  const int bad = flag[0];
  if (bad) {
    for (int e = tid; e < E; e += kPermThreads) counts[e] = 0;
    for (int e = tid; e <= E; e += kPermThreads) offsets[e] = 0;
    if (tid == 0) expert_list[0] = 0;
    if (tid == 0) atomicOr(status, bad);
    return;
  }

  // exclusive scan of the counts (E <= 1024: one element per thread)
  {
    const int e = tid;
    const int c = (e < E) ? cnt[e] : 0;
    int incl = c;
#pragma unroll
    for (int off = 1; off < 32; off <<= 1) {
      const int y = __shfl_up_sync(0xFFFFFFFFu, incl, off);
      if (lane >= off) incl += y;
    }
    __shared__ int32_t wsum[kPermWarps];
    if (lane == 31) wsum[warp] = incl;
    __syncthreads();
    if (warp == 0) {
      int ws = wsum[lane];
#pragma unroll
      for (int off = 1; off < 32; off <<= 1) {
        const int y = __shfl_up_sync(0xFFFFFFFFu, ws, off);
        if (lane >= off) ws += y;
      }
      wsum[lane] = ws;       // inclusive warp totals
    }
    __syncthreads();
    const int excl = incl - c + (warp > 0 ? wsum[warp - 1] : 0);
    if (e < E) {
      counts[e] = c;
      offsets[e] = excl;
      cnt[e] = excl;         // cursor
    }
    if (e == E - 1) offsets[E] = excl + c;
    // compact list of the experts that received pairs, ascending
    const unsigned act = __ballot_sync(0xFFFFFFFFu, c > 0);
    __syncthreads();
    if (lane == 0) wsum[warp] = __popc(act);
    __syncthreads();
    int before = 0;
    for (int w = 0; w < warp; ++w) before += wsum[w];
    if (c > 0) expert_list[1 + before + __popc(act & ((1u << lane) - 1u))] = e;
    if (tid == kPermThreads - 1) expert_list[0] = before + __popc(act);
  }
  __syncthreads();

  // stable placement; at most 32 pairs: one warp, ranks from its match masks
  if (R <= 32) {
    if (warp == 0) {
      const int e = (lane < R) ? idx[lane] : -1;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      if (e >= 0) {
        const int pos = cnt[e] + __popc(peers & ((1u << lane) - 1u));
        const int t = lane / k;
        row_token[pos] = t;
        row_slot[pos] = lane - t * k;
        slot_row[lane] = pos;
      }
    }
    return;
  }
  // chunk by chunk: warp w takes the kPermSub * 32 consecutive pairs
  // base + w * kPermSub * 32 ..., kPermSub rounds of 32; a pair's rank among
  // equal experts = the earlier rounds' count in its warp's row of whist plus
  // its lower peers in the round; then one exclusive scan over the warps per
  // expert turns the rows into bases (the histogram work is per chunk, so
  // large chunks keep it small against the pairs)
  for (int base = 0; base < R; base += kPermThreads * kPermSub) {
    for (int i = tid; i < kPermWarps * E; i += kPermThreads) whist[i] = 0;
    __syncthreads();
    const int wbase = base + warp * 32 * kPermSub;
    int es[kPermSub], rk[kPermSub];
#pragma unroll
    for (int s = 0; s < kPermSub; ++s) {
      const int p = wbase + 32 * s + lane;
      const int e = (p < R) ? idx[p] : -1;
      const unsigned peers = __match_any_sync(0xFFFFFFFFu, e);
      const int prev = (e >= 0) ? whist[warp * E + e] : 0;
      __syncwarp();
      if (e >= 0 && lane == __ffs(peers) - 1) whist[warp * E + e] = prev + __popc(peers);
      __syncwarp();
      es[s] = e;
      rk[s] = prev + __popc(peers & ((1u << lane) - 1u));
    }
    __syncthreads();
    for (int ee = tid; ee < E; ee += kPermThreads) {
      int run = cnt[ee];
      for (int w = 0; w < kPermWarps; ++w) {
        const int c = whist[w * E + ee];
        whist[w * E + ee] = run;
        run += c;
      }
      cnt[ee] = run;
    }
    __syncthreads();
#pragma unroll
    for (int s = 0; s < kPermSub; ++s) {
      if (es[s] >= 0) {
        const int p = wbase + 32 * s + lane;
        const int pos = whist[warp * E + es[s]] + rk[s];
        const int t = p / k;
        row_token[pos] = t;
        row_slot[pos] = p - t * k;
        slot_row[p] = pos;
      }
    }
    __syncthreads();
  }
}

// ---------------------------------------------------------------------------
// activation operands, one CTA of 256 threads per token row
// ---------------------------------------------------------------------------

MOE_DEV float block_max_256(float v) {
  __shared__ float red[8];
#pragma unroll
  for (int off = 16; off > 0; off >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, off));
  if ((threadIdx.x & 31) == 0) red[threadIdx.x >> 5] = v;
  __syncthreads();
  float m = red[0];
#pragma unroll
  for (int i = 1; i < 8; ++i) m = fmaxf(m, red[i]);
  __syncthreads();
  return m;
}

// grid T, block 256; W a multiple of 8
__global__ void __launch_bounds__(256) k_act_to_f16(const uint16_t* __restrict__ x, int W,
                                                  __half* __restrict__ x16,
                                                  float* __restrict__ xscale) {
  pdl_wait();
  pdl_trigger();
  const int tok = blockIdx.x;
  const uint16_t* row = x + (size_t)tok * W;
  float m = 0.0f;
  for (int i = threadIdx.x * 8; i < W; i += 256 * 8) {
    const uint4 v = ldg16(row + i);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int j = 0; j < 4; ++j) m = fmaxf(m, fmaxf(fabsf(bf16lo(wv[j])), fabsf(bf16hi(wv[j]))));
  }
  m = block_max_256(m);
  float scale, inv;
  f16_block_scale(m, scale, inv, kF16OpTop);
  for (int i = threadIdx.x * 8; i < W; i += 256 * 8) {
    const uint4 v = ldg16(row + i);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    uint32_t o[4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const __half2 h = __floats2half2_rn(bf16lo(wv[j]) * inv, bf16hi(wv[j]) * inv);
      o[j] = *reinterpret_cast<const uint32_t*>(&h);
    }
    *reinterpret_cast<uint4*>(x16 + (size_t)tok * W + i) = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (threadIdx.x == 0) xscale[tok] = scale;
}

// grid T, block 256; W a multiple of 128. MXFP4 activation operand of the
// tensor-core path: token t's row quantised block by block (the conversion in
// the file header) and written to each of its k permuted rows
// r = slot_row[t, j]: codes to q[r] and scales into the tiled layout at
// (tile, n) of row r (tile_base from k_tile_list, tiles of kTileRows
// consecutive rows of one expert). Writes nothing when the permutation was
// rejected (expert_list[0] == 0 then).
__global__ void __launch_bounds__(256) k_act_to_mxfp4_perm(
    const uint16_t* __restrict__ x, int W, int k, const int32_t* __restrict__ idx,
    const int32_t* __restrict__ slot_row, const int32_t* __restrict__ offsets,
    const int32_t* __restrict__ expert_list, const int32_t* __restrict__ tile_base,
    uint8_t* __restrict__ q, uint8_t* __restrict__ sf) {
  pdl_wait();
  pdl_trigger();
  __shared__ int32_t s_row[32], s_tile[32], s_n[32];
  if (__ldg(expert_list) == 0) return;
  const int tok = blockIdx.x;
  if (threadIdx.x < k) {
    const int j = threadIdx.x;
    const int e = __ldg(idx + (size_t)tok * k + j);
    const int r = __ldg(slot_row + (size_t)tok * k + j);
    const int local = r - __ldg(offsets + e);
    s_row[j] = r;
    s_tile[j] = __ldg(tile_base + e) + local / kTileRows;
    s_n[j] = local % kTileRows;
  }
  __syncthreads();
  const uint16_t* row = x + (size_t)tok * W;
  const int k128 = W / 128;
  for (int base = 0; base < W; base += 256 * 8) {      // uniform trip count: shuffles below
    const int i = base + threadIdx.x * 8;
    const bool ok = i < W;
    uint4 v = make_uint4(0u, 0u, 0u, 0u);
    if (ok) v = ldg16(row + i);
    const uint32_t wv[4] = {v.x, v.y, v.z, v.w};
    float f[8];
#pragma unroll
    for (int j = 0; j < 4; ++j) { f[2 * j] = bf16lo(wv[j]); f[2 * j + 1] = bf16hi(wv[j]); }
    float m = 0.0f;
#pragma unroll
    for (int j = 0; j < 8; ++j) m = fmaxf(m, fabsf(f[j]));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 1));
    m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, 2));
    int code_s = 0;
    if (m > 0.0f) {
      int ex;
      frexpf(m, &ex);                    // floor(log2 m) = ex - 1
      code_s = min(254, max(0, 127 + (ex - 1) - 2));
    }
    const float inv = ldexpf(1.0f, 127 - code_s);
    uint32_t packed = 0;
#pragma unroll
    for (int j = 0; j < 8; ++j) {
      const uint32_t c = e2m1_magnitude_code(fabsf(f[j]) * inv) | (signbit(f[j]) ? 8u : 0u);
      packed |= c << (4 * j);
    }
    if (ok) {
      for (int j = 0; j < k; ++j) {
        *reinterpret_cast<uint32_t*>(q + (size_t)s_row[j] * (W / 2) + i / 2) = packed;
        if ((threadIdx.x & 3) == 0) sf[sf_tiled_offset(s_tile[j], k128, s_n[j], i / 32)] = (uint8_t)code_s;
      }
    }
  }
}

}  // namespace moe
