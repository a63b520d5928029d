// Device helpers shared by the layer's kernels (sm_100a).
#pragma once

#include <cuda_fp16.h>
#include <cuda_runtime.h>
#include <stdint.h>

#define MOE_DEV __device__ __forceinline__

namespace moe {

// ---------------------------------------------------------------------------
// device status word (bit flags, kept in the caller's workspace)
// ---------------------------------------------------------------------------
enum : int32_t {
  kStatusBadExpertIndex = 1,   // an expert index outside [0, E)
  kStatusRepeatedExpert = 2,   // the same expert twice in one token's top-k
};

// ---------------------------------------------------------------------------
// number formats
// ---------------------------------------------------------------------------

// bf16 bit pattern -> float (exact).
MOE_DEV float bf16_to_f32(uint32_t bits16) { return __uint_as_float(bits16 << 16); }

// The two bf16 halves of a 32-bit word -> floats (exact).
MOE_DEV float bf16lo(uint32_t w) { return __uint_as_float(w << 16); }
MOE_DEV float bf16hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// float -> bf16 bits, round to nearest even (finite inputs; NaN kept quiet).
MOE_DEV uint32_t f32_to_bf16_rne(float f) {
  uint32_t b = __float_as_uint(f);
  if ((b & 0x7FFFFFFFu) > 0x7F800000u) return (b >> 16) | 0x40u;  // NaN
  b += 0x7FFFu + ((b >> 16) & 1u);
  return b >> 16;
}

// E8M0 scale code -> float: 2^(c-127); c = 0 gives the subnormal 2^-127 and
// c = 255 gives NaN (OCP MX v1.0, section 5.4).
MOE_DEV float e8m0_to_f32(uint32_t c) {
  uint32_t bits = c << 23;
  bits = (c == 0u) ? 0x00400000u : bits;
  bits = (c == 255u) ? 0x7FC00000u : bits;
  return __uint_as_float(bits);
}

// Four bytes of packed E2M1 pairs -> four f16x2 words (exact). Byte j of `w`
// becomes out[j]; its low nibble goes to the low half.
MOE_DEV void e2m1x8_to_f16x8(uint32_t w, uint32_t (&out)[4]) {
  asm("{\n\t.reg .b8 b0, b1, b2, b3;\n\t"
      "mov.b32 {b0, b1, b2, b3}, %4;\n\t"
      "cvt.rn.f16x2.e2m1x2 %0, b0;\n\t"
      "cvt.rn.f16x2.e2m1x2 %1, b1;\n\t"
      "cvt.rn.f16x2.e2m1x2 %2, b2;\n\t"
      "cvt.rn.f16x2.e2m1x2 %3, b3;\n\t}"
      : "=r"(out[0]), "=r"(out[1]), "=r"(out[2]), "=r"(out[3])
      : "r"(w));
}

// E2M1 code (0..7 magnitude) of a non-negative value already divided by the
// block scale: nearest of {0, .5, 1, 1.5, 2, 3, 4, 6}, ties to the even code
// (the OCP MX v1.0 conversion to E2M1).
MOE_DEV uint32_t e2m1_magnitude_code(float s) {
  return (uint32_t)(s > 0.25f) + (uint32_t)(s >= 0.75f) + (uint32_t)(s > 1.25f) +
         (uint32_t)(s >= 1.75f) + (uint32_t)(s > 2.5f) + (uint32_t)(s >= 3.5f) +
         (uint32_t)(s > 5.0f);
}

// Byte offset of scale j (K-block of 32 elements) of row n of tile `tile` in
// the tiled scale layout read by the tcgen05 block-scaled MMAs: per tile and
// per 128 elements of K one 512-byte block, row n at 16*(n%32) + 4*(n/32),
// four consecutive K-blocks in four consecutive bytes.
MOE_DEV size_t sf_tiled_offset(long tile, int k128, int n, int j) {
  return ((size_t)tile * k128 + (j >> 2)) * 512 + 16 * (n & 31) + 4 * (n >> 5) + (j & 3);
}

// ---------------------------------------------------------------------------
// tensor-core MMA (warp-level m16n8k16, fp32 accumulate)
// ---------------------------------------------------------------------------
MOE_DEV void mma_f16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

MOE_DEV void mma_bf16(float (&d)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 "
      "{%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// ---------------------------------------------------------------------------
// memory
// ---------------------------------------------------------------------------
MOE_DEV uint32_t smem_u32(const void* p) {
  return static_cast<uint32_t>(__cvta_generic_to_shared(p));
}

MOE_DEV void cp_async_16(uint32_t dst, const void* src) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(dst), "l"(src));
}
MOE_DEV void cp_async_4(uint32_t dst, const void* src) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(dst), "l"(src));
}
MOE_DEV void cp_async_commit() { asm volatile("cp.async.commit_group;\n" ::); }
template <int N>
MOE_DEV void cp_async_wait() { asm volatile("cp.async.wait_group %0;\n" ::"n"(N)); }

MOE_DEV void ldmatrix_x4(uint32_t (&r)[4], uint32_t addr) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// 16-byte read-only global load that does not allocate in L1 (streamed weights).
MOE_DEV uint4 ldg_stream(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

MOE_DEV uint4 ldg16(const void* p) { return __ldg(reinterpret_cast<const uint4*>(p)); }

// shared-memory loads at 32-bit shared addresses
MOE_DEV uint4 lds16(uint32_t addr) {
  uint4 v;
  asm volatile("ld.shared.v4.u32 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w) : "r"(addr));
  return v;
}
MOE_DEV uint32_t lds8(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u8 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}
MOE_DEV uint32_t lds32(uint32_t addr) {
  uint32_t v;
  asm volatile("ld.shared.u32 %0, [%1];\n" : "=r"(v) : "r"(addr));
  return v;
}
MOE_DEV void sts16(uint32_t addr, uint4 v) {
  asm volatile("st.shared.v4.u32 [%0], {%1,%2,%3,%4};\n" ::"r"(addr), "r"(v.x), "r"(v.y), "r"(v.z), "r"(v.w)
               : "memory");
}
MOE_DEV void sts32(uint32_t addr, uint32_t v) {
  asm volatile("st.shared.u32 [%0], %1;\n" ::"r"(addr), "r"(v) : "memory");
}

// ---------------------------------------------------------------------------
// misc
// ---------------------------------------------------------------------------
// Exponent of m = f * 2^e with f in [0.5, 1) for finite m > 0, read from the
// IEEE-754 fields (subnormals by their leading one).
MOE_DEV int frexp_exponent(float m) {
  const uint32_t b = __float_as_uint(m);
  const int e = (int)((b >> 23) & 0xFFu);
  return e != 0 ? e - 126 : (31 - __clz((int)(b & 0x7FFFFFu))) - 148;
}
// 2^n as fp32 for n in [-149, 127], built from its bit pattern
MOE_DEV float pow2_f32(int n) {
  return n >= -126 ? __uint_as_float((uint32_t)(n + 127) << 23) : __uint_as_float(1u << (n + 149));
}

// A fragments of the two k16 halves of one block from the row-g / row-g+8 words.
MOE_DEV void decode_block(uint32_t wg, uint32_t wg8, uint32_t (&a0)[4], uint32_t (&a1)[4]) {
  uint32_t lo[4], hi[4];
  e2m1x8_to_f16x8(wg, lo);
  e2m1x8_to_f16x8(wg8, hi);
  a0[0] = lo[0]; a0[1] = hi[0]; a0[2] = lo[1]; a0[3] = hi[1];
  a1[0] = lo[2]; a1[1] = hi[2]; a1[2] = lo[3]; a1[3] = hi[3];
}

// Operands of the CUDA-core GEMVs (the f16 token rows and h rows) have their
// largest magnitude in [2^14, 2^15): their products are exact in the fp32
// FMAs that sum them, and every bf16 value keeps all its bits down to 2^-29
// of the maximum.
constexpr int kF16OpTop = 15;

// power-of-two scale mapping a block maximum m into [2^(top-1), 2^top) as f16
MOE_DEV void f16_block_scale(float m, float& scale, float& inv, int top = 15) {
  if (!(m > 0.0f) || !isfinite(m)) { scale = 1.0f; inv = 1.0f; return; }
  const int ex = max(-100, min(127, frexp_exponent(m)));   // m = f * 2^ex, f in [0.5, 1)
  scale = pow2_f32(ex - top);
  inv = pow2_f32(top - ex);
}

// Sum of S split-K partials p[0], p[stride], ... in the order s = 0, 1, ...;
// the loads are issued sixteen at a time ahead of their additions.
MOE_DEV float sum_splits(const float* __restrict__ p, int S, size_t stride) {
  float acc = 0.0f;
  int s = 0;
  for (; s + 16 <= S; s += 16) {
    float v[16];
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __ldg(p + (size_t)(s + i) * stride);
#pragma unroll
    for (int i = 0; i < 16; ++i) acc += v[i];
  }
  for (; s + 4 <= S; s += 4) {
    float v[4];
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __ldg(p + (size_t)(s + i) * stride);
#pragma unroll
    for (int i = 0; i < 4; ++i) acc += v[i];
  }
  for (; s < S; ++s) acc += __ldg(p + (size_t)s * stride);
  return acc;
}

MOE_DEV float silu_f32(float z) { return z / (1.0f + expf(-z)); }

// Programmatic dependent launch: wait until the previous kernel of the stream
// has completed and its writes are visible (no-op for a kernel launched
// without the attribute), then let the next kernel of the stream launch
// while this one runs (it waits in its own pdl_wait before reading anything).
MOE_DEV void pdl_wait() { asm volatile("griddepcontrol.wait;\n" ::: "memory"); }
MOE_DEV void pdl_trigger() { asm volatile("griddepcontrol.launch_dependents;\n" ::: "memory"); }
MOE_DEV float sigmoid_f32(float z) { return 1.0f / (1.0f + expf(-z)); }

// Expert of the a-th non-empty segment of `offsets` (E+1 entries), or -1.
// Whole warp calls it; returns the same value in every lane.
MOE_DEV int nth_active_expert(const int32_t* __restrict__ offsets, int E, int a, int lane) {
  int seen = 0;
  for (int base = 0; base < E; base += 32) {
    const int e = base + lane;
    const int cnt = (e < E) ? (__ldg(offsets + e + 1) - __ldg(offsets + e)) : 0;
    const unsigned m = __ballot_sync(0xFFFFFFFFu, cnt > 0);
    const int c = __popc(m);
    if (seen + c > a) {
      const int want = a - seen;
      const int pre = __popc(m & ((1u << lane) - 1u));
      const unsigned hit = __ballot_sync(0xFFFFFFFFu, cnt > 0 && pre == want);
      return base + __ffs(hit) - 1;
    }
    seen += c;
  }
  return -1;
}

}  // namespace moe

namespace moe {

// acc + a * b with f16 a, b (the two halves of the f16x2 words wa, wb) and an
// fp32 accumulator; the product of two f16 values is exact in fp32.
MOE_DEV float fma_f16lo(uint32_t wa, uint32_t wb, float acc) {
  float d;
  asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a0, b0, %3;\n\t}"
      : "=f"(d) : "r"(wa), "r"(wb), "f"(acc));
  return d;
}
MOE_DEV float fma_f16hi(uint32_t wa, uint32_t wb, float acc) {
  float d;
  asm("{\n\t.reg .f16 a0, a1, b0, b1;\n\t"
      "mov.b32 {a0, a1}, %1;\n\t"
      "mov.b32 {b0, b1}, %2;\n\t"
      "fma.rn.f32.f16 %0, a1, b1, %3;\n\t}"
      : "=f"(d) : "r"(wa), "r"(wb), "f"(acc));
  return d;
}

// Dot product of one 32-element MXFP4 block (16 packed bytes) with 32 f16
// activations (16 f16x2 words), fp32 accumulation, block scale not applied.
MOE_DEV float dot_block_e2m1_f16(uint4 w, const uint32_t (&x)[16]) {
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

// Warp reduce-scatter of 32 values per lane: afterwards lane l holds the sum
// over the warp of v[l] (v[0] on return).
MOE_DEV float warp_reduce_scatter32(float (&v)[32], int lane) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const bool upper = (lane & off) != 0;
#pragma unroll
    for (int i = 0; i < off; ++i) {
      const float send = upper ? v[i] : v[i + off];
      const float keep = upper ? v[i + off] : v[i];
      v[i] = keep + __shfl_xor_sync(0xFFFFFFFFu, send, off);
    }
  }
  return v[0];
}

}  // namespace moe

namespace moe {

// ---------------------------------------------------------------------------
// mbarrier + bulk-copy (TMA, non-tensor) helpers
// ---------------------------------------------------------------------------
enum : int32_t { kStatusWaitTimeout = 4 };   // a bounded device wait gave up

MOE_DEV void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count));
}
MOE_DEV void fence_mbar_init() { asm volatile("fence.mbarrier_init.release.cluster;\n" ::); }
MOE_DEV void fence_proxy_async_smem() { asm volatile("fence.proxy.async.shared::cta;\n" ::); }

MOE_DEV void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.arrive.expect_tx.release.cta.shared::cta.b64 _, [%0], %1;\n"
               ::"r"(smem_u32(bar)), "r"(bytes));
}

// Bounded wait for phase `parity` of `bar`: false when it did not complete
// within `limit` tries (the caller reports it and leaves). Each try_wait may
// suspend the thread for up to 20 us until the phase completes, so a waiting
// warp does not spin on the issue slots; the default bound is about 5 s.
MOE_DEV bool mbar_wait(uint64_t* bar, uint32_t parity, uint32_t limit = 1u << 18) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t it = 0; it < limit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(a), "r"(parity), "r"(20000u) : "memory");
    if (done) return true;
  }
  return false;
}

// Bulk global -> shared copy completing on `bar` (16-byte aligned, bytes % 16 == 0).
MOE_DEV void bulk_g2s(void* dst, const void* src, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n"
      ::"r"(smem_u32(dst)), "l"(src), "r"(bytes), "r"(smem_u32(bar)) : "memory");
}

}  // namespace moe
