// Fifth-generation tensor core (tcgen05), tensor memory and tensor-TMA helpers
// for sm_100a, written as inline PTX.
//
// Descriptor encodings follow the PTX ISA (tcgen05 "Matrix descriptors" and
// "Instruction descriptor" tables):
//   shared-memory matrix descriptor (64 bit)
//     [0,14)  start address >> 4        [16,30) leading-dimension byte offset >> 4
//     [32,46) stride-dimension byte offset >> 4
//     [46,48) version (1 on sm_100)     [49,52) base offset   [52] LBO mode
//     [61,64) layout: 0 none (interleaved 8x16 B core matrices), 2 = 128-byte swizzle
//   block-scaled instruction descriptor (32 bit, kind::mxf4)
//     [4,6) B scale-factor id  [7,10) A format (1 = E2M1)  [10,13) B format
//     [15]/[16] A/B major (0 = K-major)  [17,23) N >> 3  [23] scale type (1 = E8M0)
//     [24,29) M >> 4  [29,31) A scale-factor id  [31] K size (0 = 64)
#pragma once

#include <cuda.h>
#include <stdint.h>

#include "common.cuh"

namespace moe {
namespace tc {

// --- tensor memory ------------------------------------------------------------
// Whole warp: allocate `ncols` (power of two >= 32) columns; the base address
// is written to shared memory at `dst`.
MOE_DEV void tmem_alloc(uint32_t* dst, uint32_t ncols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n"
               ::"r"(smem_u32(dst)), "r"(ncols) : "memory");
}
MOE_DEV void tmem_relinquish() {
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}
MOE_DEV void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(ncols)
               : "memory");
}
MOE_DEV void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory"); }
MOE_DEV void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory"); }

// Arrive once on `bar` when every tcgen05 operation this thread issued so far
// (MMAs and copies) has completed.
MOE_DEV void commit(uint64_t* bar) {
  asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n"
               ::"r"(smem_u32(bar)) : "memory");
}

// Copy one 512-byte scale-factor block (32 rows x 16 bytes in shared memory,
// described by `sdesc`) into columns taddr..taddr+3 of lanes 0-31, replicated
// into all four 32-lane quarters.
MOE_DEV void cp_sf_block(uint32_t taddr, uint64_t sdesc) {
  asm volatile("tcgen05.cp.cta_group::1.32x128b.warpx4 [%0], %1;\n" ::"r"(taddr), "l"(sdesc)
               : "memory");
}

// D[128 x N] (+)= A[128 x 64] * B[N x 64]^T with E2M1 operands and E8M0 scales
// per 32 elements of K taken from tensor memory (one thread issues).
MOE_DEV void mma_mxf4(uint32_t d, uint64_t adesc, uint64_t bdesc, uint32_t idesc, uint32_t sfa,
                      uint32_t sfb, uint32_t accumulate) {
  asm volatile(
      "{\n\t.reg .pred p;\n\t"
      "setp.ne.b32 p, %6, 0;\n\t"
      "tcgen05.mma.cta_group::1.kind::mxf4.block_scale.block32 [%0], %1, %2, %3, [%4], [%5], p;\n\t}"
      ::"r"(d), "l"(adesc), "l"(bdesc), "r"(idesc), "r"(sfa), "r"(sfb), "r"(accumulate)
      : "memory");
}

// Warp: 32 consecutive fp32 columns of this warp's 32 lanes (lane i gets row
// 32*(warp%4) + i); complete after wait_ld().
MOE_DEV void ld_32cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
      "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]),
        "=r"(r[20]), "=r"(r[21]), "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]),
        "=r"(r[26]), "=r"(r[27]), "=r"(r[28]), "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
      : "r"(taddr)
      : "memory");
}
// Warp: 16 consecutive fp32 columns (r[0..15]); complete after wait_ld().
MOE_DEV void ld_16cols(uint32_t taddr, uint32_t (&r)[32]) {
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 "
      "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
#pragma unroll
  for (int i = 16; i < 32; ++i) r[i] = 0u;
}
MOE_DEV void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory"); }

// --- descriptors ----------------------------------------------------------------
// K-major tile whose rows are 128 bytes with the 128-byte swizzle (as written
// by a tensor TMA with CU_TENSOR_MAP_SWIZZLE_128B), 8-row groups 1024 bytes
// apart. `addr` is the shared address of the first K chunk used by the MMA
// (tile base, 1024-byte aligned, plus 32 bytes per 64 E2M1 elements).
MOE_DEV uint64_t desc_sw128(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(1024 >> 4) << 32) |
         ((uint64_t)1 << 46) | ((uint64_t)2 << 61);
}
// Scale-factor block: 32 rows of 16 bytes, unswizzled, 8-row groups 128 bytes apart.
MOE_DEV uint64_t desc_sf(uint32_t addr) {
  return (uint64_t)((addr & 0x3FFFFu) >> 4) | ((uint64_t)1 << 16) | ((uint64_t)(128 >> 4) << 32) |
         ((uint64_t)1 << 46);
}
// kind::mxf4 with E8M0 scales, M = 128, both operands K-major, scale ids 0.
MOE_DEV uint32_t idesc_mxf4(int N) {
  return (1u << 7) | (1u << 10) | ((uint32_t)(N >> 3) << 17) | (1u << 23) | ((128u >> 4) << 24);
}
MOE_DEV uint32_t idesc_sf_id(uint32_t idesc, uint32_t id) { return idesc | (id << 4) | (id << 29); }

// --- tensor TMA -----------------------------------------------------------------
MOE_DEV void tma_load_2d(void* dst, const CUtensorMap* map, int x, int y, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes "
      "[%0], [%1, {%2, %3}], [%4];\n"
      ::"r"(smem_u32(dst)), "l"(reinterpret_cast<uint64_t>(map)), "r"(x), "r"(y),
        "r"(smem_u32(bar))
      : "memory");
}
// bulk prefetch of global memory into L2 (no completion to wait for):
// address 16-byte aligned, bytes a multiple of 16
MOE_DEV void prefetch_l2(const void* p, uint32_t bytes) {
  asm volatile("cp.async.bulk.prefetch.L2.global [%0], %1;\n" ::"l"(reinterpret_cast<uint64_t>(p)), "r"(bytes)
               : "memory");
}
MOE_DEV void prefetch_map(const CUtensorMap* map) {
  asm volatile("prefetch.tensormap [%0];\n" ::"l"(reinterpret_cast<uint64_t>(map)) : "memory");
}

MOE_DEV void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.release.cta.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar))
               : "memory");
}

// Bounded wait on phase `parity` of `bar` that also gives up as soon as
// another role of the CTA has raised `*abort`. Returns false when it gave up
// (raising `*abort` itself after `limit` tries: about four seconds by
// default).
MOE_DEV bool wait_or_abort(uint64_t* bar, uint32_t parity, volatile int* abort,
                           uint32_t limit = 1u << 22) {
  const uint32_t a = smem_u32(bar);
  for (uint32_t it = 0; it < limit; ++it) {
    uint32_t done;
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2, %3;\n\t"
        "selp.u32 %0, 1, 0, p;\n\t}"
        : "=r"(done) : "r"(a), "r"(parity), "r"(1000u) : "memory");
    if (done) return true;
    if (*abort) return false;
  }
  *abort = 1;
  return false;
}

}  // namespace tc
}  // namespace moe
