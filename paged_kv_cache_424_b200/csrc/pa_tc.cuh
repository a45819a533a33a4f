// pa_tc.cuh -- sm_100a tensor-core plumbing for the GQA decode kernel:
// tiled TMA loads, 5th-generation tensor-core MMAs (tcgen05) with their
// accumulators in tensor memory (TMEM), TMEM allocation and loads.
//
// Shared-memory matrix descriptors (PTX ISA, tcgen05 "matrix descriptor"):
//   bits  0-13  start address >> 4
//   bits 16-29  leading-dimension byte offset >> 4
//   bits 32-45  stride-dimension byte offset >> 4
//   bits 46-47  version (1 on sm_100)
//   bits 49-51  base offset (0: every tile here is 1024-byte aligned)
//   bit  52     leading-dimension offset mode (0)
//   bits 61-63  swizzle (2 = 128-byte swizzle)
// With the 128-byte swizzle an "atom" is 8 rows of 128 bytes (1024 bytes)
// whose 16-byte chunks are permuted by XOR with the row index; the TMA's
// SWIZZLE_128B mode writes exactly that pattern when the tile is 1024-byte
// aligned.
//   K-major operand (rows = M or N, the 64 K-elements of an atom row
//   contiguous): SBO = byte distance between 8-row groups, LBO unused (16).
//   MN-major operand (the 64 M/N-elements of an atom row contiguous, rows =
//   K): LBO = byte distance between 64-element M/N atoms, SBO = byte
//   distance between 8-row K groups.
// With one-byte elements (E4M3) an atom row holds 128 elements.
// Instruction descriptor (kind::f16 and kind::f8f6f4): bits 4-5 D format
// (1 = f32), 7-9 A format and 10-12 B format (kind::f16: 0 = f16, 1 = bf16;
// kind::f8f6f4: 0 = E4M3; A and B always the same type here), bit 15 / 16
// A / B major (0 = K, 1 = MN), bits 17-22 N >> 3, bits 24-28 M >> 4.
// One kind::f16 MMA takes K = 16 elements, one kind::f8f6f4 MMA K = 32: 32
// bytes of each K-major row either way.
#pragma once

#include <cuda.h>

#include "pa_common.cuh"

namespace pa {
namespace tc {

__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo, uint32_t sbo) {
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFF);
    d |= (uint64_t)((lbo >> 4) & 0x3FFF) << 16;
    d |= (uint64_t)((sbo >> 4) & 0x3FFF) << 32;
    d |= (uint64_t)1 << 46;   // version
    d |= (uint64_t)2 << 61;   // 128-byte swizzle
    return d;
}

__host__ __device__ constexpr uint32_t instr_desc_f16(bool bf16, bool a_mn_major, int M, int N) {
    return (1u << 4) | ((bf16 ? 1u : 0u) << 7) | ((bf16 ? 1u : 0u) << 10) | ((a_mn_major ? 1u : 0u) << 15) |
           ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// E4M3 x E4M3 -> f32; B K-major, A K-major or MN-major.
__host__ __device__ constexpr uint32_t instr_desc_e4m3(bool a_mn_major, int M, int N) {
    return (1u << 4) | ((a_mn_major ? 1u : 0u) << 15) | ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

// D[tmem] (+)= A[smem] * B[smem], issued by one thread.
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                        bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// The same for E4M3 operands (kind::f8f6f4).
__device__ __forceinline__ void mma_e4m3(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc, uint32_t idesc,
                                         bool accumulate) {
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f8f6f4 [%0], %1, %2, %3, p;\n\t}"
        ::"r"(d_tmem), "l"(a_desc), "l"(b_desc), "r"(idesc), "r"((uint32_t)accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 operation this thread issued so
// far has completed.
__device__ __forceinline__ void commit(uint64_t *bar) {
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(smem_addr(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// TMEM allocation (one full warp; writes the base address to *dst).
__device__ __forceinline__ void tmem_alloc(uint32_t *dst, uint32_t ncols) {
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_addr(dst)), "r"(ncols)
                 : "memory");
}
// Give up this CTA's right to allocate TMEM (it allocates once).  While a CTA
// holds that right the next CTA cannot be placed on the SM, so a CTA must
// release it right after its one allocation to keep several CTAs per SM.
__device__ __forceinline__ void tmem_relinquish() {
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}
__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols) {
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// 16 consecutive 32-bit columns of this thread's TMEM lane (warp w reads
// lanes 32 (w % 4) .. + 31; the lane field of taddr names the quadrant base).
__device__ __forceinline__ void tmem_ld16(uint32_t taddr, float *v) {
    uint32_t r[16];
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15}, [%16];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]), "=r"(r[15])
        : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 16; ++i) v[i] = __uint_as_float(r[i]);
}

// 8 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld8(uint32_t taddr, float *v) {
    uint32_t r[8];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x8.b32 {%0,%1,%2,%3,%4,%5,%6,%7}, [%8];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 8; ++i) v[i] = __uint_as_float(r[i]);
}

// 4 consecutive 32-bit columns of this thread's TMEM lane.
__device__ __forceinline__ void tmem_ld4(uint32_t taddr, float *v) {
    uint32_t r[4];
    asm volatile("tcgen05.ld.sync.aligned.32x32b.x4.b32 {%0,%1,%2,%3}, [%4];"
                 : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
                 : "r"(taddr));
    asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory");
#pragma unroll
    for (int i = 0; i < 4; ++i) v[i] = __uint_as_float(r[i]);
}

// The first N (4, 8 or 16) columns of this thread's TMEM lane.
template <int N>
__device__ __forceinline__ void tmem_ld(uint32_t taddr, float *v) {
    static_assert(N == 4 || N == 8 || N == 16, "4, 8 or 16 columns");
    if constexpr (N == 4) tmem_ld4(taddr, v);
    else if constexpr (N == 8) tmem_ld8(taddr, v);
    else tmem_ld16(taddr, v);
}

// 2-D tiled TMA load of box (x, y) of `tmap` into shared memory, completing
// on `bar`.  No multicast.  x * element size must be a multiple of 16 bytes.
__device__ __forceinline__ void tma_load_2d(void *dst, const CUtensorMap *tmap, int x, int y, uint64_t *bar) {
    asm volatile(
        "cp.async.bulk.tensor.2d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], [%1, {%2, %3}], [%4];" ::"r"(
            smem_addr(dst)),
        "l"(reinterpret_cast<uint64_t>(tmap)), "r"(x), "r"(y), "r"(smem_addr(bar))
        : "memory");
}

// Byte offset of element (row, col) of a 128-byte-swizzled K-major tile
// region whose rows are 128 bytes (64 16-bit elements).
__device__ __forceinline__ uint32_t sw128_offset(int row, int col) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((col >> 3) ^ row) & 7) << 4) + (col & 7) * 2);
}

// The same for a tile of one-byte elements (rows of 128 elements).
__device__ __forceinline__ uint32_t sw128_offset8(int row, int col) {
    return (uint32_t)((row >> 3) * 1024 + (row & 7) * 128 + ((((col >> 4) ^ row) & 7) << 4) + (col & 15));
}

}  // namespace tc
}  // namespace pa
