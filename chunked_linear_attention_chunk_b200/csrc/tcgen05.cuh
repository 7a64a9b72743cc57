// tcgen05.cuh -- 5th-generation tensor core (tcgen05 / TMEM) helpers for sm_100a.
//
// Conventions used by libkda:
//   * MMAs are kind::f16 with bfloat16 operands and float32 accumulation in tensor
//     memory (TMEM), issued by one thread; completion is signalled on an mbarrier with
//     tcgen05.commit.
//   * Operands live in shared memory in the canonical swizzled layouts:
//       K-major,  128-byte swizzle: rows of 64 bf16 (128 B), 16-byte chunks XOR (row & 7),
//                 8-row groups 1024 B apart; K beyond 64 is a further 64-column block.
//       MN-major, 64-byte swizzle:  rows (one per K index) of 32 bf16 (64 B), chunks XOR
//                 ((row >> 1) & 3), 8-row groups 512 B apart.
//       MN-major, 128-byte swizzle: rows of 64 bf16 (128 B) per K index, chunks XOR (row & 7),
//                 8-row groups 1024 B apart; further 64-element MN blocks `lbo` bytes apart.
//   * Accumulator of an M = 128 MMA: row i lives in TMEM lane i, column j in column
//     (base + j); warp w of the CTA reads lanes [32 w, 32 w + 32).
#pragma once

#include <stdint.h>

#include "kda_common.cuh"

namespace kda {
namespace tc {

// ------------------------------------------------------------------ descriptors
enum Swizzle : uint32_t { kSwNone = 0, kSw128 = 2, kSw64 = 4, kSw32 = 6 };

// Shared-memory matrix descriptor (sm_100 format: version 1 in bits 46-47).
__device__ __forceinline__ uint64_t smem_desc(uint32_t saddr, uint32_t lbo_bytes, uint32_t sbo_bytes, Swizzle sw)
{
    uint64_t d = 0;
    d |= (uint64_t)((saddr >> 4) & 0x3FFFu);
    d |= (uint64_t)((lbo_bytes >> 4) & 0x3FFFu) << 16;
    d |= (uint64_t)((sbo_bytes >> 4) & 0x3FFFu) << 32;
    d |= (uint64_t)1 << 46;
    d |= (uint64_t)sw << 61;
    return d;
}

// Instruction descriptor for kind::f16, bf16 x bf16 -> f32, dense.
//   a_mn / b_mn: operand stored MN-major (transposed) instead of K-major.
__host__ __device__ constexpr uint32_t idesc_bf16(int M, int N, bool a_mn, bool b_mn)
{
    return (1u << 4)                      // D format: f32
           | (1u << 7)                    // A format: bf16
           | (1u << 10)                   // B format: bf16
           | ((a_mn ? 1u : 0u) << 15)     // A major
           | ((b_mn ? 1u : 0u) << 16)     // B major
           | ((uint32_t)(N >> 3) << 17)   // N / 8
           | ((uint32_t)(M >> 4) << 24);  // M / 16
}

// ------------------------------------------------------------------ TMEM management
// Allocate `ncols` TMEM columns (power of two >= 32); one full warp calls this.  The
// TMEM base address is written to *slot (shared memory).
__device__ __forceinline__ void tmem_alloc(uint32_t *slot, uint32_t ncols)
{
    asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;" ::"r"(smem_u32(slot)),
                 "r"(ncols)
                 : "memory");
    asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t ncols)
{
    asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;" ::"r"(taddr), "r"(ncols) : "memory");
}

// ------------------------------------------------------------------ MMA and completion
__device__ __forceinline__ void mma_bf16(uint32_t d_tmem, uint64_t adesc, uint64_t bdesc, uint32_t idesc,
                                         uint32_t accumulate)
{
    asm volatile(
        "{\n\t.reg .pred p;\n\t"
        "setp.ne.b32 p, %4, 0;\n\t"
        "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n\t}" ::"r"(d_tmem),
        "l"(adesc), "l"(bdesc), "r"(idesc), "r"(accumulate)
        : "memory");
}

// Arrive once on `bar` when every tcgen05 MMA issued so far by this thread completes.
__device__ __forceinline__ void commit(uint64_t *bar)
{
    asm volatile("tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];" ::"r"(
                     smem_u32(bar))
                 : "memory");
}

__device__ __forceinline__ void fence_before_sync() { asm volatile("tcgen05.fence::before_thread_sync;" ::: "memory"); }
__device__ __forceinline__ void fence_after_sync() { asm volatile("tcgen05.fence::after_thread_sync;" ::: "memory"); }

// Generic-proxy shared-memory writes become visible to the tensor core (async proxy).
__device__ __forceinline__ void fence_smem_to_async() { asm volatile("fence.proxy.async.shared::cta;" ::: "memory"); }

// ------------------------------------------------------------------ TMEM -> registers
// 32 consecutive 32-bit columns of this thread's lane.
__device__ __forceinline__ void ld_32x32b_x32(uint32_t taddr, uint32_t (&r)[32])
{
    asm volatile(
        "tcgen05.ld.sync.aligned.32x32b.x32.b32 "
        "{%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,%15,"
        "%16,%17,%18,%19,%20,%21,%22,%23,%24,%25,%26,%27,%28,%29,%30,%31}, [%32];"
        : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]), "=r"(r[7]),
          "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]), "=r"(r[14]),
          "=r"(r[15]), "=r"(r[16]), "=r"(r[17]), "=r"(r[18]), "=r"(r[19]), "=r"(r[20]), "=r"(r[21]),
          "=r"(r[22]), "=r"(r[23]), "=r"(r[24]), "=r"(r[25]), "=r"(r[26]), "=r"(r[27]), "=r"(r[28]),
          "=r"(r[29]), "=r"(r[30]), "=r"(r[31])
        : "r"(taddr)
        : "memory");
}

__device__ __forceinline__ void wait_ld() { asm volatile("tcgen05.wait::ld.sync.aligned;" ::: "memory"); }

// TMEM address of (lane, column) relative to an allocation base.
__device__ __forceinline__ uint32_t taddr(uint32_t base, uint32_t lane, uint32_t col)
{
    return base + (lane << 16) + col;
}

// ------------------------------------------------------------------ canonical layouts
// Byte offset of element (row, k) in a K-major, 128-byte-swizzled bf16 operand with
// `rows` rows (k < 64 * nblocks); blocks of 64 k-columns are rows*128 bytes apart.
__host__ __device__ constexpr uint32_t kmaj_sw128(int row, int k, int rows)
{
    return (uint32_t)(k >> 6) * rows * 128u + (uint32_t)row * 128u +
           ((uint32_t)(((k & 63) >> 3) ^ (row & 7)) << 4) + (uint32_t)(k & 7) * 2u;
}

// Byte offset of element (k, n) in an MN-major, 64-byte-swizzled bf16 operand with 32
// n-columns (one row of 64 bytes per k).
__host__ __device__ constexpr uint32_t mnmaj_sw64(int k, int n)
{
    return (uint32_t)k * 64u + ((uint32_t)((n >> 3) ^ ((k >> 1) & 3)) << 4) + (uint32_t)(n & 7) * 2u;
}

// Byte offset of element (k, m) in an MN-major, 128-byte-swizzled bf16 operand whose
// mn-extent is split in 64-element blocks of `krows` rows each (blocks krows*128 B apart).
__host__ __device__ constexpr uint32_t mnmaj_sw128(int k, int m, int krows)
{
    return (uint32_t)(m >> 6) * krows * 128u + (uint32_t)k * 128u +
           ((uint32_t)(((m & 63) >> 3) ^ (k & 7)) << 4) + (uint32_t)(m & 7) * 2u;
}

}  // namespace tc
}  // namespace kda
