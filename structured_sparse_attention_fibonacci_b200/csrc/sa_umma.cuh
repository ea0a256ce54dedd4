// Fifth-generation tensor-core building blocks (sm_100a): tensor-memory
// (TMEM) allocation, tcgen05.mma issued by one thread with operands described
// by shared-memory matrix descriptors, completion through tcgen05.commit on an
// mbarrier, and tcgen05.ld of accumulator rows into registers.
//
// Shared-memory matrix descriptor (64 bits): start address >> 4 in bits
// [0, 14), leading-dimension byte offset >> 4 in [16, 30), stride-dimension
// byte offset >> 4 in [32, 46), the descriptor version 1 in [46, 48), base
// offset 0, and the swizzle mode in [61, 64) (0 none, 2 128-byte).  The
// layouts used here, for 16-bit elements:
//  * K-major, 128-byte swizzle: rows of 64 elements (128 bytes) at a 128-byte
//    pitch, 16-byte chunk c of row r at position c ^ (r & 7) within each
//    1024-byte group of 8 rows (what a tensor copy with 128-byte swizzling
//    writes); stride offset 1024 (next 8 rows); a k step of 16 elements
//    advances the start address by 32 bytes.
//  * MN-major, 128-byte swizzle: the same byte layout read the other way: a
//    row is one k index holding 64 consecutive n (or m) elements; stride offset
//    1024 (next 8 k rows); a k step of 16 advances the start by 2048 bytes.
//  * K-major, no swizzle ("core matrices"): 8 rows x 16 bytes per 128-byte core
//    matrix; leading offset = bytes between the two core matrices of one k
//    step (k 0..7 and 8..15), stride offset = bytes between groups of 8 rows.
//
// Instruction descriptor (kind::f16, 32 bits): accumulator format (1 = fp32)
// in bits [4, 6), A and B formats (0 = fp16) in [7, 10) and [10, 13), A and B
// major-ness (0 K, 1 MN) in bits 15 and 16, N >> 3 in [17, 23), M >> 4 in
// [24, 29).
//
// Accumulator layout (cta_group::1, M = 128): row m of D is TMEM lane m,
// column n is TMEM column (base + n); warp w of the CTA reads lanes
// [32 (w % 4), 32 (w % 4) + 32), one row per thread, with tcgen05.ld.32x32b.
#pragma once

#include <cstdint>

#include "sa_stage.cuh"

namespace sa {
namespace umma {

__host__ __device__ constexpr uint32_t idesc_f16(int M, int N, bool b_mn_major) {
  return (1u << 4) | (0u << 7) | (0u << 10) | (0u << 15) | ((b_mn_major ? 1u : 0u) << 16) |
         ((uint32_t)(N >> 3) << 17) | ((uint32_t)(M >> 4) << 24);
}

constexpr int kSwizzleNone = 0, kSwizzle128 = 2;

__device__ __forceinline__ uint64_t sdesc(uint32_t start, uint32_t lbo, uint32_t sbo, int swz) {
  return (uint64_t)((start >> 4) & 0x3FFFu) | ((uint64_t)((lbo >> 4) & 0x3FFFu) << 16) |
         ((uint64_t)((sbo >> 4) & 0x3FFFu) << 32) | (1ull << 46) | ((uint64_t)swz << 61);
}

// Warp-wide (one full warp): allocate `cols` TMEM columns (a power of two
// >= 32); the base address is written to shared memory at `dst`.
__device__ __forceinline__ void tmem_alloc(uint32_t dst, uint32_t cols) {
  asm volatile("tcgen05.alloc.cta_group::1.sync.aligned.shared::cta.b32 [%0], %1;\n" ::"r"(dst),
               "r"(cols)
               : "memory");
  asm volatile("tcgen05.relinquish_alloc_permit.cta_group::1.sync.aligned;\n" ::: "memory");
}

__device__ __forceinline__ void tmem_dealloc(uint32_t taddr, uint32_t cols) {
  asm volatile("tcgen05.dealloc.cta_group::1.sync.aligned.b32 %0, %1;\n" ::"r"(taddr), "r"(cols)
               : "memory");
}

// Ordering of tcgen05 operations across a CTA barrier.
__device__ __forceinline__ void fence_before_sync() {
  asm volatile("tcgen05.fence::before_thread_sync;\n" ::: "memory");
}
__device__ __forceinline__ void fence_after_sync() {
  asm volatile("tcgen05.fence::after_thread_sync;\n" ::: "memory");
}

// D[tmem] (+)= A[smem] . B[smem]^T (one thread issues).
__device__ __forceinline__ void mma_f16(uint32_t d_tmem, uint64_t a_desc, uint64_t b_desc,
                                        uint32_t idesc, bool accumulate) {
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "setp.ne.b32 p, %4, 0;\n"
      "tcgen05.mma.cta_group::1.kind::f16 [%0], %1, %2, %3, p;\n"
      "}\n" ::"r"(d_tmem),
      "l"(a_desc), "l"(b_desc), "r"(idesc), "r"(accumulate ? 1u : 0u)
      : "memory");
}

// Arrive on `bar` once every tcgen05.mma this thread issued so far completes.
__device__ __forceinline__ void commit(uint64_t* bar) {
  asm volatile(
      "tcgen05.commit.cta_group::1.mbarrier::arrive::one.shared::cluster.b64 [%0];\n" ::"r"(
          stage::smem_u32(bar))
      : "memory");
}

// 16 consecutive fp32 columns of this thread's accumulator row (warp-wide).
__device__ __forceinline__ void ld16(uint32_t taddr, float (&v)[16]) {
  uint32_t r[16];
  asm volatile(
      "tcgen05.ld.sync.aligned.32x32b.x16.b32 {%0,%1,%2,%3,%4,%5,%6,%7,%8,%9,%10,%11,%12,%13,%14,"
      "%15}, [%16];\n"
      : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3]), "=r"(r[4]), "=r"(r[5]), "=r"(r[6]),
        "=r"(r[7]), "=r"(r[8]), "=r"(r[9]), "=r"(r[10]), "=r"(r[11]), "=r"(r[12]), "=r"(r[13]),
        "=r"(r[14]), "=r"(r[15])
      : "r"(taddr)
      : "memory");
  asm volatile("tcgen05.wait::ld.sync.aligned;\n" ::: "memory");
#pragma unroll
  for (int e = 0; e < 16; ++e) v[e] = __uint_as_float(r[e]);
}

}  // namespace umma
}  // namespace sa
