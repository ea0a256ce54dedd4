// Tensor-core building blocks of the staged kernels: warp-level mma.sync
// (m16n8k16 / m16n8k8, fp32 accumulate), ldmatrix fragment loads from a
// 128-byte-swizzled row ring, and 3-D tensor-map (TMA) staging of 8-row boxes.
//
// Swizzled ring.  Row r of a 16-bit [T][64] array lives in slot
// s = r mod rows (rows a multiple of 16) at byte s * 128, and its 16-byte
// chunk c at position c ^ (s & 7): the layout the tensor copy writes with
// 128-byte swizzling into a 1024-byte-aligned ring.  Eight consecutive rows
// then put any one chunk in eight different bank groups, so an ldmatrix of
// an 8 x 8 tile (eight rows, one chunk each) is conflict-free.  Boxes are 8
// rows starting at a row that is a multiple of 8 (one 1024-byte swizzle atom
// per box); rows outside [0, T) arrive zero-filled.
//
// The mma wrappers are plain (non-volatile) asm: pure register operations the
// compiler may schedule; ldmatrix stays volatile (it reads shared memory) and
// callers issue a tile's loads before its mma chain.
//
// Fragment layouts (PTX mma.m16n8k16, row-major A, column-major B), lane
// l = 4 g + t:  A regs: (g, 2t..2t+1), (g+8, 2t..2t+1), (g, 2t+8..), (g+8, 2t+8..);
// B regs: k = 2t..2t+1 and 2t+8..2t+9 of column g; C: (g, 2t), (g, 2t+1),
// (g+8, 2t), (g+8, 2t+1).
#pragma once

#include <cuda.h>
#include <cuda_fp16.h>

#include "sa_stage.cuh"

namespace sa {
namespace tc {

using stage::Stager;

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0,%1,%2,%3}, [%4];\n"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

__device__ __forceinline__ void mma_f16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                        uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, {%8,%9}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

__device__ __forceinline__ void mma_bf16(float (&c)[4], const uint32_t (&a)[4], uint32_t b0,
                                         uint32_t b1) {
  asm(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5,%6,%7}, "
      "{%8,%9}, {%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// m16n8k8: A regs (g, 2t..2t+1), (g+8, 2t..2t+1); B reg k = 2t..2t+1 of column g.
__device__ __forceinline__ void mma_bf16_k8(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.bf16.bf16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ void mma_f16_k8(float (&c)[4], uint32_t a0, uint32_t a1, uint32_t b0) {
  asm(
      "mma.sync.aligned.m16n8k8.row.col.f32.f16.f16.f32 {%0,%1,%2,%3}, {%4,%5}, {%6}, "
      "{%0,%1,%2,%3};\n"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a0), "r"(a1), "r"(b0));
}

__device__ __forceinline__ uint32_t pack_h2(float lo, float hi) {
  const __half2 h = __floats2half2_rn(lo, hi);
  return *reinterpret_cast<const uint32_t*>(&h);
}

// Two fp32 values as a bf16 pair rounded to nearest (hi) plus the bf16 pair of
// what that rounding left (lo): hi + lo holds each value to about 2^-17 of
// itself, where hi alone is off by up to 2^-9.  The P.V products run on
// bf16 tensor cores (V is bf16); feeding them both halves of the weights keeps
// the output's error at fp32-accumulation level.
__device__ __forceinline__ void split_bf16x2(float a, float b, uint32_t& hi, uint32_t& lo) {
  const __nv_bfloat162 h = __floats2bfloat162_rn(a, b);
  const float2 hf = __bfloat1622float2(h);
  const __nv_bfloat162 l = __floats2bfloat162_rn(a - hf.x, b - hf.y);
  hi = *reinterpret_cast<const uint32_t*>(&h);
  lo = *reinterpret_cast<const uint32_t*>(&l);
}

// A ring of `rows` 128-byte slots at shared address `base`.  Slots are
// rows modulo `rows`: with POW2 (rows a power of two) a mask; otherwise a
// multiply-high by inv = floor((2^32 - 1) / rows) (the quotient is exact or
// one short, which one subtraction corrects) after adding bias = 64 rows, a
// multiple of rows that makes every row the kernels stage (at least
// -(W + 143)) non-negative.
struct Ring {
  uint32_t base;
  int rows;
  uint32_t inv;
  int bias;
};

__host__ __device__ __forceinline__ Ring make_ring(uint32_t base, int rows) {
  Ring r;
  r.base = base;
  r.rows = rows;
  r.inv = 0xFFFFFFFFu / (uint32_t)rows;
  r.bias = 64 * rows;
  return r;
}

template <bool POW2>
__device__ __forceinline__ int ring_slot(const Ring& r, int row) {
  if (POW2) return row & (r.rows - 1);
  const uint32_t x = (uint32_t)(row + r.bias);
  const int s = (int)(x - __umulhi(x, r.inv) * (uint32_t)r.rows);
  return s >= r.rows ? s - r.rows : s;
}

// Shared address of 16-byte chunk `ch` of row `row`.
template <bool POW2>
__device__ __forceinline__ uint32_t swz_addr(const Ring& r, int row, int ch) {
  const int slot = ring_slot<POW2>(r, row);
  return r.base + (uint32_t)(slot * 128 + ((ch ^ (slot & 7)) << 4));
}

// One 8-row box of a 3-D [units][T][64] 16-bit tensor map (row coordinate may
// be negative or >= T: zero fill) into shared memory at dst (1024-aligned).
__device__ __forceinline__ void tma_rows8(uint32_t dst, const CUtensorMap* map, int row, int unit,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.tensor.3d.shared::cluster.global.tile.mbarrier::complete_tx::bytes [%0], "
      "[%1, {%2, %3, %4}], [%5];\n" ::"r"(dst),
      "l"(reinterpret_cast<uint64_t>(map)), "r"(0), "r"(row), "r"(unit),
      "r"(stage::smem_u32(bar))
      : "memory");
}

// Register (thread 0) and issue the copies of rows [a, b) (multiples of 8,
// b - a <= ring rows) of `unit` into the ring (a box of 8 rows never wraps:
// rows is a multiple of 8).  Completes on the round's barrier
// (stage::stage_commit_wait).
template <bool POW2>
__device__ __forceinline__ void stage_tiles(Stager& s, const Ring& ring, const CUtensorMap* map,
                                            int unit, int a, int b) {
#ifdef SA_DEBUG_BOUNDS
  if (b - a > ring.rows || (a & 7) || (b & 7)) {   // beyond the ring, or not whole boxes
    if (threadIdx.x == 0) atomicOr(s.err, stage::kErrBounds);
    return;
  }
#endif
  stage::dbg_staged(s, ring.rows, a, b);
  if (threadIdx.x != 0 || a >= b) return;
  stage::mbar_expect_tx(s.bar, (uint32_t)(b - a) * 128u);
  for (int r = a; r < b; r += 8)
    tma_rows8(ring.base + (uint32_t)ring_slot<POW2>(ring, r) * 128u, map, r, unit, s.bar);
}

// B fragments of one n tile of A . X^T for 8 swizzled ring rows row0 ..
// row0 + 7 of a 16-bit [T][64] array: k steps 0..3 (dims 16 ks ..) as
// b[kp][0..1] (k step 2 kp) and b[kp][2..3] (k step 2 kp + 1).
template <bool POW2>
__device__ __forceinline__ void qk_load(const Ring& ring, int row0, int lane,
                                        uint32_t (&b)[2][4]) {
  int slot = ring_slot<POW2>(ring, row0) + (lane & 7);
  if (slot >= ring.rows) slot -= ring.rows;
  const uint32_t base = ring.base + (uint32_t)slot * 128u;
  const int x = slot & 7, m = lane >> 3;
  ldsm_x4(base + (uint32_t)((m ^ x) << 4), b[0]);
  ldsm_x4(base + (uint32_t)(((4 + m) ^ x) << 4), b[1]);
}

__device__ __forceinline__ int floor8(int x) { return x & ~7; }
__device__ __forceinline__ int ceil8(int x) { return (x + 7) & ~7; }
__device__ __forceinline__ int floor16(int x) { return x & ~15; }

}  // namespace tc

// Host: a 3-D tensor map over a 16-bit [units][T][64] array (boxes of 8 rows,
// 128-byte swizzle, zero fill out of bounds).  sa_tmap.cu.
cudaError_t make_rows_map(CUtensorMap* map, const void* base, int T, long long units);

}  // namespace sa
