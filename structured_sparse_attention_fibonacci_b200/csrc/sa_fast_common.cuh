// Building blocks of the staged bf16 / head-dim-64 kernels (forward and
// backward): the row ring in shared memory, its loads and stores, the 16-dim
// lane slices and the 4-lane reduce-scatter.  See sa_fast.cu for the layout.
#pragma once

#include "sa_device.cuh"
#include "sa_internal.h"
#include <cuda_fp16.h>

namespace sa {
namespace fast {

constexpr int kD = 64;
constexpr int kChunks = 8;             // 16-byte chunks per bf16 row
constexpr int kFastM = 128;            // rows (queries or keys) per CTA = threads per CTA


__device__ __forceinline__ void unpack8(const uint4 u, float* x) {
  x[0] = bf16lo(u.x); x[1] = bf16hi(u.x); x[2] = bf16lo(u.y); x[3] = bf16hi(u.y);
  x[4] = bf16lo(u.z); x[5] = bf16hi(u.z); x[6] = bf16lo(u.w); x[7] = bf16hi(u.w);
}

// Rotated K rows are staged as fp16 of (RoPE(K) * kKeyStage): fp16 keeps 8x
// finer rounding than bf16 (2^-11 vs 2^-8 relative), and the 2^-8 factor
// moves its range to |RoPE(K)| < 65504 * 256 (about 1.7e7).  Queries carry
// the inverse factor, so scores come out unscaled.
constexpr float kKeyStage = 1.f / 256.f;
constexpr float kKeyUnstage = 256.f;

__device__ __forceinline__ void unpack8_h(const uint4 u, float* x) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const float2 f = __half22float2(*reinterpret_cast<const __half2*>(&w[e]));
    x[2 * e] = f.x;
    x[2 * e + 1] = f.y;
  }
}

__device__ __forceinline__ uint4 pack8_h(const float* x) {
  uint32_t w[4];
#pragma unroll
  for (int e = 0; e < 4; ++e) {
    const __half2 h = __floats2half2_rn(x[2 * e], x[2 * e + 1]);
    w[e] = *reinterpret_cast<const uint32_t*>(&h);
  }
  return make_uint4(w[0], w[1], w[2], w[3]);
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

__device__ __forceinline__ int swz(int slot) { return (slot >> 2) & 7; }

// This lane's 16 dims of ring slot `slot` (F16: a staged rotated-K row).
template <bool F16 = false>
__device__ __forceinline__ void ring_load(const uint4* ring, int slot, int c, float (&x)[16]) {
  const int s = swz(slot);
  if (F16) {
    unpack8_h(ring[slot * kChunks + (c ^ s)], x);
    unpack8_h(ring[slot * kChunks + ((c + 4) ^ s)], x + 8);
  } else {
    unpack8(ring[slot * kChunks + (c ^ s)], x);
    unpack8(ring[slot * kChunks + ((c + 4) ^ s)], x + 8);
  }
}

// Dot product and axpy over a lane's 16 dims with packed fp32 FMAs
// (two per instruction).
__device__ __forceinline__ float dot16(const float (&q)[16], const float (&x)[16]) {
  float2 a = make_float2(0.f, 0.f), b = make_float2(0.f, 0.f);
#pragma unroll
  for (int h = 0; h < 16; h += 4) {
    a = __ffma2_rn(make_float2(q[h], q[h + 1]), make_float2(x[h], x[h + 1]), a);
    b = __ffma2_rn(make_float2(q[h + 2], q[h + 3]), make_float2(x[h + 2], x[h + 3]), b);
  }
  return (a.x + b.x) + (a.y + b.y);
}

__device__ __forceinline__ void axpy16(float (&o)[16], float p, const float (&x)[16]) {
  const float2 pp = make_float2(p, p);
#pragma unroll
  for (int h = 0; h < 16; h += 2) {
    const float2 r = __ffma2_rn(pp, make_float2(x[h], x[h + 1]), make_float2(o[h], o[h + 1]));
    o[h] = r.x;
    o[h + 1] = r.y;
  }
}

// p[q][l] are partial sums held by the 4 lanes of a group (lane c = 2*hi+lo);
// out[l] receives the sum over the 4 lanes of p[c][l].
template <int L>
__device__ __forceinline__ void reduce_scatter4(const float (&p)[4][L], float (&out)[L], int c) {
  const bool hi = (c >> 1) & 1, lo = c & 1;
  float r[2][L];
#pragma unroll
  for (int j = 0; j < 2; ++j)
#pragma unroll
    for (int l = 0; l < L; ++l) {
      const float keep = hi ? p[2 + j][l] : p[j][l];
      const float send = hi ? p[j][l] : p[2 + j][l];
      r[j][l] = keep + __shfl_xor_sync(0xffffffffu, send, 2);
    }
#pragma unroll
  for (int l = 0; l < L; ++l) {
    const float keep = lo ? r[1][l] : r[0][l];
    const float send = lo ? r[0][l] : r[1][l];
    out[l] = keep + __shfl_xor_sync(0xffffffffu, send, 1);
  }
}

// Stage rows [a, b) of src (bf16 [T][64]) into ring slots row % ring_rows,
// rotating K rows by RoPE at their own position.  One task = one row and one
// RoPE pair-chunk p (dims [8p, 8p+8) and [32+8p, 32+8p+8)).
template <bool ROT>
__device__ __forceinline__ void stage_rows(uint4* ring, int ring_rows, const __nv_bfloat16* src,
                                           const float2* rope, int a, int b) {
  const int n = (b - a) * 4;
  for (int task = threadIdx.x; task < n; task += blockDim.x) {
    const int row = a + (task >> 2), p = task & 3;
    const uint4* g = reinterpret_cast<const uint4*>(src + (size_t)row * kD);
    uint4 u0 = __ldg(g + p), u1 = __ldg(g + p + 4);
    if (ROT) {
      float x1[8], x2[8];
      unpack8(u0, x1);
      unpack8(u1, x2);
      const float4* cs = reinterpret_cast<const float4*>(rope + (size_t)row * 32 + 8 * p);
#pragma unroll
      for (int h = 0; h < 8; h += 2) {
        const float4 t = __ldg(cs + h / 2);
        float a0 = x1[h], b0 = x2[h], a1 = x1[h + 1], b1 = x2[h + 1];
        x1[h] = (a0 * t.x - b0 * t.y) * kKeyStage;  x2[h] = (b0 * t.x + a0 * t.y) * kKeyStage;
        x1[h + 1] = (a1 * t.z - b1 * t.w) * kKeyStage;
        x2[h + 1] = (b1 * t.z + a1 * t.w) * kKeyStage;
      }
      u0 = pack8_h(x1);
      u1 = pack8_h(x2);
    }
    const int slot = row & (ring_rows - 1);   // ring_rows is a power of two
    const int s = swz(slot);
    ring[slot * kChunks + (p ^ s)] = u0;
    ring[slot * kChunks + ((p + 4) ^ s)] = u1;
  }
}

// Asynchronous 16-byte global -> shared copy (completes at cp_async_wait_all).
__device__ __forceinline__ void cp_async16(void* smem_dst, const void* gsrc) {
  const unsigned d = (unsigned)__cvta_generic_to_shared(smem_dst);
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16;\n" ::"r"(d), "l"(gsrc) : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// Copy rows [a, b) of a bf16 [T][64] array into ring slots row & (ring_rows-1),
// every 16-byte chunk in flight at once (all rows here are < T).  The caller
// synchronises the CTA afterwards.
__device__ __forceinline__ void stage_copy(uint4* ring, int ring_rows, const __nv_bfloat16* src,
                                           int a, int b) {
  const int n = (b - a) * kChunks;
  for (int task = threadIdx.x; task < n; task += blockDim.x) {
    const int row = a + (task >> 3), ch = task & 7;
    const int slot = row & (ring_rows - 1);
    cp_async16(ring + slot * kChunks + (ch ^ swz(slot)),
               reinterpret_cast<const uint4*>(src + (size_t)row * kD) + ch);
  }
  cp_async_wait_all();
}

// Stage rows [a, b) (all < T) rotated by RoPE at their own positions, times
// `mul`, as fp16 (OUT_F16: keys) or bf16 (queries).  Every raw row chunk is
// first copied asynchronously into its ring slot; meanwhile each thread loads
// the cos/sin of the first row of its run and the per-row angle step theta_j
// (table row 1) for its RoPE pair-chunk p; after the copies land (one CTA
// barrier) each thread rotates its run of consecutive rows in place, stepping
// the angle by theta_j per row (a run is at most a few rows, so the fp32
// recurrence stays within ~1e-6 of the table).  The caller synchronises after.
template <bool OUT_F16>
__device__ __forceinline__ void stage_rotate(uint4* ring, int ring_rows, const __nv_bfloat16* src,
                                             const float2* rope, int a, int b, float mul) {
  const int n = b - a;
  if (n <= 0) return;
  for (int task = threadIdx.x; task < n * kChunks; task += blockDim.x) {
    const int row = a + (task >> 3), ch = task & 7;
    const int slot = row & (ring_rows - 1);
    cp_async16(ring + slot * kChunks + (ch ^ swz(slot)),
               reinterpret_cast<const uint4*>(src + (size_t)row * kD) + ch);
  }
  const int runs = blockDim.x >> 2;
  const int L = (n + runs - 1) / runs;
  const int p = threadIdx.x & 3;
  const int r0 = a + (int)(threadIdx.x >> 2) * L;
  const int r1 = min(r0 + L, b);
  float2 cs[8];
  if (r0 < r1) {
    const float4* g0 = reinterpret_cast<const float4*>(rope + (size_t)r0 * 32 + 8 * p);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 u = __ldg(g0 + h);
      cs[2 * h] = make_float2(u.x, u.y); cs[2 * h + 1] = make_float2(u.z, u.w);
    }
  }
  cp_async_wait_all();
  __syncthreads();
  if (r0 >= r1) return;
  float2 st[8];      // the same table row for every run: cached after first use
  {
    const float4* g1 = reinterpret_cast<const float4*>(rope + 32 + 8 * p);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 w = __ldg(g1 + h);
      st[2 * h] = make_float2(w.x, w.y); st[2 * h + 1] = make_float2(w.z, w.w);
    }
  }
  for (int row = r0; row < r1; ++row) {
    const int slot = row & (ring_rows - 1);
    const int sw = swz(slot);
    uint4* c0 = ring + slot * kChunks + (p ^ sw);
    uint4* c1 = ring + slot * kChunks + ((p + 4) ^ sw);
    float x1[8], x2[8];
    unpack8(*c0, x1);
    unpack8(*c1, x2);
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float a0 = x1[h], b0 = x2[h];
      x1[h] = (a0 * cs[h].x - b0 * cs[h].y) * mul;
      x2[h] = (b0 * cs[h].x + a0 * cs[h].y) * mul;
      const float c2 = cs[h].x * st[h].x - cs[h].y * st[h].y;
      cs[h].y = cs[h].y * st[h].x + cs[h].x * st[h].y;
      cs[h].x = c2;
    }
    *c0 = OUT_F16 ? pack8_h(x1) : pack8(x1);
    *c1 = OUT_F16 ? pack8_h(x2) : pack8(x2);
  }
}

// Sink rows 0..S-1 into a plain (unswizzled) buffer.
template <bool ROT>
__device__ __forceinline__ void stage_sinks(uint4* buf, int S, const __nv_bfloat16* src,
                                            const float2* rope) {
  for (int task = threadIdx.x; task < S * 4; task += blockDim.x) {
    const int row = task >> 2, p = task & 3;
    const uint4* g = reinterpret_cast<const uint4*>(src + (size_t)row * kD);
    uint4 u0 = __ldg(g + p), u1 = __ldg(g + p + 4);
    if (ROT) {
      float x1[8], x2[8];
      unpack8(u0, x1);
      unpack8(u1, x2);
      const float4* cs = reinterpret_cast<const float4*>(rope + (size_t)row * 32 + 8 * p);
#pragma unroll
      for (int h = 0; h < 8; h += 2) {
        const float4 t = __ldg(cs + h / 2);
        float a0 = x1[h], b0 = x2[h], a1 = x1[h + 1], b1 = x2[h + 1];
        x1[h] = (a0 * t.x - b0 * t.y) * kKeyStage;  x2[h] = (b0 * t.x + a0 * t.y) * kKeyStage;
        x1[h + 1] = (a1 * t.z - b1 * t.w) * kKeyStage;
        x2[h + 1] = (b1 * t.z + a1 * t.w) * kKeyStage;
      }
      u0 = pack8_h(x1);
      u1 = pack8_h(x2);
    }
    buf[row * kChunks + p] = u0;
    buf[row * kChunks + p + 4] = u1;
  }
}

template <bool F16 = false>
__device__ __forceinline__ void sink_load(const uint4* buf, int s, int c, float (&x)[16]) {
  if (F16) {
    unpack8_h(buf[s * kChunks + c], x);
    unpack8_h(buf[s * kChunks + c + 4], x + 8);
  } else {
    unpack8(buf[s * kChunks + c], x);
    unpack8(buf[s * kChunks + c + 4], x + 8);
  }
}

}  // namespace fast
}  // namespace sa
