// Building blocks of the staged bf16 / head-dim-64 kernels (forward and
// backward): 16-bit packing, the 16-dim lane slices and the 4-lane
// reduce-scatter.  Row staging is in sa_stage.cuh.
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

// Whether any of 8 finite values would overflow fp16 (|x| >= 65520 rounds to
// infinity): the range limit of the 16-bit staged operands.
__device__ __forceinline__ bool half_overflow8(const float* x) {
  bool over = false;
#pragma unroll
  for (int h = 0; h < 8; ++h) over |= isfinite(x[h]) && fabsf(x[h]) >= 65520.f;
  return over;
}

__device__ __forceinline__ uint4 pack8(const float* x) {
  return make_uint4(pack_bf16x2(x[0], x[1]), pack_bf16x2(x[2], x[3]), pack_bf16x2(x[4], x[5]),
                    pack_bf16x2(x[6], x[7]));
}

// Dot product and axpy over a lane's 16 dims with packed fp32 FMAs (two per
// instruction).  The dot product keeps one packed accumulator chain: measured
// on B200 faster than two chains summed at the end (two more adds per call).
__device__ __forceinline__ float dot16(const float (&q)[16], const float (&x)[16]) {
  float2 a = make_float2(0.f, 0.f);
#pragma unroll
  for (int h = 0; h < 16; h += 2)
    a = __ffma2_rn(make_float2(q[h], q[h + 1]), make_float2(x[h], x[h + 1]), a);
  return a.x + a.y;
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

}  // namespace fast
}  // namespace sa
