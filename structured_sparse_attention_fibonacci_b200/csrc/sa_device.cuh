// Device helpers shared by the sparse-attention kernels.
//
// Method: "Depth-Staggered Fibonacci Spacing for Sparse Attention" (C. A.
// Capps), technical summary, Methodology ("Attended set", "Scaling",
// "Implementation"). The conventions implemented here are spelled out in
// include/sparse_attn.h.
#pragma once

#include <cuda_bf16.h>
#include <cuda_runtime.h>
#include <math.h>
#include <stdint.h>

#include "sparse_attn.h"

namespace sa {

// ---- offset geometry ("Scaling": d_k = alpha * f_k) -----------------------
// d_k is one IEEE fp32 product (no contraction); floor/ceil on that float.
struct OffGeo {
  int lo;     // floor(d)
  int c;      // ceil(d): the member exists for query i iff i - c >= 0
  float w;    // d - lo (exact)
  float wa;   // 1 - w
  int ok;     // d in [0, 2^24); otherwise the layer's outputs are NaN
  int f;
};

__device__ __forceinline__ OffGeo offset_geometry(float alpha, int f) {
  OffGeo g;
  const float d = __fmul_rn(alpha, (float)f);
  g.f = f;
  g.ok = (d >= 0.f) && (d < 16777216.f);
  const float fl = g.ok ? floorf(d) : 0.f;
  g.lo = (int)fl;
  g.c = g.ok ? (int)ceilf(d) : 0;
  g.w = g.ok ? __fsub_rn(d, fl) : 0.f;
  g.wa = __fsub_rn(1.f, g.w);
  return g;
}

// ---- element conversion -----------------------------------------------------
template <typename T> struct Elt;
template <> struct Elt<float> {
  static constexpr int kBytes = 4;
};
template <> struct Elt<__nv_bfloat16> {
  static constexpr int kBytes = 2;
};

__device__ __forceinline__ float bf16lo(uint32_t u) { return __uint_as_float(u << 16); }
__device__ __forceinline__ float bf16hi(uint32_t u) { return __uint_as_float(u & 0xffff0000u); }

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 h = __floats2bfloat162_rn(lo, hi);  // round to nearest even
  return *reinterpret_cast<uint32_t*>(&h);
}

// Load N consecutive elements starting at p (aligned to N * sizeof(T) bytes)
// into fp32 registers, with the widest vector loads that the alignment allows.
template <typename T, int N>
__device__ __forceinline__ void load_row(const T* __restrict__ p, float (&out)[N]) {
  constexpr int kBytes = N * Elt<T>::kBytes;
  if constexpr (kBytes % 16 == 0) {
#pragma unroll
    for (int v = 0; v < kBytes / 16; ++v) {
      const uint4 u = __ldg(reinterpret_cast<const uint4*>(p) + v);
      const uint32_t w[4] = {u.x, u.y, u.z, u.w};
      if constexpr (sizeof(T) == 4) {
#pragma unroll
        for (int e = 0; e < 4; ++e) out[v * 4 + e] = __uint_as_float(w[e]);
      } else {
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          out[v * 8 + 2 * e] = bf16lo(w[e]);
          out[v * 8 + 2 * e + 1] = bf16hi(w[e]);
        }
      }
    }
  } else if constexpr (kBytes == 8) {
    const uint2 u = __ldg(reinterpret_cast<const uint2*>(p));
    if constexpr (sizeof(T) == 4) {
      out[0] = __uint_as_float(u.x);
      out[1] = __uint_as_float(u.y);
    } else {
      out[0] = bf16lo(u.x); out[1] = bf16hi(u.x);
      out[2] = bf16lo(u.y); out[3] = bf16hi(u.y);
    }
  } else if constexpr (kBytes == 4) {
    const uint32_t u = __ldg(reinterpret_cast<const unsigned int*>(p));
    if constexpr (sizeof(T) == 4) {
      out[0] = __uint_as_float(u);
    } else {
      out[0] = bf16lo(u); out[1] = bf16hi(u);
    }
  } else {
    static_assert(kBytes == 2, "unsupported vector width");
    const unsigned short u = __ldg(reinterpret_cast<const unsigned short*>(p));
    out[0] = __uint_as_float(((uint32_t)u) << 16);
  }
}

// Store N consecutive elements (fp32 -> T with round-to-nearest-even).
template <typename T, int N>
__device__ __forceinline__ void store_row(T* __restrict__ p, const float (&in)[N]) {
  if constexpr (sizeof(T) == 4) {
    if constexpr (N % 4 == 0) {
#pragma unroll
      for (int v = 0; v < N / 4; ++v)
        reinterpret_cast<float4*>(p)[v] = make_float4(in[4 * v], in[4 * v + 1], in[4 * v + 2], in[4 * v + 3]);
    } else if constexpr (N == 2) {
      reinterpret_cast<float2*>(p)[0] = make_float2(in[0], in[1]);
    } else {
#pragma unroll
      for (int e = 0; e < N; ++e) reinterpret_cast<float*>(p)[e] = in[e];
    }
  } else {
    if constexpr (N % 8 == 0) {
#pragma unroll
      for (int v = 0; v < N / 8; ++v)
        reinterpret_cast<uint4*>(p)[v] = make_uint4(
            pack_bf16x2(in[8 * v], in[8 * v + 1]), pack_bf16x2(in[8 * v + 2], in[8 * v + 3]),
            pack_bf16x2(in[8 * v + 4], in[8 * v + 5]), pack_bf16x2(in[8 * v + 6], in[8 * v + 7]));
    } else if constexpr (N == 4) {
      reinterpret_cast<uint2*>(p)[0] = make_uint2(pack_bf16x2(in[0], in[1]), pack_bf16x2(in[2], in[3]));
    } else if constexpr (N == 2) {
      reinterpret_cast<uint32_t*>(p)[0] = pack_bf16x2(in[0], in[1]);
    } else {
      static_assert(N == 1, "unsupported vector width");
      reinterpret_cast<__nv_bfloat16*>(p)[0] = __float2bfloat16_rn(in[0]);
    }
  }
}

// ---- RoPE on lane-held pairs ("RoPE before the gather") ---------------------
// A lane holds x1[h] = x[j0 + h] and x2[h] = x[D/2 + j0 + h] for h < N; cs[h] =
// (cos, sin) of pos * theta_{j0+h}. Forward rotation and its transpose.
template <int N>
__device__ __forceinline__ void rope_fwd(float (&x1)[N], float (&x2)[N], const float2 (&cs)[N]) {
#pragma unroll
  for (int h = 0; h < N; ++h) {
    const float a = x1[h], b = x2[h];
    x1[h] = a * cs[h].x - b * cs[h].y;
    x2[h] = b * cs[h].x + a * cs[h].y;
  }
}

template <int N>
__device__ __forceinline__ void rope_bwd(float (&x1)[N], float (&x2)[N], const float2 (&cs)[N]) {
#pragma unroll
  for (int h = 0; h < N; ++h) {
    const float a = x1[h], b = x2[h];
    x1[h] = a * cs[h].x + b * cs[h].y;
    x2[h] = b * cs[h].x - a * cs[h].y;
  }
}

template <int N>
__device__ __forceinline__ void load_cs(const float2* __restrict__ p, float2 (&cs)[N]) {
  if constexpr (N % 2 == 0) {
#pragma unroll
    for (int v = 0; v < N / 2; ++v) {
      const float4 u = __ldg(reinterpret_cast<const float4*>(p) + v);
      cs[2 * v] = make_float2(u.x, u.y);
      cs[2 * v + 1] = make_float2(u.z, u.w);
    }
  } else {
#pragma unroll
    for (int h = 0; h < N; ++h) cs[h] = __ldg(p + h);
  }
}

// Sum over the 8 lanes of a lane group (lanes 8g .. 8g+7); every lane of the
// warp must call it.
__device__ __forceinline__ float group8_sum(float v) {
  v += __shfl_xor_sync(0xffffffffu, v, 4);
  v += __shfl_xor_sync(0xffffffffu, v, 2);
  v += __shfl_xor_sync(0xffffffffu, v, 1);
  return v;
}

}  // namespace sa
