// RoPE pre-pass of the staged kernels ("RoPE before the gather",
// "Depth-Staggered Fibonacci Spacing for Sparse Attention", technical summary,
// Methodology): Y = fp16(RoPE(X) * mul) for every row of a bf16 [units][T][64]
// array, each row rotated at its own position.  The staged kernels then copy
// rotated rows straight from global into shared memory with bulk copies, so
// no per-row rotation work remains inside them.
#include <cuda_fp16.h>

#include "sa_fast_common.cuh"

namespace sa {

namespace {

using namespace fast;

// One thread per (row, RoPE pair-chunk p): dims [8p, 8p+8) pair with
// [32+8p, 32+8p+8).  A finite rotated value that overflows fp16 sets bit 2
// of the error word (the staged kernels' range limit).
__global__ void __launch_bounds__(256) k_rope_rows(const __nv_bfloat16* __restrict__ X,
                                                   const float2* __restrict__ rope, int T,
                                                   long long n_rows, float mul,
                                                   __half* __restrict__ Y, unsigned* err) {
  const long long task = (long long)blockIdx.x * blockDim.x + threadIdx.x;
  if (task >= n_rows * 4) return;
  const long long row = task >> 2;
  const int p = (int)(task & 3);
  const int pos = (int)(row % T);
  const uint4* g = reinterpret_cast<const uint4*>(X + row * kD);
  float x1[8], x2[8];
  unpack8(__ldg(g + p), x1);
  unpack8(__ldg(g + p + 4), x2);
  const float4* cs = reinterpret_cast<const float4*>(rope + (size_t)pos * 32 + 8 * p);
#pragma unroll
  for (int h = 0; h < 8; h += 2) {
    const float4 t = __ldg(cs + h / 2);
    const float a0 = x1[h], b0 = x2[h], a1 = x1[h + 1], b1 = x2[h + 1];
    x1[h] = (a0 * t.x - b0 * t.y) * mul;
    x2[h] = (b0 * t.x + a0 * t.y) * mul;
    x1[h + 1] = (a1 * t.z - b1 * t.w) * mul;
    x2[h + 1] = (b1 * t.z + a1 * t.w) * mul;
  }
  if (half_overflow8(x1) | half_overflow8(x2)) atomicOr(err, 4u);
  uint4* y = reinterpret_cast<uint4*>(Y + row * kD);
  y[p] = pack8_h(x1);
  y[p + 4] = pack8_h(x2);
}

__device__ unsigned g_prep_err;   // bit 2: a rotated value beyond fp16's range

}  // namespace

cudaError_t launch_rope_rows(const void* x, const float2* rope, int T, long long n_rows, float mul,
                             void* y, cudaStream_t st, const char* trace_name) {
  if (n_rows <= 0) return cudaSuccess;
  const long long tasks = n_rows * 4;
  const unsigned grid = (unsigned)((tasks + 255) / 256);
  unsigned* err = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&err), g_prep_err);
  if (e != cudaSuccess) return e;
  trace_mark(trace_name, st, true);
  k_rope_rows<<<grid, 256, 0, st>>>(reinterpret_cast<const __nv_bfloat16*>(x), rope, T, n_rows,
                                    mul, reinterpret_cast<__half*>(y), err);
  trace_mark(trace_name, st, false);
  return cudaGetLastError();
}

cudaError_t prep_read_error(unsigned* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_prep_err, sizeof(unsigned));
  if (e != cudaSuccess || !clear || *out == 0) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_prep_err, &zero, sizeof(unsigned));
}

}  // namespace sa
