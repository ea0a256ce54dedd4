// Throughput probe of the CUDA cores' fp32 FMA pipe: the peak of the ALU
// roofline that the CUDA-core kernels (the far offsets' gathers are diagonal
// dot products and axpys, not dense contractions) are held against.
//
// Every thread runs kChains independent FMA chains of `iters` steps on
// registers only, either scalar fma.rn.f32 or packed fma.rn.f32x2 (two FMAs
// per instruction).  No memory traffic inside the loop; one store per thread
// at the end keeps the chains live.  FLOPs per launch:
//   blocks * threads * iters * kChains * 2 (FMA) * (packed ? 2 : 1).
#include "sa_internal.h"
#include "sparse_attn.h"

namespace sa {
namespace {

constexpr int kChains = 8;

template <bool PACKED>
__global__ void __launch_bounds__(256) k_fma_probe(float* out, int iters, float a, float b) {
  if (PACKED) {
    float2 x[kChains];
#pragma unroll
    for (int j = 0; j < kChains; ++j) x[j] = make_float2(threadIdx.x + j, j - 1.f);
    const float2 aa = make_float2(a, a), bb = make_float2(b, b);
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int j = 0; j < kChains; ++j) x[j] = __ffma2_rn(x[j], aa, bb);
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kChains; ++j) s += x[j].x + x[j].y;
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  } else {
    float x[kChains];
#pragma unroll
    for (int j = 0; j < kChains; ++j) x[j] = threadIdx.x + j;
    for (int i = 0; i < iters; ++i) {
#pragma unroll
      for (int j = 0; j < kChains; ++j) x[j] = fmaf(x[j], a, b);
    }
    float s = 0.f;
#pragma unroll
    for (int j = 0; j < kChains; ++j) s += x[j];
    out[blockIdx.x * blockDim.x + threadIdx.x] = s;
  }
}

}  // namespace
}  // namespace sa

extern "C" sa_status sparse_attn_diag_fma_probe(int32_t blocks, int32_t threads, int32_t iters,
                                                int32_t packed, float* out, void* stream) {
  if (blocks < 1 || threads < 32 || threads > 256 || threads % 32 || iters < 1 || !out)
    return SA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // a = 1 - 2^-20 and b = 2^-21 keep every chain finite for any iteration count
  const float a = 0.99999905f, b = 4.76837158e-7f;
  if (packed)
    sa::k_fma_probe<true><<<blocks, threads, 0, st>>>(out, iters, a, b);
  else
    sa::k_fma_probe<false><<<blocks, threads, 0, st>>>(out, iters, a, b);
  return cudaGetLastError() == cudaSuccess ? SA_OK : SA_ERR_CUDA;
}
