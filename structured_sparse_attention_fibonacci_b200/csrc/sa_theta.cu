// Learned-alpha parametrisation: one free parameter theta per layer, mapped
// into the constraint alpha in [0.5, 1.5] ("Depth-Staggered Fibonacci Spacing
// for Sparse Attention", Methodology: the scalar is constrained to [0.5, 1.5];
// experimental variables: the learned schedule has one free parameter theta per
// layer, initialised at alpha = 1, trained by gradient descent).  The page does
// not give the map; the one used here is alpha = 0.5 + sigmoid(theta), which is
// smooth, stays inside the interval, and gives alpha = 1 at theta = 0; its
// gradient is dtheta = dalpha * sigmoid(theta) * (1 - sigmoid(theta)).
#include "sa_internal.h"

namespace sa {

namespace {

__device__ __forceinline__ float sigmoid(float x) { return 1.f / (1.f + expf(-x)); }

__global__ void k_alpha_from_theta(int L, const float* theta, float* alpha) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l < L) alpha[l] = 0.5f + sigmoid(theta[l]);
}

__global__ void k_dtheta(int L, const float* theta, const float* dalpha, float* dtheta) {
  const int l = blockIdx.x * blockDim.x + threadIdx.x;
  if (l < L) {
    const float s = sigmoid(theta[l]);
    dtheta[l] = dalpha[l] * (s * (1.f - s));
  }
}

}  // namespace

cudaError_t launch_alpha_from_theta(int L, const float* theta, float* alpha, cudaStream_t st) {
  trace_mark("alpha_from_theta", st, true);
  k_alpha_from_theta<<<(L + 127) / 128, 128, 0, st>>>(L, theta, alpha);
  trace_mark("alpha_from_theta", st, false);
  return cudaGetLastError();
}

cudaError_t launch_dtheta(int L, const float* theta, const float* dalpha, float* dtheta,
                          cudaStream_t st) {
  trace_mark("dtheta", st, true);
  k_dtheta<<<(L + 127) / 128, 128, 0, st>>>(L, theta, dalpha, dtheta);
  trace_mark("dtheta", st, false);
  return cudaGetLastError();
}

}  // namespace sa
