// Tensor-map encoding for the tensor-core kernels.  The driver's
// cuTensorMapEncodeTiled is reached through the runtime's driver entry point,
// so the library links against no driver library directly.
#include <cudaTypedefs.h>

#include <mutex>

#include "sa_tc.cuh"

namespace sa {

namespace {

std::once_flag g_encode_once;
PFN_cuTensorMapEncodeTiled_v12000 g_encode = nullptr;

void load_encode() {
  void* fn = nullptr;
  cudaDriverEntryPointQueryResult q;
  if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &fn, cudaEnableDefault, &q) ==
          cudaSuccess &&
      q == cudaDriverEntryPointSuccess)
    g_encode = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(fn);
}

}  // namespace

cudaError_t make_rows_map(CUtensorMap* map, const void* base, int T, long long units) {
  std::call_once(g_encode_once, load_encode);
  if (!g_encode) return cudaErrorNotSupported;
  const cuuint64_t dims[3] = {64, (cuuint64_t)T, (cuuint64_t)units};
  const cuuint64_t strides[2] = {128, (cuuint64_t)T * 128};   // bytes, dims 1 and 2
  const cuuint32_t box[3] = {64, 8, 1};
  const cuuint32_t estr[3] = {1, 1, 1};
  const CUresult r = g_encode(map, CU_TENSOR_MAP_DATA_TYPE_UINT16, 3, const_cast<void*>(base), dims,
                              strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                              CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
                              CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS ? cudaSuccess : cudaErrorInvalidValue;
}

}  // namespace sa
