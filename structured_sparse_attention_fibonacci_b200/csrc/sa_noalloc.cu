// Forward entry point that allocates no device memory.
//
// sparse_attn_fwd keeps its RoPE cos/sin table in device memory that the
// library allocates on first use.  Some callers cannot let a library allocate:
// applications whose device memory belongs to a pooling allocator that must
// account for every byte, and embedders or latency-critical services that
// forbid allocation after start-up (cudaMalloc can synchronise the device and
// can fail under memory pressure at an arbitrary point of a run).
// sparse_attn_fwd_noalloc serves them: its
// only scratch is the RoPE table, kept in the fixed-size file-scope device
// array below, which every GPU that loads this library holds until the process
// exits.  Inputs and outputs are still the caller's buffers.
#include <mutex>
#include <vector>

#include "sa_internal.h"
#include "sparse_attn.h"

// The RoPE table of a call needs T * (D/2) * 8 bytes (for D = 64, T up to
// 32768 fits).
static __device__ __align__(256) unsigned char g_noalloc_scratch[SA_NOALLOC_SCRATCH_BYTES];

namespace {

std::mutex g_addr_mu;
std::vector<std::pair<int, void*>> g_addr;   // device ordinal -> device address of the array

// Device address of g_noalloc_scratch on the current device.  In host code the
// array's name is only a host-side stand-in: a kernel must be given the address
// cudaGetSymbolAddress returns for the device that is current, looked up once
// per device (this lookup is what the first call on a device does).
sa_status scratch_address(void** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_addr_mu);
  for (const auto& e : g_addr)
    if (e.first == dev) { *out = e.second; return SA_OK; }
  void* ptr = nullptr;
  if (cudaGetSymbolAddress(&ptr, g_noalloc_scratch) != cudaSuccess || !ptr) return SA_ERR_CUDA;
  g_addr.push_back({dev, ptr});
  *out = ptr;
  return SA_OK;
}

bool aligned(const void* p, uintptr_t a) { return (reinterpret_cast<uintptr_t>(p) & (a - 1)) == 0; }

}  // namespace

extern "C" sa_status sparse_attn_fwd_noalloc(const sa_params* p, const void* q, const void* k,
                                             const void* v, const float* alpha, void* o,
                                             float* lse, void* stream) {
  sa::Problem pb;
  sa_status s = sa::validate_params(p, &pb);
  if (s != SA_OK) return s;
  if (!q || !k || !v || !alpha || !o) return SA_ERR_INVALID_ARG;
  if (!aligned(q, 16) || !aligned(k, 16) || !aligned(v, 16) || !aligned(o, 16) ||
      (lse && !aligned(lse, 4)) || !aligned(alpha, 4))
    return SA_ERR_INVALID_ARG;
  const size_t table_bytes = (size_t)pb.T * (pb.D / 2) * sizeof(float2);
  if (table_bytes > SA_NOALLOC_SCRATCH_BYTES) return SA_ERR_UNSUPPORTED;
  void* scratch = nullptr;
  if ((s = scratch_address(&scratch)) != SA_OK) return s;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  // The whole table used by this call is rewritten first, on the same stream,
  // so nothing a previous call left in the array is read.
  float2* rope = reinterpret_cast<float2*>(scratch);
  if (sa::launch_rope_table(rope, pb.T, pb.D, (double)p->rope_base, st) != cudaSuccess)
    return SA_ERR_CUDA;
  sa::FwdPtrs a = {q, k, v, alpha, o, lse, rope};
  int launches = 0;
  if (sa::launch_fwd_dispatch(pb, a, st, &launches) != cudaSuccess) return SA_ERR_CUDA;
  return SA_OK;
}
