// C ABI of the sparse-attention library: argument validation, workspace
// sizing, the per-device RoPE table cache and kernel dispatch.  Declarations
// and the contract (layouts, ownership, errors) are in include/sparse_attn.h.
#include <math.h>
#include <string.h>

#include <algorithm>
#include <mutex>
#include <vector>

#include "sa_internal.h"
#include "sparse_attn.h"

namespace {

thread_local int32_t g_last_launches = 0;
int g_force_general = 0;  // diagnostics: route every call through the general kernels
int g_fwd_select = 0;     // diagnostics: 0 auto, 1 CUDA-core staged, 2 mma.sync, 3 tcgen05 forward
long long g_wait_limit = 0;  // diagnostics: staging wait limit in SM clocks (0: default)
int g_plant_stall = 0;       // diagnostics: failure-path test of the bounded waits

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

sa_status build_problem(const sa_params* p, sa::Problem* pb) {
  if (!p) return SA_ERR_INVALID_ARG;
  if (p->L < 1 || p->B < 1 || p->H < 1 || p->T < 1) return SA_ERR_INVALID_ARG;
  if (p->window < 1 || p->n_sinks < 0 || p->n_offsets < 0) return SA_ERR_INVALID_ARG;
  if (p->n_offsets > SA_MAX_OFFSETS || p->n_sinks > SA_MAX_SINKS) return SA_ERR_UNSUPPORTED;
  if (p->n_offsets > 0 && !p->offsets) return SA_ERR_INVALID_ARG;
  if (!(p->rope_base > 0.f) || !isfinite(p->rope_base) || !isfinite(p->scale))
    return SA_ERR_INVALID_ARG;
  if (p->dtype != SA_DTYPE_F32 && p->dtype != SA_DTYPE_BF16) return SA_ERR_INVALID_ARG;
  if (p->D != 16 && p->D != 32 && p->D != 64 && p->D != 128) return SA_ERR_UNSUPPORTED;
  // index ranges: positions and per-unit offsets stay in int32, grids in 2^31
  if (p->T > (1 << 24)) return SA_ERR_UNSUPPORTED;
  const long long units = (long long)p->L * p->B * p->H;
  if (units * (((long long)p->T + 15) / 16) >= (1LL << 31)) return SA_ERR_UNSUPPORTED;
  pb->L = p->L; pb->B = p->B; pb->H = p->H; pb->T = p->T; pb->D = p->D;
  pb->W = p->window; pb->n_off = p->n_offsets; pb->S = p->n_sinks;
  pb->scale = p->scale > 0.f ? p->scale : (float)(1.0 / sqrt((double)p->D));
  pb->dtype = p->dtype;
  for (int k = 0; k < p->n_offsets; ++k) {
    if (p->offsets[k] < 1) return SA_ERR_INVALID_ARG;
    pb->f[k] = p->offsets[k];
  }
  return SA_OK;
}

// ---- RoPE cos/sin table, one per (device, D, base), grown on demand ---------
struct RopeTable {
  int dev, D;
  float base;
  int T_cap;
  float2* ptr;
};
std::mutex g_rope_mu;
std::vector<RopeTable> g_rope;  // superseded tables stay allocated until exit

sa_status rope_table(int T, int D, float base, cudaStream_t st, const float2** out) {
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return SA_ERR_CUDA;
  std::lock_guard<std::mutex> lock(g_rope_mu);
  for (auto it = g_rope.rbegin(); it != g_rope.rend(); ++it) {
    if (it->dev == dev && it->D == D && it->base == base && it->T_cap >= T) {
      *out = it->ptr;
      return SA_OK;
    }
  }
  int cap = 4096;
  while (cap < T) cap *= 2;
  float2* ptr = nullptr;
  if (cudaMalloc(&ptr, (size_t)cap * (D / 2) * sizeof(float2)) != cudaSuccess) return SA_ERR_CUDA;
  if (sa::launch_rope_table(ptr, cap, D, (double)base, st) != cudaSuccess ||
      cudaStreamSynchronize(st) != cudaSuccess) {
    cudaFree(ptr);
    return SA_ERR_CUDA;
  }
  g_rope.push_back({dev, D, base, cap, ptr});
  *out = ptr;
  return SA_OK;
}

// ---- kernel tracing ---------------------------------------------------------
struct TraceRec {
  const char* name;
  cudaEvent_t a, b;
};
std::mutex g_trace_mu;
bool g_trace_on = false;
std::vector<TraceRec> g_trace;       // completed begin/end pairs
std::vector<cudaEvent_t> g_ev_pool;  // reusable events
TraceRec g_open = {nullptr, nullptr, nullptr};

cudaEvent_t take_event() {
  if (!g_ev_pool.empty()) {
    cudaEvent_t e = g_ev_pool.back();
    g_ev_pool.pop_back();
    return e;
  }
  cudaEvent_t e = nullptr;
  cudaEventCreate(&e);
  return e;
}

}  // namespace

namespace sa {
sa_status validate_params(const sa_params* p, Problem* pb) { return build_problem(p, pb); }

cudaError_t launch_fwd_dispatch(const Problem& pb, const FwdPtrs& a, cudaStream_t st,
                                int* launches) {
  return (!g_force_general && fast_fwd_supported(pb))
             ? launch_fwd_fast(pb, a, nullptr, st, launches)
             : launch_fwd_general(pb, a, st, launches);
}

WaitCfg wait_cfg() { return WaitCfg{g_wait_limit, g_plant_stall}; }

void trace_mark(const char* kernel, cudaStream_t st, bool begin) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  if (!g_trace_on) return;
  cudaEvent_t e = take_event();
  if (!e) return;
  cudaEventRecord(e, st);
  if (begin) {
    g_open = {kernel, e, nullptr};
  } else if (g_open.name == kernel) {
    g_open.b = e;
    g_trace.push_back(g_open);
    g_open = {nullptr, nullptr, nullptr};
  } else {
    g_ev_pool.push_back(e);
  }
}
}  // namespace sa

extern "C" {

const char* sparse_attn_status_string(sa_status s) {
  switch (s) {
    case SA_OK: return "ok";
    case SA_ERR_INVALID_ARG: return "invalid argument";
    case SA_ERR_UNSUPPORTED: return "unsupported configuration";
    case SA_ERR_WORKSPACE: return "workspace too small";
    case SA_ERR_CUDA: return "CUDA error";
    case SA_ERR_INTERNAL: return "internal error";
  }
  return "unknown status";
}

int32_t sparse_attn_last_launch_count(void) { return g_last_launches; }

void sparse_attn_force_general(int on) { g_force_general = on != 0; }

void sparse_attn_select_forward(int which) {
  g_fwd_select = (which >= 1 && which <= 3) ? which : 0;
}

void sparse_attn_set_wait_limit(long long clocks) { g_wait_limit = clocks > 0 ? clocks : 0; }

void sparse_attn_plant_stall(int on) { g_plant_stall = on != 0; }

void sparse_attn_trace_enable(int on) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  g_trace_on = on != 0;
}

int32_t sparse_attn_trace_read(int32_t max, const char** names, double* total_ms,
                               int32_t* counts) {
  std::lock_guard<std::mutex> lock(g_trace_mu);
  std::vector<const char*> nm;
  std::vector<double> ms;
  std::vector<int32_t> ct;
  for (const TraceRec& r : g_trace) {
    float t = 0.f;
    cudaEventSynchronize(r.b);
    cudaEventElapsedTime(&t, r.a, r.b);
    size_t k = 0;
    while (k < nm.size() && nm[k] != r.name) ++k;
    if (k == nm.size()) { nm.push_back(r.name); ms.push_back(0.0); ct.push_back(0); }
    ms[k] += t;
    ct[k] += 1;
    g_ev_pool.push_back(r.a);
    g_ev_pool.push_back(r.b);
  }
  g_trace.clear();
  for (size_t k = 0; k < nm.size() && (int32_t)k < max; ++k) {
    if (names) names[k] = nm[k];
    if (total_ms) total_ms[k] = ms[k];
    if (counts) counts[k] = ct[k];
  }
  return (int32_t)nm.size();
}

int32_t sparse_attn_device_error(int clear) {
  unsigned fwd = 0, fwd_tc = 0, fwd_umma = 0, bwd = 0, prep = 0;
  if (sa::fast_fwd_read_error(&fwd, clear != 0) != cudaSuccess ||
      sa::fast_fwd_tc_read_error(&fwd_tc, clear != 0) != cudaSuccess ||
      sa::fwd_umma_read_error(&fwd_umma, clear != 0) != cudaSuccess ||
      sa::fast_bwd_read_error(&bwd, clear != 0) != cudaSuccess ||
      sa::prep_read_error(&prep, clear != 0) != cudaSuccess)
    return -1;
  return (int32_t)(fwd | fwd_tc | fwd_umma | bwd | prep);
}

size_t sparse_attn_workspace_size(const sa_params* p, int backward) {
  sa::Problem pb;
  if (build_problem(p, &pb) != SA_OK) return 0;
  if (!backward) return sa::fast_fwd_workspace(pb);
  // enough for whichever backward path a call takes (see sparse_attn_force_general)
  size_t need = sa::general_bwd_layout(pb).total;
  if (sa::fast_bwd_supported(pb)) need = std::max(need, sa::fast_bwd_workspace(pb));
  return need;
}

}  // extern "C"

namespace {

// Shared by sparse_attn_fwd and sparse_attn_fwd_prior (beta may be null).
sa_status fwd_impl(const sa_params* p, const void* q, const void* k, const void* v,
                   const float* alpha, const float* beta, void* o, float* lse, void* workspace,
                   size_t workspace_bytes, void* stream) {
  sa::Problem pb;
  sa_status s = build_problem(p, &pb);
  if (s != SA_OK) return s;
  if (!q || !k || !v || !alpha || !o) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && !aligned4(lse)) || !aligned4(alpha) || (beta && !aligned4(beta)))
    return SA_ERR_INVALID_ARG;
  const size_t need = sparse_attn_workspace_size(p, 0);
  if (workspace_bytes < need || (need && (!workspace || !aligned16(workspace))))
    return SA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float2* rope = nullptr;
  if ((s = rope_table(pb.T, pb.D, p->rope_base, st, &rope)) != SA_OK) return s;
  sa::FwdPtrs a = {q, k, v, alpha, o, lse, rope, beta};
  int launches = 0;
  cudaError_t e;
  if (g_force_general || !sa::fast_fwd_supported(pb))
    e = sa::launch_fwd_general(pb, a, st, &launches);
  else if (g_fwd_select == 3 && sa::umma_fwd_supported(pb))
    e = sa::launch_fwd_umma(pb, a, workspace, st, &launches);
  else if (g_fwd_select == 2 ? sa::tc_fwd_supported(pb)
                              : (g_fwd_select == 0 && sa::tc_fwd_preferred(pb)))
    e = sa::launch_fwd_tc(pb, a, workspace, st, &launches);
  else
    e = sa::launch_fwd_fast(pb, a, workspace, st, &launches);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  g_last_launches = launches;
  return SA_OK;
}

// Shared by sparse_attn_fwd_train and sparse_attn_fwd_prior with a context.
sa_status fwd_train_impl(const sa_params* p, const void* q, const void* k, const void* v,
                         const float* alpha, const float* beta, void* o, float* lse,
                         void* context, size_t context_bytes, void* stream) {
  sa::Problem pb;
  sa_status s = build_problem(p, &pb);
  if (s != SA_OK) return s;
  if (!q || !k || !v || !alpha || !o) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && !aligned4(lse)) || !aligned4(alpha) || (beta && !aligned4(beta)))
    return SA_ERR_INVALID_ARG;
  const size_t need = sparse_attn_context_size(p);
  if (need == 0) return SA_ERR_UNSUPPORTED;
  if (context_bytes < need || !context || !aligned16(context)) return SA_ERR_WORKSPACE;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float2* rope = nullptr;
  if ((s = rope_table(pb.T, pb.D, p->rope_base, st, &rope)) != SA_OK) return s;
  sa::FwdPtrs a = {q, k, v, alpha, o, lse, rope, beta};
  const sa::CtxLayout cl = sa::ctx_layout(pb);
  char* cb = reinterpret_cast<char*>(context);
  int launches = 0;
  if (sa::launch_fwd_fast(pb, a, cb + cl.khat_off, st, &launches,
                          reinterpret_cast<float*>(cb + cl.p_off),
                          reinterpret_cast<float*>(cb + cl.dt_off), cb + cl.qhat_off) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  g_last_launches = launches;
  return SA_OK;
}

// Shared by sparse_attn_bwd, sparse_attn_bwd_ctx and sparse_attn_bwd_prior
// (beta / dbeta may be null; a context selects the context backward).
sa_status bwd_impl(const sa_params* p, const void* q, const void* k, const void* v,
                   const void* o, const float* lse, const void* dout, const float* alpha,
                   const float* beta, const void* context, void* dq, void* dk, void* dv,
                   float* dalpha, float* dbeta, void* workspace, size_t workspace_bytes,
                   void* stream) {
  sa::Problem pb;
  sa_status s = build_problem(p, &pb);
  if (s != SA_OK) return s;
  const void* tensors[] = {q, k, v, o, dout, dq, dk, dv};
  for (const void* x : tensors)
    if (!x || !aligned16(x)) return SA_ERR_INVALID_ARG;
  const void* vectors[] = {alpha, dalpha};
  for (const void* x : vectors)
    if (!x || !aligned4(x)) return SA_ERR_INVALID_ARG;
  if ((lse && !aligned4(lse)) || (beta && !aligned4(beta)) || (dbeta && !aligned4(dbeta)))
    return SA_ERR_INVALID_ARG;
  size_t need;
  if (context) {
    if (sparse_attn_context_size(p) == 0) return SA_ERR_UNSUPPORTED;
    if (!aligned16(context)) return SA_ERR_INVALID_ARG;
    need = sa::fast_bwd_workspace(pb);
    if (workspace_bytes < need || !workspace || !aligned16(workspace)) return SA_ERR_WORKSPACE;
  } else {
    if (!lse) return SA_ERR_INVALID_ARG;
    need = sparse_attn_workspace_size(p, 1);
    if (workspace_bytes < need || (need && (!workspace || !aligned16(workspace))))
      return SA_ERR_WORKSPACE;
  }
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float2* rope = nullptr;
  if ((s = rope_table(pb.T, pb.D, p->rope_base, st, &rope)) != SA_OK) return s;
  sa::BwdPtrs a = {q, k, v, o, dout, lse, alpha, dq, dk, dv, dalpha, rope, workspace, beta, dbeta};
  int launches = 0;
  cudaError_t e;
  if (context)
    e = sa::launch_bwd_fast(pb, a, st, &launches, context);
  else
    e = (!g_force_general && sa::fast_bwd_supported(pb))
            ? sa::launch_bwd_fast(pb, a, st, &launches)
            : sa::launch_bwd_general(pb, a, st, &launches);
  if (e != cudaSuccess) return SA_ERR_CUDA;
  g_last_launches = launches;
  return SA_OK;
}

}  // namespace

extern "C" {

sa_status sparse_attn_fwd(const sa_params* p, const void* q, const void* k, const void* v,
                          const float* alpha, void* o, float* lse, void* workspace,
                          size_t workspace_bytes, void* stream) {
  return fwd_impl(p, q, k, v, alpha, nullptr, o, lse, workspace, workspace_bytes, stream);
}

sa_status sparse_attn_fwd_prior(const sa_params* p, const void* q, const void* k, const void* v,
                                const float* alpha, const float* beta, void* o, float* lse,
                                void* workspace, size_t workspace_bytes, void* context,
                                size_t context_bytes, void* stream) {
  if (!beta) return SA_ERR_INVALID_ARG;
  return context ? fwd_train_impl(p, q, k, v, alpha, beta, o, lse, context, context_bytes, stream)
                 : fwd_impl(p, q, k, v, alpha, beta, o, lse, workspace, workspace_bytes, stream);
}

sa_status sparse_attn_bwd_prior(const sa_params* p, const void* q, const void* k, const void* v,
                                const void* o, const float* lse, const void* dout,
                                const float* alpha, const float* beta, const void* context,
                                void* dq, void* dk, void* dv, float* dalpha, float* dbeta,
                                void* workspace, size_t workspace_bytes, void* stream) {
  if (!beta || !dbeta) return SA_ERR_INVALID_ARG;
  return bwd_impl(p, q, k, v, o, lse, dout, alpha, beta, context, dq, dk, dv, dalpha, dbeta,
                  workspace, workspace_bytes, stream);
}

sa_status sparse_attn_decode(const sa_params* p, int32_t pos, const void* q, const void* k,
                             const void* v, const float* alpha, void* o, float* lse,
                             void* stream) {
  return sparse_attn_decode_prior(p, pos, q, k, v, alpha, nullptr, o, lse, stream);
}

sa_status sparse_attn_decode_prior(const sa_params* p, int32_t pos, const void* q, const void* k,
                                   const void* v, const float* alpha, const float* beta, void* o,
                                   float* lse, void* stream) {
  sa::Problem pb;
  sa_status s = build_problem(p, &pb);
  if (s != SA_OK) return s;
  if (pos < 0 || pos >= pb.T) return SA_ERR_INVALID_ARG;
  if (!sa::decode_supported(pb)) return SA_ERR_UNSUPPORTED;
  if (!q || !k || !v || !alpha || !o) return SA_ERR_INVALID_ARG;
  if (!aligned16(q) || !aligned16(k) || !aligned16(v) || !aligned16(o) ||
      (lse && !aligned4(lse)) || !aligned4(alpha) || (beta && !aligned4(beta)))
    return SA_ERR_INVALID_ARG;
  cudaStream_t st = reinterpret_cast<cudaStream_t>(stream);
  const float2* rope = nullptr;
  if ((s = rope_table(pb.T, pb.D, p->rope_base, st, &rope)) != SA_OK) return s;
  if (sa::launch_decode(pb, pos, q, k, v, alpha, rope, o, lse, st, beta) != cudaSuccess)
    return SA_ERR_CUDA;
  g_last_launches = 1;
  return SA_OK;
}

sa_status sparse_attn_alpha_from_theta(int32_t L, const float* theta, float* alpha,
                                       void* stream) {
  if (L < 1 || !theta || !alpha || !aligned4(theta) || !aligned4(alpha))
    return SA_ERR_INVALID_ARG;
  if (sa::launch_alpha_from_theta(L, theta, alpha, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  g_last_launches = 1;
  return SA_OK;
}

sa_status sparse_attn_dtheta(int32_t L, const float* theta, const float* dalpha, float* dtheta,
                             void* stream) {
  if (L < 1 || !theta || !dalpha || !dtheta || !aligned4(theta) || !aligned4(dalpha) ||
      !aligned4(dtheta))
    return SA_ERR_INVALID_ARG;
  if (sa::launch_dtheta(L, theta, dalpha, dtheta, reinterpret_cast<cudaStream_t>(stream)) !=
      cudaSuccess)
    return SA_ERR_CUDA;
  g_last_launches = 1;
  return SA_OK;
}

size_t sparse_attn_context_size(const sa_params* p) {
  sa::Problem pb;
  if (build_problem(p, &pb) != SA_OK) return 0;
  if (!sa::fast_fwd_supported(pb) || !sa::fast_bwd_supported(pb)) return 0;
  return sa::ctx_layout(pb).total;
}

sa_status sparse_attn_fwd_train(const sa_params* p, const void* q, const void* k, const void* v,
                                const float* alpha, void* o, float* lse, void* context,
                                size_t context_bytes, void* stream) {
  return fwd_train_impl(p, q, k, v, alpha, nullptr, o, lse, context, context_bytes, stream);
}

sa_status sparse_attn_bwd_ctx(const sa_params* p, const void* q, const void* k, const void* v,
                              const void* o, const float* lse, const void* dout,
                              const float* alpha, const void* context, void* dq, void* dk,
                              void* dv, float* dalpha, void* workspace, size_t workspace_bytes,
                              void* stream) {
  if (!context) return SA_ERR_INVALID_ARG;
  return bwd_impl(p, q, k, v, o, lse, dout, alpha, nullptr, context, dq, dk, dv, dalpha, nullptr,
                  workspace, workspace_bytes, stream);
}

sa_status sparse_attn_bwd(const sa_params* p, const void* q, const void* k, const void* v,
                          const void* o, const float* lse, const void* dout, const float* alpha,
                          void* dq, void* dk, void* dv, float* dalpha, void* workspace,
                          size_t workspace_bytes, void* stream) {
  if (!lse) return SA_ERR_INVALID_ARG;
  return bwd_impl(p, q, k, v, o, lse, dout, alpha, nullptr, nullptr, dq, dk, dv, dalpha, nullptr,
                  workspace, workspace_bytes, stream);
}

}  // extern "C"
