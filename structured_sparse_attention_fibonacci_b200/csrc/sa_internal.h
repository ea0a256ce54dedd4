// Internal interface between the C ABI (sa_api.cu) and the kernel files.
#pragma once

#include <cuda_runtime.h>
#include <stddef.h>
#include <stdint.h>

#include "sparse_attn.h"

namespace sa {

// Validated problem description shared by every launcher.
struct Problem {
  int L, B, H, T, D, W, n_off, S;
  float scale;                  // resolved (1/sqrt(D) when the caller passed <= 0)
  sa_dtype dtype;
  int f[SA_MAX_OFFSETS];
  int64_t units() const { return (int64_t)L * B * H; }
};

struct FwdPtrs {
  const void* q; const void* k; const void* v;
  const float* alpha;
  void* o; float* lse;
  const float2* rope;           // [T_cap][D/2] (cos, sin)
  const float* beta;            // log-prior on offset members [units][T], or nullptr
};

struct BwdPtrs {
  const void* q; const void* k; const void* v; const void* o; const void* dout;
  const float* lse; const float* alpha;
  void* dq; void* dk; void* dv; float* dalpha;
  const float2* rope;
  void* workspace;
  const float* beta;            // log-prior on offset members [units][T], or nullptr
  float* dbeta;                 // its gradient [units][T], or nullptr
};

// Workspace carving of the general backward (offsets in bytes).
struct BwdLayout {
  size_t d_off, dal_off, sink_off, total;
  int n_qtiles;                 // query tiles per (layer, batch, head) unit
};

BwdLayout general_bwd_layout(const Problem& pb);

// Argument validation shared by every C entry point (defined in sa_api.cu).
sa_status validate_params(const sa_params* p, Problem* pb);
// Forward dispatch shared by the C entry points: the staged kernel where it
// applies (and the general kernels are not forced), else the general kernel.
cudaError_t launch_fwd_dispatch(const Problem& pb, const FwdPtrs& a, cudaStream_t st,
                                int* launches);

// Diagnostics of the bounded staging waits (sa_api.cu): the wait limit in SM
// clocks (0: the kernels' default) and whether launches plant a stall in
// their first staging round (sparse_attn_set_wait_limit / _plant_stall).
struct WaitCfg {
  long long limit;
  int stall;
};
WaitCfg wait_cfg();

// Tracing hook: brackets one kernel launch with events when tracing is on.
// Call with begin = true just before the launch and false just after it.
void trace_mark(const char* kernel, cudaStream_t st, bool begin);

// Each launcher returns the first CUDA error it saw and adds the number of
// kernels it enqueued to *launches.
// Staged bf16 / D=64 forward (sa_fast.cu).  With keys_ws (fast_fwd_workspace
// bytes) the keys are rotated once by the RoPE pre-pass; with nullptr raw K
// rows are staged and rotated in shared memory (the allocation-free path).
bool fast_fwd_supported(const Problem& pb);
size_t fast_fwd_smem(const Problem& pb, int* ring_rows, int* sc_stride);
size_t fast_fwd_workspace(const Problem& pb);
// With save_p / save_dt / save_q (the training context) it also stores every
// member's probability ([units][W+S+n_off][T]) and every offset's row-score
// difference ([units][n_off][T]), fp32, and the rotated, scaled queries
// (fp16 of RoPE(Q) * scale / 256, [units][T][64]) for sparse_attn_bwd_ctx.
cudaError_t launch_fwd_fast(const Problem& pb, const FwdPtrs& a, void* keys_ws, cudaStream_t st,
                            int* launches, float* save_p = nullptr, float* save_dt = nullptr,
                            void* save_q = nullptr);
// Tensor-core bf16 / D=64 forward (sa_fwd_tc.cu); keys_ws as for the staged
// forward (fast_fwd_workspace bytes, required).
bool tc_fwd_supported(const Problem& pb);
// Where the tensor-core forward is the faster one: windows of 48 and more,
// except where its shared memory leaves it one CTA per SM while the CUDA-core
// forward keeps two (measured on B200; at W = 12 it runs 25% slower).  Its
// ring of staged rows is a power of two, or a multiple of 16 where that fits
// more CTAs per SM (W = 64 and 128 with 15 offsets and 4 sinks).
bool tc_fwd_preferred(const Problem& pb);
size_t tc_fwd_smem(const Problem& pb, int* ring_rows, int* sc_stride);
cudaError_t launch_fwd_tc(const Problem& pb, const FwdPtrs& a, void* keys_ws, cudaStream_t st,
                          int* launches);
cudaError_t fast_fwd_tc_read_error(unsigned* out, bool clear);
// Fifth-generation tensor-core bf16 / D=64 forward (sa_fwd_umma.cu): the
// window band and the sinks as tcgen05 GEMMs with accumulators in tensor
// memory, the offset members on the CUDA cores; keys_ws as for the staged
// forward.  Applies while the band plus 16 sink rows is at most 256 rows
// (W <= 113 with sinks, 129 without) and S <= 16.  Runs only when selected
// (sparse_attn_select_forward(3)): measured on B200 it is within 4% of the
// mma.sync forward at W = 64..112 and slower elsewhere.
bool umma_fwd_supported(const Problem& pb);
cudaError_t launch_fwd_umma(const Problem& pb, const FwdPtrs& a, void* keys_ws, cudaStream_t st,
                            int* launches);
cudaError_t fwd_umma_read_error(unsigned* out, bool clear);

// Device error words of the staged kernels (bit 0: a bounded staging wait
// gave up); optionally cleared after reading.
cudaError_t fast_fwd_read_error(unsigned* out, bool clear);
cudaError_t fast_bwd_read_error(unsigned* out, bool clear);

// RoPE pre-pass (sa_prep.cu): y = fp16(RoPE(x) * mul) for n_rows rows of a bf16
// [units][T][64] array, row r rotated at position r % T.
cudaError_t launch_rope_rows(const void* x, const float2* rope, int T, long long n_rows, float mul,
                             void* y, cudaStream_t st, const char* trace_name);
// The pre-pass's error word (bit 2: a finite rotated value beyond fp16's range).
cudaError_t prep_read_error(unsigned* out, bool clear);

// Staged bf16 / D=64 backward (sa_fast_bwd.cu).
bool fast_bwd_supported(const Problem& pb);
size_t fast_bwd_workspace(const Problem& pb);
// With ctx (a training context from the saving forward) the query side loads
// the probabilities and row-score differences instead of recomputing scores,
// and the rotated keys come from the context (no key pre-pass).
cudaError_t launch_bwd_fast(const Problem& pb, const BwdPtrs& a, cudaStream_t st, int* launches,
                            const void* ctx = nullptr);

// Training context layout (shared by sa_api.cu and the kernels' launchers).
struct CtxLayout {
  size_t khat_off, qhat_off, p_off, dt_off, total;
};
inline CtxLayout ctx_layout(const Problem& pb) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t units = (size_t)pb.units(), T = (size_t)pb.T;
  CtxLayout c;
  c.khat_off = 0;
  c.qhat_off = up(units * T * 64 * 2);
  c.p_off = c.qhat_off + up(units * T * 64 * 2);
  c.dt_off = c.p_off + up(units * (size_t)(pb.W + pb.S + pb.n_off) * T * sizeof(float));
  c.total = c.dt_off + up(units * (size_t)pb.n_off * T * sizeof(float));
  return c;
}

// dalpha[l] = fixed-order sum of part[l * per_layer .. (l+1) * per_layer).
cudaError_t launch_reduce_dalpha(const float* part, int L, int per_layer, float* dalpha,
                                 cudaStream_t st);

cudaError_t launch_rope_table(float2* tab, int T, int D, double base, cudaStream_t st);
// Learned-alpha map (sa_theta.cu): alpha = 0.5 + sigmoid(theta) and its gradient.
cudaError_t launch_alpha_from_theta(int L, const float* theta, float* alpha, cudaStream_t st);
cudaError_t launch_dtheta(int L, const float* theta, const float* dalpha, float* dtheta,
                          cudaStream_t st);
// Single-token decode (sa_decode.cu): pb.T is the cache length, pos < pb.T.
// Whether the decode kernel takes this problem (its member list fits shared memory).
bool decode_supported(const Problem& pb);
// beta: the new queries' log-prior on their offset members [units], or nullptr.
cudaError_t launch_decode(const Problem& pb, int pos, const void* q, const void* k, const void* v,
                          const float* alpha, const float2* rope, void* o, float* lse,
                          cudaStream_t st, const float* beta = nullptr);
cudaError_t launch_fwd_general(const Problem& pb, const FwdPtrs& a, cudaStream_t st, int* launches);
cudaError_t launch_bwd_general(const Problem& pb, const BwdPtrs& a, cudaStream_t st, int* launches);

}  // namespace sa
