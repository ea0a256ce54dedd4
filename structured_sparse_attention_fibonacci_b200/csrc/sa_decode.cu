// Single-token decode with a KV cache: the attention output of one new query
// per (layer, batch, head) at position `pos`, against cache rows 0..pos (the
// new token's own row included).  The members and their weights are those of
// row `pos` of the forward ("Depth-Staggered Fibonacci Spacing for Sparse
// Attention", technical summary, Methodology: attended set, scaling,
// interpolation with RoPE before the gather); the page measures inference
// latency for exactly this gather (Results, efficiency).
//
// One warp per (layer, batch, head).  Scores: lanes take members in turn; a
// member's key row (two rows for an interpolated offset) is loaded, rotated
// at its own position and dotted with the rotated query held in shared
// memory.  Softmax: warp reductions.  Output: lanes take head dims, walking
// the members in order with their weights.  Only the W + S + 2 * n_offsets
// rows a query attends are read from the cache.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {

namespace {

constexpr int kDecWarps = 4;
constexpr int kDecMaxMembers = 256 + SA_MAX_SINKS + SA_MAX_OFFSETS;

struct DecArgs {
  long long units;
  int B, H, Tc, W, n_off, S, pos;
  float scale;
  int f[SA_MAX_OFFSETS];
  const void* q; const void* k; const void* v;
  const float* alpha; const float2* rope;
  void* o; float* lse;
  const float* beta;                   // log-prior on the offset members [units], or nullptr
};

// q_hat . RoPE(K[row]) over D dims; q_hat in shared memory.
template <typename T, int D>
__device__ __forceinline__ float key_dot(const T* K, const float2* rope, int row, const float* qh) {
  constexpr int HALF = D / 2, N = (HALF < 8 ? HALF : 8);
  float acc = 0.f;
#pragma unroll
  for (int j0 = 0; j0 < HALF; j0 += N) {
    float x1[N], x2[N];
    float2 cs[N];
    load_row<T, N>(K + (size_t)row * D + j0, x1);
    load_row<T, N>(K + (size_t)row * D + HALF + j0, x2);
    load_cs<N>(rope + (size_t)row * HALF + j0, cs);
    rope_fwd<N>(x1, x2, cs);
#pragma unroll
    for (int h = 0; h < N; ++h) acc += qh[j0 + h] * x1[h] + qh[HALF + j0 + h] * x2[h];
  }
  return acc;
}

template <typename T>
__device__ __forceinline__ float load_elt(const T* p);
template <>
__device__ __forceinline__ float load_elt<float>(const float* p) { return __ldg(p); }
template <>
__device__ __forceinline__ float load_elt<__nv_bfloat16>(const __nv_bfloat16* p) {
  return __bfloat162float(*p);
}

template <typename T>
__device__ __forceinline__ void store_elt(T* p, float x);
template <>
__device__ __forceinline__ void store_elt<float>(float* p, float x) { *p = x; }
template <>
__device__ __forceinline__ void store_elt<__nv_bfloat16>(__nv_bfloat16* p, float x) {
  *p = __float2bfloat16_rn(x);
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecWarps * 32) k_decode(const DecArgs a) {
  __shared__ float s_q[kDecWarps][D];
  __shared__ float s_w[kDecWarps][kDecMaxMembers];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const long long unit = (long long)blockIdx.x * kDecWarps + warp;
  if (unit >= a.units) return;           // warps are independent (warp-level sync only)
  const int layer = (int)(unit / (a.B * a.H));
  const int W = a.W, S = a.S, n_off = a.n_off, pos = a.pos, Tc = a.Tc;
  const T* Q = reinterpret_cast<const T*>(a.q) + (size_t)unit * D;
  const T* K = reinterpret_cast<const T*>(a.k) + (size_t)unit * Tc * D;
  const T* V = reinterpret_cast<const T*>(a.v) + (size_t)unit * Tc * D;
  T* O = reinterpret_cast<T*>(a.o) + (size_t)unit * D;
  float* sw = s_w[warp];
  float* sq = s_q[warp];

  // offset geometry: lane k holds offset k
  OffGeo og{};
  int bad = 0;
  if (lane < n_off) {
    og = offset_geometry(__ldg(a.alpha + layer), a.f[lane]);
    bad = !og.ok;
  }
  bad = __any_sync(0xffffffffu, bad);
  if (bad) {
    for (int d = lane; d < D; d += 32) store_elt<T>(O + d, __int_as_float(0x7fc00000));
    if (lane == 0 && a.lse) a.lse[unit] = __int_as_float(0x7fc00000);
    return;
  }

  // Prefetch into L2 every cache row the query reads (K and V of the window,
  // the sinks and both rows of each offset): the rows are scattered over the
  // cache, and the dependent steps below then find them in L2.
  {
    constexpr int kLines = (D * (int)sizeof(T) + 127) / 128;
    auto prefetch_row = [&](int row) {
#pragma unroll
      for (int ln = 0; ln < kLines; ++ln) {
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(K + (size_t)row * D + ln * 128 / sizeof(T)));
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(V + (size_t)row * D + ln * 128 / sizeof(T)));
      }
    };
    for (int m = lane; m < W + S; m += 32) {
      const int row = m < W ? pos - m : m - W;
      if (row >= 0 && row <= pos) prefetch_row(row);
    }
    if (lane < n_off && pos - og.c >= 0) {
      prefetch_row(pos - og.lo);
      if (og.w != 0.f) prefetch_row(pos - og.lo - 1);
    }
  }

  // rotated, scaled query at position pos
  for (int j = lane; j < D / 2; j += 32) {
    const float x1 = load_elt<T>(Q + j), x2 = load_elt<T>(Q + D / 2 + j);
    const float2 cs = __ldg(a.rope + (size_t)pos * (D / 2) + j);
    sq[j] = (x1 * cs.x - x2 * cs.y) * a.scale;
    sq[D / 2 + j] = (x2 * cs.x + x1 * cs.y) * a.scale;
  }
  __syncwarp();

  // scores of every member (window lags, sinks, offsets); invalid ones -inf
  const int n = W + S + n_off;
  float mx = -INFINITY;
  for (int m = lane; m < n; m += 32) {
    float s = -INFINITY;
    if (m < W) {
      const int row = pos - m;
      if (row >= 0) s = key_dot<T, D>(K, a.rope, row, sq);
    } else if (m < W + S) {
      const int row = m - W;
      if (row <= pos) s = key_dot<T, D>(K, a.rope, row, sq);
    }
    sw[m] = s;
  }
  // offsets: lane k's geometry, so the offset members go by lane; each
  // carries the query's log-prior (0 without one)
  const float prior = a.beta ? __ldg(a.beta + unit) : 0.f;
  for (int k0 = 0; k0 < n_off; k0 += 32) {
    const int k = k0 + lane;
    if (k < n_off) {
      float s = -INFINITY;
      if (pos - og.c >= 0) {
        s = og.wa * key_dot<T, D>(K, a.rope, pos - og.lo, sq);
        if (og.w != 0.f) s += og.w * key_dot<T, D>(K, a.rope, pos - og.lo - 1, sq);
        s += prior;
      }
      sw[W + S + k] = s;
    }
  }
  __syncwarp();
  for (int m = lane; m < n; m += 32) mx = fmaxf(mx, sw[m]);
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) mx = fmaxf(mx, __shfl_xor_sync(0xffffffffu, mx, off));
  float l = 0.f;
  for (int m = lane; m < n; m += 32) {
    const float e = sw[m] == -INFINITY ? 0.f : __expf(sw[m] - mx);
    sw[m] = e;
    l += e;
  }
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) l += __shfl_xor_sync(0xffffffffu, l, off);
  __syncwarp();
  if (lane == 0 && a.lse) a.lse[unit] = mx + __logf(l);
  const float inv = 1.f / l;

  // output: lanes take dims d = lane, lane + 32, ...; members go in chunks
  // of kChunk whose loads are all issued before any is consumed (the loop is
  // bound by load latency, not arithmetic).  Member m's rows: window lag
  // pos - m, sink m - W, offset rows pos - lo (weight 1 - w) and
  // pos - lo - 1 (weight w).
  constexpr int DPL = (D + 31) / 32;
  constexpr int kChunk = 8;
  float o[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) o[u] = 0.f;
  for (int m0 = 0; m0 < n; m0 += kChunk) {
    int ra[kChunk], rb[kChunk];
    float wa[kChunk], wb[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      const int m = m0 + j;
      const float p = m < n ? sw[m] : 0.f;
      ra[j] = 0; rb[j] = 0; wa[j] = 0.f; wb[j] = 0.f;
      if (m < W + S) {
        ra[j] = m < W ? max(pos - m, 0) : min(m - W, pos);
        wa[j] = p;
      } else {
        const int k = min(m - W - S, n_off - 1);
        const int lo = __shfl_sync(0xffffffffu, og.lo, k & 31);
        const float w = __shfl_sync(0xffffffffu, og.w, k & 31);
        const float ww = __shfl_sync(0xffffffffu, og.wa, k & 31);
        if (p != 0.f) {
          ra[j] = pos - lo; wa[j] = p * ww;
          if (w != 0.f) { rb[j] = pos - lo - 1; wb[j] = p * w; }
        }
      }
    }
#pragma unroll
    for (int u = 0; u < DPL; ++u) {
      const int d = lane + 32 * u;
      if (d < D) {
        float xa[kChunk], xb[kChunk];
#pragma unroll
        for (int j = 0; j < kChunk; ++j) {
          xa[j] = load_elt<T>(V + (size_t)ra[j] * D + d);
          xb[j] = load_elt<T>(V + (size_t)rb[j] * D + d);
        }
#pragma unroll
        for (int j = 0; j < kChunk; ++j) o[u] += wa[j] * xa[j] + wb[j] * xb[j];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int d = lane + 32 * u;
    if (d < D) store_elt<T>(O + d, o[u] * inv);
  }
}

template <typename T, int D>
cudaError_t launch_t(const DecArgs& a, long long units, cudaStream_t st) {
  const unsigned grid = (unsigned)((units + kDecWarps - 1) / kDecWarps);
  trace_mark("decode", st, true);
  k_decode<T, D><<<grid, kDecWarps * 32, 0, st>>>(a);
  trace_mark("decode", st, false);
  return cudaGetLastError();
}

}  // namespace

bool decode_supported(const Problem& pb) { return pb.W <= 256; }

cudaError_t launch_decode(const Problem& pb, int pos, const void* q, const void* k, const void* v,
                          const float* alpha, const float2* rope, void* o, float* lse,
                          cudaStream_t st, const float* beta) {
  DecArgs a = {};
  a.B = pb.B; a.H = pb.H; a.Tc = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S; a.pos = pos;
  a.scale = pb.scale;
  for (int j = 0; j < pb.n_off; ++j) a.f[j] = pb.f[j];
  a.q = q; a.k = k; a.v = v; a.alpha = alpha; a.rope = rope; a.o = o; a.lse = lse;
  a.beta = beta;
  const long long units = pb.units();
  a.units = units;
  const bool f32 = pb.dtype == SA_DTYPE_F32;
  switch (pb.D) {
    case 16: return f32 ? launch_t<float, 16>(a, units, st) : launch_t<__nv_bfloat16, 16>(a, units, st);
    case 32: return f32 ? launch_t<float, 32>(a, units, st) : launch_t<__nv_bfloat16, 32>(a, units, st);
    case 64: return f32 ? launch_t<float, 64>(a, units, st) : launch_t<__nv_bfloat16, 64>(a, units, st);
    default: return f32 ? launch_t<float, 128>(a, units, st) : launch_t<__nv_bfloat16, 128>(a, units, st);
  }
}

}  // namespace sa
