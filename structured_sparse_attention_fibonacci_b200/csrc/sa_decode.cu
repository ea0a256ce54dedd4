// Single-token decode with a KV cache: the attention output of one new query
// per (layer, batch, head) at position `pos`, against cache rows 0..pos (the
// new token's own row included).  The members and their weights are those of
// row `pos` of the forward ("Depth-Staggered Fibonacci Spacing for Sparse
// Attention", technical summary, Methodology: attended set, scaling,
// interpolation with RoPE before the gather); the page measures inference
// latency for exactly this gather (Results, efficiency).
//
// One CTA of 128 threads per (layer, batch, head), so that a step is a few
// dependent memory rounds deep (a single-token step is latency-bound):
//   1. the member table, an L2 prefetch of every row it names, and the
//      rotated, scaled query;
//   2. scores, four threads per member, each a quarter of the head dims: the
//      key row(s) (two rows for an interpolated offset, loaded together)
//      rotated at their own positions and dotted with the query;
//   3. a block-wide softmax;
//   4. the output: the four warps take every fourth member, lanes take head
//      dims, and the warps' partial sums meet in shared memory.
// Only the W + S + 2 * n_offsets rows a query attends are read from the cache.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {

namespace {

constexpr int kDecThreads = 128;                 // one CTA (4 warps) per unit
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kDecMaxMembers = 256 + SA_MAX_SINKS + SA_MAX_OFFSETS;

struct DecArgs {
  int B, H, Tc, W, n_off, S, pos;
  float scale;
  int f[SA_MAX_OFFSETS];
  const void* q; const void* k; const void* v;
  const float* alpha; const float2* rope;
  void* o; float* lse;
  const float* beta;                   // log-prior on the offset members [units], or nullptr
};

// Quarter `part` (0..3) of q_hat . (wa RoPE(K[ra]) + wb RoPE(K[rb])): the
// rotation pairs [part * D/8, (part + 1) * D/8) of both rows (rb < 0: one
// row), whose loads are all issued before any is used.
template <typename T, int D>
__device__ __forceinline__ float member_score_part(const T* K, const float2* rope, int ra, int rb,
                                                   float wa, float wb, const float* qh,
                                                   int part) {
  constexpr int HALF = D / 2, P = D / 8;
  const int j0 = part * P;
  const bool two = rb >= 0;
  const int rb_ = two ? rb : ra;
  float a1[P], a2[P], b1[P], b2[P];
  float2 ca[P], cb[P];
  load_row<T, P>(K + (size_t)ra * D + j0, a1);
  load_row<T, P>(K + (size_t)ra * D + HALF + j0, a2);
  load_cs<P>(rope + (size_t)ra * HALF + j0, ca);
  load_row<T, P>(K + (size_t)rb_ * D + j0, b1);
  load_row<T, P>(K + (size_t)rb_ * D + HALF + j0, b2);
  load_cs<P>(rope + (size_t)rb_ * HALF + j0, cb);
  rope_fwd<P>(a1, a2, ca);
  rope_fwd<P>(b1, b2, cb);
  float acc_a = 0.f, acc_b = 0.f;
#pragma unroll
  for (int h = 0; h < P; ++h) {
    acc_a += qh[j0 + h] * a1[h] + qh[HALF + j0 + h] * a2[h];
    acc_b += qh[j0 + h] * b1[h] + qh[HALF + j0 + h] * b2[h];
  }
  return two ? wa * acc_a + wb * acc_b : wa * acc_a;
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

// Block-wide reduction of one value per thread (max or sum); every thread
// gets the result.
template <bool MAX>
__device__ __forceinline__ float block_reduce(float x, float* s_red) {
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) {
    const float y = __shfl_xor_sync(0xffffffffu, x, off);
    x = MAX ? fmaxf(x, y) : x + y;
  }
  if ((threadIdx.x & 31) == 0) s_red[threadIdx.x >> 5] = x;
  __syncthreads();
  float r = s_red[0];
#pragma unroll
  for (int w = 1; w < kDecWarps; ++w) r = MAX ? fmaxf(r, s_red[w]) : r + s_red[w];
  __syncthreads();
  return r;
}

template <typename T, int D>
__global__ void __launch_bounds__(kDecThreads) k_decode(const DecArgs a) {
  __shared__ float s_q[D];
  __shared__ float s_p[kDecMaxMembers];          // scores, then unnormalised weights
  __shared__ int s_ra[kDecMaxMembers], s_rb[kDecMaxMembers];   // rows (ra < 0: absent)
  __shared__ float s_wa[kDecMaxMembers], s_wb[kDecMaxMembers];
  __shared__ float s_o[kDecWarps][D];            // per-warp partial outputs
  __shared__ float s_red[kDecWarps];
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  const int unit = blockIdx.x, t = threadIdx.x, warp = t >> 5, lane = t & 31;
  const int layer = unit / (a.B * a.H);
  const int W = a.W, S = a.S, n_off = a.n_off, pos = a.pos, Tc = a.Tc;
  const int n = W + S + n_off;
  const T* Q = reinterpret_cast<const T*>(a.q) + (size_t)unit * D;
  const T* K = reinterpret_cast<const T*>(a.k) + (size_t)unit * Tc * D;
  const T* V = reinterpret_cast<const T*>(a.v) + (size_t)unit * Tc * D;
  T* O = reinterpret_cast<T*>(a.o) + (size_t)unit * D;

  int bad = 0;
  if (t < n_off) {
    sg[t] = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    bad = !sg[t].ok;
  }
  if (__syncthreads_or(bad)) {     // an offset with no defined row: NaN outputs
    for (int d = t; d < D; d += kDecThreads) store_elt<T>(O + d, __int_as_float(0x7fc00000));
    if (t == 0 && a.lse) a.lse[unit] = __int_as_float(0x7fc00000);
    return;
  }

  // member table (window lag m, sink m - W, offset m - W - S) and an L2
  // prefetch of every K and V row it names; the rotated, scaled query
  constexpr int kLines = (D * (int)sizeof(T) + 127) / 128;
  for (int m = t; m < n; m += kDecThreads) {
    int ra = -1, rb = -1;
    float wa = 1.f, wb = 0.f;
    if (m < W) {
      if (pos - m >= 0) ra = pos - m;
    } else if (m < W + S) {
      if (m - W <= pos) ra = m - W;
    } else {
      const OffGeo g = sg[m - W - S];
      if (pos - g.c >= 0) {
        ra = pos - g.lo;
        wa = g.wa;
        if (g.w != 0.f) { rb = pos - g.lo - 1; wb = g.w; }
      }
    }
    s_ra[m] = ra; s_rb[m] = rb; s_wa[m] = wa; s_wb[m] = wb;
#pragma unroll
    for (int ln = 0; ln < kLines; ++ln) {
      if (ra >= 0) {
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(K + (size_t)ra * D + ln * 128 / sizeof(T)));
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(V + (size_t)ra * D + ln * 128 / sizeof(T)));
      }
      if (rb >= 0) {
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(K + (size_t)rb * D + ln * 128 / sizeof(T)));
        asm volatile("prefetch.global.L2 [%0];\n" ::"l"(V + (size_t)rb * D + ln * 128 / sizeof(T)));
      }
    }
  }
  for (int j = t; j < D / 2; j += kDecThreads) {
    const float x1 = load_elt<T>(Q + j), x2 = load_elt<T>(Q + D / 2 + j);
    const float2 cs = __ldg(a.rope + (size_t)pos * (D / 2) + j);
    s_q[j] = (x1 * cs.x - x2 * cs.y) * a.scale;
    s_q[D / 2 + j] = (x2 * cs.x + x1 * cs.y) * a.scale;
  }
  __syncthreads();

  // scores, four threads per member (a quarter of the dims each, summed by
  // two shuffles); offset members carry the query's log-prior
  const float prior = a.beta ? __ldg(a.beta + unit) : 0.f;
  float mx = -INFINITY;
  for (int m0 = 0; m0 < n; m0 += kDecThreads / 4) {     // uniform over the block
    const int m = m0 + (t >> 2), part = t & 3;
    const int ra = m < n ? s_ra[m] : -1;
    float s = ra >= 0 ? member_score_part<T, D>(K, a.rope, ra, s_rb[m], s_wa[m], s_wb[m], s_q,
                                                part)
                      : 0.f;
    s += __shfl_xor_sync(0xffffffffu, s, 1);
    s += __shfl_xor_sync(0xffffffffu, s, 2);
    if (m < n && part == 0) {
      s = ra >= 0 ? s + (m >= W + S ? prior : 0.f) : -INFINITY;
      s_p[m] = s;
      mx = fmaxf(mx, s);
    }
  }
  mx = block_reduce<true>(mx, s_red);
  float l = 0.f;
  for (int m = t; m < n; m += kDecThreads) {
    const float e = s_p[m] == -INFINITY ? 0.f : __expf(s_p[m] - mx);
    s_p[m] = e;
    l += e;
  }
  l = block_reduce<false>(l, s_red);     // (its barriers also publish s_p)
  if (t == 0 && a.lse) a.lse[unit] = mx + __logf(l);

  // output: warp w takes members w, w + 4, ...; lanes take dims lane,
  // lane + 32, ...; the loads of up to kChunk members are issued together
  constexpr int DPL = (D + 31) / 32;
  constexpr int kChunk = 8;
  float o[DPL];
#pragma unroll
  for (int u = 0; u < DPL; ++u) o[u] = 0.f;
  for (int m0 = warp; m0 < n; m0 += kDecWarps * kChunk) {
    int ra[kChunk], rb[kChunk];
    float pa[kChunk], pb[kChunk];
#pragma unroll
    for (int j = 0; j < kChunk; ++j) {
      const int m = m0 + j * kDecWarps;
      const bool in = m < n && s_ra[m] >= 0;
      const float p = in ? s_p[m] : 0.f;
      ra[j] = in ? s_ra[m] : 0;
      rb[j] = in && s_rb[m] >= 0 ? s_rb[m] : ra[j];
      pa[j] = p * (in ? s_wa[m] : 0.f);
      pb[j] = in && s_rb[m] >= 0 ? p * s_wb[m] : 0.f;
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
        for (int j = 0; j < kChunk; ++j) o[u] += pa[j] * xa[j] + pb[j] * xb[j];
      }
    }
  }
#pragma unroll
  for (int u = 0; u < DPL; ++u) {
    const int d = lane + 32 * u;
    if (d < D) s_o[warp][d] = o[u];
  }
  __syncthreads();
  const float inv = 1.f / l;
  for (int d = t; d < D; d += kDecThreads) {
    float acc = 0.f;
#pragma unroll
    for (int w = 0; w < kDecWarps; ++w) acc += s_o[w][d];
    store_elt<T>(O + d, acc * inv);
  }
}

template <typename T, int D>
cudaError_t launch_t(const DecArgs& a, long long units, cudaStream_t st) {
  trace_mark("decode", st, true);
  k_decode<T, D><<<(unsigned)units, kDecThreads, 0, st>>>(a);
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
  const bool f32 = pb.dtype == SA_DTYPE_F32;
  switch (pb.D) {
    case 16: return f32 ? launch_t<float, 16>(a, units, st) : launch_t<__nv_bfloat16, 16>(a, units, st);
    case 32: return f32 ? launch_t<float, 32>(a, units, st) : launch_t<__nv_bfloat16, 32>(a, units, st);
    case 64: return f32 ? launch_t<float, 64>(a, units, st) : launch_t<__nv_bfloat16, 64>(a, units, st);
    default: return f32 ? launch_t<float, 128>(a, units, st) : launch_t<__nv_bfloat16, 128>(a, units, st);
  }
}

}  // namespace sa
