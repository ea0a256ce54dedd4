// General kernels: every dtype (fp32, bf16) and head dim (16, 32, 64, 128),
// any window, sink count and offset table.  They read K/V rows straight
// through L1/L2 and rotate them on the fly from the RoPE table, one lane group
// of 8 lanes per query (or key).  Every member loop is warp-uniform: a lane
// group whose query lacks a member still takes part in the shuffles and
// discards the result, so no shuffle ever runs under divergence.
//
// Method: "Depth-Staggered Fibonacci Spacing for Sparse Attention" (C. A.
// Capps), technical summary, Methodology -- "Attended set" (window plus
// Fibonacci offsets), "Scaling" (d_k = alpha f_k), "Implementation" (linear
// K/V interpolation so gradients reach alpha; RoPE before the gather).
// Optional log-prior beta [units][T] on the offset members' scores
// ("pi-Attention: Periodic Sparse Transformers for Efficient Long-Context
// Modeling", Core components: local and skip logits fused in one softmax
// through a log-prior), with its gradient dbeta = sum of the offset members'
// dscores.
#include "sa_device.cuh"
#include "sa_internal.h"

namespace sa {

constexpr int kGenWarps = 4;                 // 128 threads
constexpr int kGenPerCta = kGenWarps * 4;    // 4 lane groups of 8 per warp

struct GenArgs {
  int B, H, T, W, n_off, S, n_tiles;
  float scale;
  int f[SA_MAX_OFFSETS];
  const void* q; const void* k; const void* v; const void* o; const void* dout;
  const float* lse; const float* alpha; const float2* rope;
  void* out_o; float* out_lse;               // forward outputs
  void* dq; void* dk; void* dv;              // backward outputs
  float* dvec;                               // D_i = dO_i . O_i   [units][T]
  float* dal_part;                           // [units][n_tiles]
  float* sink_k; float* sink_v;              // [units][n_tiles][S][D]
  const float* beta; float* dbeta;           // log-prior on offset members [units][T]
};

// Per-CTA offset geometry for this layer; returns nonzero when some offset
// has no defined row (the layer's outputs are then NaN).
__device__ __forceinline__ int cta_geometry(const GenArgs& a, int layer, OffGeo* sg) {
  int bad = 0;
  if ((int)threadIdx.x < a.n_off) {
    sg[threadIdx.x] = offset_geometry(__ldg(a.alpha + layer), a.f[threadIdx.x]);
    bad = !sg[threadIdx.x].ok;
  }
  return __syncthreads_or(bad);
}

// Row r of K rotated at position r, restricted to this lane's pairs.
template <typename T, int D>
__device__ __forceinline__ void load_krot(const T* K, const float2* rope, int r, int j0,
                                          float (&x1)[D / 16], float (&x2)[D / 16]) {
  constexpr int N = D / 16, HALF = D / 2;
  float2 cs[N];
  load_row<T, N>(K + (size_t)r * D + j0, x1);
  load_row<T, N>(K + (size_t)r * D + HALF + j0, x2);
  load_cs<N>(rope + (size_t)r * HALF + j0, cs);
  rope_fwd<N>(x1, x2, cs);
}

template <typename T, int D>
__device__ __forceinline__ void load_plain(const T* X, int r, int j0, float (&x1)[D / 16],
                                           float (&x2)[D / 16]) {
  load_row<T, D / 16>(X + (size_t)r * D + j0, x1);
  load_row<T, D / 16>(X + (size_t)r * D + D / 2 + j0, x2);
}

// ---------------------------------------------------------------------------
// Forward: online softmax over the members in order window, sinks, offsets.
template <typename T, int D>
__global__ void __launch_bounds__(kGenWarps * 32) k_fwd_general(const GenArgs a) {
  constexpr int N = D / 16, HALF = D / 2;
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int bad = cta_geometry(a, layer, sg);

  const int lane = threadIdx.x & 31, c = lane & 7;
  const int i = tile * kGenPerCta + (threadIdx.x >> 3);
  const bool active = i < a.T;
  const int qi = active ? i : a.T - 1;
  const int j0 = c * N;
  const size_t ub = (size_t)unit * a.T * D;
  const T* Q = reinterpret_cast<const T*>(a.q) + ub;
  const T* K = reinterpret_cast<const T*>(a.k) + ub;
  const T* V = reinterpret_cast<const T*>(a.v) + ub;

  float q1[N], q2[N];
  load_krot<T, D>(Q, a.rope, qi, j0, q1, q2);
#pragma unroll
  for (int h = 0; h < N; ++h) { q1[h] *= a.scale; q2[h] *= a.scale; }

  float m = -INFINITY, l = 0.f, o1[N], o2[N];
#pragma unroll
  for (int h = 0; h < N; ++h) { o1[h] = 0.f; o2[h] = 0.f; }
  const float prior = a.beta ? __ldg(a.beta + (size_t)unit * a.T + qi) : 0.f;

  auto visit = [&](bool valid, int ra, int rb, float wa, float wb, float bias) {
    float k1[N], k2[N];
    load_krot<T, D>(K, a.rope, valid ? ra : 0, j0, k1, k2);
    const bool two = valid && rb >= 0;
    if (two) {
      float b1[N], b2[N];
      load_krot<T, D>(K, a.rope, rb, j0, b1, b2);
#pragma unroll
      for (int h = 0; h < N; ++h) { k1[h] = wa * k1[h] + wb * b1[h]; k2[h] = wa * k2[h] + wb * b2[h]; }
    }
    float part = 0.f;
#pragma unroll
    for (int h = 0; h < N; ++h) part += q1[h] * k1[h] + q2[h] * k2[h];
    const float s = group8_sum(part) + bias;
    if (valid) {
      float v1[N], v2[N];
      load_plain<T, D>(V, ra, j0, v1, v2);
      if (two) {
        float b1[N], b2[N];
        load_plain<T, D>(V, rb, j0, b1, b2);
#pragma unroll
        for (int h = 0; h < N; ++h) { v1[h] = wa * v1[h] + wb * b1[h]; v2[h] = wa * v2[h] + wb * b2[h]; }
      }
      const float mn = fmaxf(m, s);
      const float corr = expf(m - mn), p = expf(s - mn);
      l = l * corr + p;
#pragma unroll
      for (int h = 0; h < N; ++h) { o1[h] = o1[h] * corr + p * v1[h]; o2[h] = o2[h] * corr + p * v2[h]; }
      m = mn;
    }
  };

  for (int t = 0; t < a.W; ++t) visit(qi - t >= 0, qi - t, -1, 1.f, 0.f, 0.f);
  for (int s = 0; s < a.S; ++s) visit(s <= qi, s, -1, 1.f, 0.f, 0.f);
  for (int k = 0; k < a.n_off; ++k) {
    const OffGeo g = sg[k];
    const int ra = qi - g.lo;
    visit(g.ok && qi - g.c >= 0, ra, g.w != 0.f ? ra - 1 : -1, g.wa, g.w, prior);
  }

  if (active) {
    const float inv = bad ? __int_as_float(0x7fc00000) : 1.f / l;
#pragma unroll
    for (int h = 0; h < N; ++h) { o1[h] *= inv; o2[h] *= inv; }
    T* O = reinterpret_cast<T*>(a.out_o) + ub + (size_t)i * D;
    store_row<T, N>(O + j0, o1);
    store_row<T, N>(O + HALF + j0, o2);
    if (c == 0 && a.out_lse)
      a.out_lse[(size_t)unit * a.T + i] = bad ? __int_as_float(0x7fc00000) : m + logf(l);
  }
}

// ---------------------------------------------------------------------------
// Backward, query side: dQ, D_i, d-alpha partials, sink-key partials.
template <typename T, int D>
__global__ void __launch_bounds__(kGenWarps * 32) k_bwd_q_general(const GenArgs a) {
  constexpr int N = D / 16, HALF = D / 2;
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ float s_red[kGenWarps];
  extern __shared__ float s_sink[];          // [kGenWarps][2][S][D]
  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int bad = cta_geometry(a, layer, sg);
  const float qnan = __int_as_float(0x7fc00000);

  const int lane = threadIdx.x & 31, c = lane & 7, warp = threadIdx.x >> 5;
  const int i = tile * kGenPerCta + (threadIdx.x >> 3);
  const bool active = i < a.T;
  const int qi = active ? i : a.T - 1;
  const int j0 = c * N;
  const size_t ub = (size_t)unit * a.T * D;
  const T* Q = reinterpret_cast<const T*>(a.q) + ub;
  const T* K = reinterpret_cast<const T*>(a.k) + ub;
  const T* V = reinterpret_cast<const T*>(a.v) + ub;
  const T* Og = reinterpret_cast<const T*>(a.o) + ub;
  const T* dO = reinterpret_cast<const T*>(a.dout) + ub;

  float q1[N], q2[N], g1[N], g2[N];
  load_krot<T, D>(Q, a.rope, qi, j0, q1, q2);
#pragma unroll
  for (int h = 0; h < N; ++h) { q1[h] *= a.scale; q2[h] *= a.scale; }
  load_plain<T, D>(dO, qi, j0, g1, g2);
  float Dsum;
  {
    float o1[N], o2[N];
    load_plain<T, D>(Og, qi, j0, o1, o2);
    float part = 0.f;
#pragma unroll
    for (int h = 0; h < N; ++h) part += g1[h] * o1[h] + g2[h] * o2[h];
    Dsum = group8_sum(part);
  }
  const float lse_i = __ldg(a.lse + (size_t)unit * a.T + qi);
  const float prior = a.beta ? __ldg(a.beta + (size_t)unit * a.T + qi) : 0.f;
  float dq1[N], dq2[N];
#pragma unroll
  for (int h = 0; h < N; ++h) { dq1[h] = 0.f; dq2[h] = 0.f; }
  float dal = 0.f, dprior = 0.f;

  // One member: returns its dsigma (g) and p; both 0 when it does not exist.
  // koff >= 0 marks an offset member (adds its d-alpha term).
  auto visit = [&](bool valid, int ra, int rb, float wa, float wb, int koff, float& g_out,
                   float& p_out) {
    float ka1[N], ka2[N], va1[N], va2[N];
    const int r0 = valid ? ra : 0;
    load_krot<T, D>(K, a.rope, r0, j0, ka1, ka2);
    load_plain<T, D>(V, r0, j0, va1, va2);
    // second row: read when interpolating, and for d-alpha whenever it exists
    const int rs = (koff >= 0) ? ra - 1 : -1;
    const bool has_b = valid && rs >= 0;
    float kb1[N], kb2[N], vb1[N], vb2[N];
#pragma unroll
    for (int h = 0; h < N; ++h) { kb1[h] = kb2[h] = vb1[h] = vb2[h] = 0.f; }
    if (has_b) {
      load_krot<T, D>(K, a.rope, rs, j0, kb1, kb2);
      load_plain<T, D>(V, rs, j0, vb1, vb2);
    }
    const bool two = valid && rb >= 0;
    float s_part = 0.f, dp_part = 0.f;
    float key1[N], key2[N];
#pragma unroll
    for (int h = 0; h < N; ++h) {
      key1[h] = two ? wa * ka1[h] + wb * kb1[h] : ka1[h];
      key2[h] = two ? wa * ka2[h] + wb * kb2[h] : ka2[h];
      const float v1 = two ? wa * va1[h] + wb * vb1[h] : va1[h];
      const float v2 = two ? wa * va2[h] + wb * vb2[h] : va2[h];
      s_part += q1[h] * key1[h] + q2[h] * key2[h];
      dp_part += g1[h] * v1 + g2[h] * v2;
    }
    const float s = group8_sum(s_part) + (koff >= 0 ? prior : 0.f);
    const float dp = group8_sum(dp_part);
    const float p = valid ? expf(s - lse_i) : 0.f;
    const float g = p * (dp - Dsum);
    if (valid) {
#pragma unroll
      for (int h = 0; h < N; ++h) { dq1[h] += g * key1[h]; dq2[h] += g * key2[h]; }
    }
    if (koff >= 0) dprior += g;
    if (has_b) {
      float t = 0.f;
#pragma unroll
      for (int h = 0; h < N; ++h)
        t += g * (q1[h] * (kb1[h] - ka1[h]) + q2[h] * (kb2[h] - ka2[h])) +
             p * (g1[h] * (vb1[h] - va1[h]) + g2[h] * (vb2[h] - va2[h]));
      dal += (float)sg[koff].f * t;
    }
    g_out = g;
    p_out = p;
  };

  // lanes past the end (i >= T) take part in the shuffles but own no member
  float gdummy, pdummy;
  for (int t = 0; t < a.W; ++t)
    visit(active && qi - t >= 0, qi - t, -1, 1.f, 0.f, -1, gdummy, pdummy);
  for (int k = 0; k < a.n_off; ++k) {
    const OffGeo g = sg[k];
    const int ra = qi - g.lo;
    visit(active && g.ok && qi - g.c >= 0, ra, g.w != 0.f ? ra - 1 : -1, g.wa, g.w, k, gdummy,
          pdummy);
  }
  // Sinks: this warp's contributions to the sink rows' dK~ and dV, summed over
  // its four lane groups (fixed butterfly order), parked in shared memory.
  for (int s = 0; s < a.S; ++s) {
    float gs, ps;
    visit(active && s <= qi, s, -1, 1.f, 0.f, -1, gs, ps);
    float ck1[N], ck2[N], cv1[N], cv2[N];
#pragma unroll
    for (int h = 0; h < N; ++h) {
      ck1[h] = gs * q1[h]; ck2[h] = gs * q2[h];
      cv1[h] = ps * g1[h]; cv2[h] = ps * g2[h];
#pragma unroll
      for (int off = 8; off <= 16; off <<= 1) {
        ck1[h] += __shfl_xor_sync(0xffffffffu, ck1[h], off);
        ck2[h] += __shfl_xor_sync(0xffffffffu, ck2[h], off);
        cv1[h] += __shfl_xor_sync(0xffffffffu, cv1[h], off);
        cv2[h] += __shfl_xor_sync(0xffffffffu, cv2[h], off);
      }
    }
    if (lane < 8) {
      float* sk = s_sink + ((size_t)(warp * 2 + 0) * a.S + s) * D;
      float* sv = s_sink + ((size_t)(warp * 2 + 1) * a.S + s) * D;
#pragma unroll
      for (int h = 0; h < N; ++h) {
        sk[j0 + h] = ck1[h]; sk[HALF + j0 + h] = ck2[h];
        sv[j0 + h] = cv1[h]; sv[HALF + j0 + h] = cv2[h];
      }
    }
  }

  if (active) {
    float2 cs[N];
    load_cs<N>(a.rope + (size_t)qi * HALF + j0, cs);
    rope_bwd<N>(dq1, dq2, cs);
#pragma unroll
    for (int h = 0; h < N; ++h) {
      dq1[h] = bad ? qnan : dq1[h] * a.scale;
      dq2[h] = bad ? qnan : dq2[h] * a.scale;
    }
    T* dQ = reinterpret_cast<T*>(a.dq) + ub + (size_t)i * D;
    store_row<T, N>(dQ + j0, dq1);
    store_row<T, N>(dQ + HALF + j0, dq2);
    if (c == 0) a.dvec[(size_t)unit * a.T + i] = Dsum;
    if (c == 0 && a.dbeta) a.dbeta[(size_t)unit * a.T + i] = bad ? qnan : dprior;
  }
  // d-alpha partial of this CTA: butterfly over the warp, then warps in order.
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) dal += __shfl_xor_sync(0xffffffffu, dal, off);
  if (lane == 0) s_red[warp] = dal;
  __syncthreads();
  if (threadIdx.x == 0) {
    float acc = 0.f;
    for (int w = 0; w < kGenWarps; ++w) acc += s_red[w];
    a.dal_part[(size_t)unit * a.n_tiles + tile] = bad ? qnan : acc;
  }
  if (a.S > 0) {
    const size_t per = (size_t)a.S * D;
    float* gk = a.sink_k + ((size_t)unit * a.n_tiles + tile) * per;
    float* gv = a.sink_v + ((size_t)unit * a.n_tiles + tile) * per;
    for (size_t e = threadIdx.x; e < per; e += blockDim.x) {
      float ak = 0.f, av = 0.f;
      for (int w = 0; w < kGenWarps; ++w) {
        ak += s_sink[(size_t)(w * 2 + 0) * per + e];
        av += s_sink[(size_t)(w * 2 + 1) * per + e];
      }
      gk[e] = ak;
      gv[e] = av;
    }
  }
}

// ---------------------------------------------------------------------------
// Backward, key side: each key row r walks the fixed set of queries whose
// members read it, recomputes their scores, and accumulates dK and dV with no
// atomics.  Members of a query that read row r:
//   window t      : query r + t                       (weight 1)
//   offset k, row a = i - lo   : query r + lo          (weight 1 - w)
//   offset k, row b = i - lo-1 : query r + lo + 1      (weight w, when w != 0)
// Sink rows r < S add the query-side partials of their sink members.
template <typename T, int D>
__global__ void __launch_bounds__(kGenWarps * 32) k_bwd_kv_general(const GenArgs a) {
  constexpr int N = D / 16, HALF = D / 2;
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int bad = cta_geometry(a, layer, sg);
  const float qnan = __int_as_float(0x7fc00000);

  const int lane = threadIdx.x & 31, c = lane & 7;
  const int r = tile * kGenPerCta + (threadIdx.x >> 3);
  const bool active = r < a.T;
  const int rr = active ? r : a.T - 1;
  const int j0 = c * N;
  const size_t ub = (size_t)unit * a.T * D;
  const T* Q = reinterpret_cast<const T*>(a.q) + ub;
  const T* K = reinterpret_cast<const T*>(a.k) + ub;
  const T* V = reinterpret_cast<const T*>(a.v) + ub;
  const T* dO = reinterpret_cast<const T*>(a.dout) + ub;
  const float* lse = a.lse + (size_t)unit * a.T;
  const float* dvec = a.dvec + (size_t)unit * a.T;

  float kr1[N], kr2[N], vr1[N], vr2[N];
  load_krot<T, D>(K, a.rope, rr, j0, kr1, kr2);
  load_plain<T, D>(V, rr, j0, vr1, vr2);
  float dk1[N], dk2[N], dv1[N], dv2[N];
#pragma unroll
  for (int h = 0; h < N; ++h) { dk1[h] = dk2[h] = dv1[h] = dv2[h] = 0.f; }

  // Query i's member reads row r with weight wr and row `other` with wo;
  // offset members carry query i's log-prior.
  auto source = [&](bool valid, int i, int other, float wr, float wo, bool off) {
    const int ii = valid ? i : 0;
    float q1[N], q2[N], g1[N], g2[N];
    load_krot<T, D>(Q, a.rope, ii, j0, q1, q2);
#pragma unroll
    for (int h = 0; h < N; ++h) { q1[h] *= a.scale; q2[h] *= a.scale; }
    load_plain<T, D>(dO, ii, j0, g1, g2);
    float key1[N], key2[N], val1[N], val2[N];
#pragma unroll
    for (int h = 0; h < N; ++h) { key1[h] = kr1[h]; key2[h] = kr2[h]; val1[h] = vr1[h]; val2[h] = vr2[h]; }
    if (valid && other >= 0) {
      float ko1[N], ko2[N], vo1[N], vo2[N];
      load_krot<T, D>(K, a.rope, other, j0, ko1, ko2);
      load_plain<T, D>(V, other, j0, vo1, vo2);
#pragma unroll
      for (int h = 0; h < N; ++h) {
        key1[h] = wr * kr1[h] + wo * ko1[h]; key2[h] = wr * kr2[h] + wo * ko2[h];
        val1[h] = wr * vr1[h] + wo * vo1[h]; val2[h] = wr * vr2[h] + wo * vo2[h];
      }
    }
    float s_part = 0.f, dp_part = 0.f;
#pragma unroll
    for (int h = 0; h < N; ++h) {
      s_part += q1[h] * key1[h] + q2[h] * key2[h];
      dp_part += g1[h] * val1[h] + g2[h] * val2[h];
    }
    const float s = group8_sum(s_part) + ((off && a.beta) ? __ldg(a.beta + (size_t)unit * a.T + ii) : 0.f);
    const float dp = group8_sum(dp_part);
    if (valid) {
      const float p = expf(s - __ldg(lse + ii));
      const float g = p * (dp - __ldg(dvec + ii));
      const float gw = wr * g, pw = wr * p;
#pragma unroll
      for (int h = 0; h < N; ++h) {
        dk1[h] += gw * q1[h]; dk2[h] += gw * q2[h];
        dv1[h] += pw * g1[h]; dv2[h] += pw * g2[h];
      }
    }
  };

  for (int t = 0; t < a.W; ++t) source(active && rr + t < a.T, rr + t, -1, 1.f, 0.f, false);
  for (int k = 0; k < a.n_off; ++k) {
    const OffGeo g = sg[k];
    if (!g.ok) continue;                                     // CTA-uniform
    const int ia = rr + g.lo;                                // r is row a
    source(active && ia < a.T && ia - g.c >= 0, ia, g.w != 0.f ? rr - 1 : -1, g.wa, g.w, true);
    if (g.w != 0.f) {                                        // r is row b
      const int ib = rr + g.lo + 1;
      source(active && ib < a.T, ib, rr + 1, g.w, g.wa, true);
    }
  }
  if (active && rr < a.S) {
    const size_t per = (size_t)a.S * D;
    const float* gk = a.sink_k + (size_t)unit * a.n_tiles * per + (size_t)rr * D;
    const float* gv = a.sink_v + (size_t)unit * a.n_tiles * per + (size_t)rr * D;
    // four tiles' loads in flight (the sum stays in tile order)
#pragma unroll 4
    for (int t = 0; t < a.n_tiles; ++t) {
#pragma unroll
      for (int h = 0; h < N; ++h) {
        dk1[h] += gk[t * per + j0 + h]; dk2[h] += gk[t * per + HALF + j0 + h];
        dv1[h] += gv[t * per + j0 + h]; dv2[h] += gv[t * per + HALF + j0 + h];
      }
    }
  }
  if (active) {
    float2 cs[N];
    load_cs<N>(a.rope + (size_t)rr * HALF + j0, cs);
    rope_bwd<N>(dk1, dk2, cs);
    if (bad) {
#pragma unroll
      for (int h = 0; h < N; ++h) dk1[h] = dk2[h] = dv1[h] = dv2[h] = qnan;
    }
    T* dK = reinterpret_cast<T*>(a.dk) + ub + (size_t)r * D;
    T* dV = reinterpret_cast<T*>(a.dv) + ub + (size_t)r * D;
    store_row<T, N>(dK + j0, dk1);
    store_row<T, N>(dK + HALF + j0, dk2);
    store_row<T, N>(dV + j0, dv1);
    store_row<T, N>(dV + HALF + j0, dv2);
  }
}

// Per-layer d-alpha: fixed-order sum of the per-CTA partials of one layer.
__global__ void __launch_bounds__(256) k_reduce_dalpha(const float* part, int per_layer, float* dalpha) {
  __shared__ float s[256];
  const float* p = part + (size_t)blockIdx.x * per_layer;
  float acc = 0.f;
  for (int e = threadIdx.x; e < per_layer; e += 256) acc += p[e];
  s[threadIdx.x] = acc;
  __syncthreads();
  for (int w = 128; w >= 1; w >>= 1) {
    if ((int)threadIdx.x < w) s[threadIdx.x] += s[threadIdx.x + w];
    __syncthreads();
  }
  if (threadIdx.x == 0) dalpha[blockIdx.x] = s[0];
}

// RoPE table: tab[t][j] = (cos, sin)(t * base^(-2j/D)) in double, rounded.
__global__ void k_rope_table(float2* tab, int T, int D, double base) {
  const int half = D / 2;
  const size_t n = (size_t)T * half;
  for (size_t e = blockIdx.x * (size_t)blockDim.x + threadIdx.x; e < n;
       e += (size_t)gridDim.x * blockDim.x) {
    const int t = (int)(e / half), j = (int)(e % half);
    const double theta = pow(base, -2.0 * (double)j / (double)D);
    double sn, cs;
    sincos((double)t * theta, &sn, &cs);
    tab[e] = make_float2((float)cs, (float)sn);
  }
}

// ---------------------------------------------------------------------------
static GenArgs make_args(const Problem& pb) {
  GenArgs a = {};
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = (pb.T + kGenPerCta - 1) / kGenPerCta;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  return a;
}

BwdLayout general_bwd_layout(const Problem& pb) {
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  BwdLayout lay;
  lay.n_qtiles = (pb.T + kGenPerCta - 1) / kGenPerCta;
  const size_t units = (size_t)pb.units();
  lay.d_off = 0;
  lay.dal_off = up(units * pb.T * sizeof(float));
  lay.sink_off = lay.dal_off + up(units * lay.n_qtiles * sizeof(float));
  lay.total = lay.sink_off + up(2 * units * lay.n_qtiles * (size_t)pb.S * pb.D * sizeof(float));
  return lay;
}

cudaError_t launch_reduce_dalpha(const float* part, int L, int per_layer, float* dalpha,
                                 cudaStream_t st) {
  trace_mark("reduce_dalpha", st, true);
  k_reduce_dalpha<<<L, 256, 0, st>>>(part, per_layer, dalpha);
  trace_mark("reduce_dalpha", st, false);
  return cudaGetLastError();
}

cudaError_t launch_rope_table(float2* tab, int T, int D, double base, cudaStream_t st) {
  const size_t n = (size_t)T * (D / 2);
  const int grid = (int)((n + 255) / 256 < 4096 ? (n + 255) / 256 : 4096);
  k_rope_table<<<grid, 256, 0, st>>>(tab, T, D, base);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t fwd_t(const Problem& pb, const FwdPtrs& p, cudaStream_t st) {
  GenArgs a = make_args(pb);
  a.q = p.q; a.k = p.k; a.v = p.v; a.alpha = p.alpha; a.rope = p.rope;
  a.out_o = p.o; a.out_lse = p.lse; a.beta = p.beta;
  const long long grid = (long long)pb.units() * a.n_tiles;
  trace_mark("fwd_general", st, true);
  k_fwd_general<T, D><<<(unsigned)grid, kGenWarps * 32, 0, st>>>(a);
  trace_mark("fwd_general", st, false);
  return cudaGetLastError();
}

template <typename T, int D>
static cudaError_t bwd_t(const Problem& pb, const BwdPtrs& p, cudaStream_t st, int* launches) {
  GenArgs a = make_args(pb);
  const BwdLayout lay = general_bwd_layout(pb);
  char* ws = reinterpret_cast<char*>(p.workspace);
  a.q = p.q; a.k = p.k; a.v = p.v; a.o = p.o; a.dout = p.dout; a.lse = p.lse;
  a.alpha = p.alpha; a.rope = p.rope;
  a.dq = p.dq; a.dk = p.dk; a.dv = p.dv;
  a.beta = p.beta; a.dbeta = p.dbeta;
  a.dvec = reinterpret_cast<float*>(ws + lay.d_off);
  a.dal_part = reinterpret_cast<float*>(ws + lay.dal_off);
  a.sink_k = reinterpret_cast<float*>(ws + lay.sink_off);
  a.sink_v = a.sink_k + (size_t)pb.units() * lay.n_qtiles * pb.S * pb.D;
  const unsigned grid = (unsigned)((long long)pb.units() * a.n_tiles);
  const size_t smem = (size_t)kGenWarps * 2 * pb.S * pb.D * sizeof(float);
  if (smem > 48 * 1024) {
    cudaError_t e = cudaFuncSetAttribute(k_bwd_q_general<T, D>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem);
    if (e != cudaSuccess) return e;
  }
  trace_mark("bwd_q_general", st, true);
  k_bwd_q_general<T, D><<<grid, kGenWarps * 32, smem, st>>>(a);
  trace_mark("bwd_q_general", st, false);
  cudaError_t e = cudaGetLastError();
  if (e != cudaSuccess) return e;
  trace_mark("bwd_kv_general", st, true);
  k_bwd_kv_general<T, D><<<grid, kGenWarps * 32, 0, st>>>(a);
  trace_mark("bwd_kv_general", st, false);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_reduce_dalpha(a.dal_part, pb.L, pb.B * pb.H * a.n_tiles, p.dalpha, st)) !=
      cudaSuccess)
    return e;
  *launches += 3;
  return cudaSuccess;
}

template <typename T>
static cudaError_t fwd_d(const Problem& pb, const FwdPtrs& p, cudaStream_t st) {
  switch (pb.D) {
    case 16: return fwd_t<T, 16>(pb, p, st);
    case 32: return fwd_t<T, 32>(pb, p, st);
    case 64: return fwd_t<T, 64>(pb, p, st);
    case 128: return fwd_t<T, 128>(pb, p, st);
  }
  return cudaErrorInvalidValue;
}

template <typename T>
static cudaError_t bwd_d(const Problem& pb, const BwdPtrs& p, cudaStream_t st, int* n) {
  switch (pb.D) {
    case 16: return bwd_t<T, 16>(pb, p, st, n);
    case 32: return bwd_t<T, 32>(pb, p, st, n);
    case 64: return bwd_t<T, 64>(pb, p, st, n);
    case 128: return bwd_t<T, 128>(pb, p, st, n);
  }
  return cudaErrorInvalidValue;
}

cudaError_t launch_fwd_general(const Problem& pb, const FwdPtrs& p, cudaStream_t st, int* launches) {
  cudaError_t e = pb.dtype == SA_DTYPE_F32 ? fwd_d<float>(pb, p, st) : fwd_d<__nv_bfloat16>(pb, p, st);
  if (e == cudaSuccess) *launches += 1;
  return e;
}

cudaError_t launch_bwd_general(const Problem& pb, const BwdPtrs& p, cudaStream_t st, int* launches) {
  return pb.dtype == SA_DTYPE_F32 ? bwd_d<float>(pb, p, st, launches)
                                  : bwd_d<__nv_bfloat16>(pb, p, st, launches);
}

}  // namespace sa
