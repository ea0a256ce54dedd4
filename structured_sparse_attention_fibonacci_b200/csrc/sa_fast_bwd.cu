// Staged backward for bf16 inputs with head dim 64.  Same tiling, lane mapping
// and lag-ordered row ring as the staged forward (sa_fast.cu).
//
// Query side (k_bwd_q_fast), one CTA per tile of 128 queries, three passes:
//   1. K ring: scores sigma_m = q_hat . key_m and, per offset, the row-score
//      difference dtau = q_hat . (K~[i-lo-1] - K~[i-lo]);
//   2. V ring: dp_m = dO . value_m and dpi = dO . (V[i-lo-1] - V[i-lo]);
//      owner lane: p_m = softmax of its own scores, D_i = sum_m p_m dp_m,
//      g_m = p_m (dp_m - D_i), d-alpha += f_k (g_k dtau_k + p_k dpi_k)
//      (the gradient through w_k = alpha f_k - lo_k: "Implementation" lets
//      gradients reach alpha through the interpolation);
//   3. K ring again: dq_hat = sum_m g_m key_m, dQ = scale * RoPE^T(dq_hat).
//   It also writes, per query, the weights the key side needs -- the window
//   weights with the near offsets folded in (G for dK, P for dV) and g_k, p_k
//   of every far offset -- plus per-tile d-alpha and sink-row partials.
// Key side (k_bwd_kv_fast), one CTA per tile of 128 keys, no atomics: the
//   source queries of a key tile are staged in increasing lead order (rotated,
//   scaled Q rows for dK; dO rows for dV, with their weights) and every key
//   accumulates its own dK~ / dV in registers:
//     window lead t : query r + t        (weight G[t] / P[t])
//     far offset k  : query r + lo       (row a, weight (1-w) g_k / (1-w) p_k)
//                     query r + lo + 1   (row b, weight w g_k / w p_k)
//   then dK = RoPE^T(dK~).  Sink rows add the query side's per-tile partials.
#include <algorithm>

#include "sa_fast_common.cuh"

namespace sa {

namespace {

using namespace fast;

struct FastBwdArgs {
  int B, H, T, W, n_off, S, n_tiles;
  int ring_rows, sc_stride, gpart, slot_pitch, wpitch;
  float scale;
  int f[SA_MAX_OFFSETS];                 // ascending
  const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
  const __nv_bfloat16* dout;
  const float* lse; const float* alpha; const float2* rope;
  __nv_bfloat16* dq; __nv_bfloat16* dk; __nv_bfloat16* dv;
  __nv_bfloat16* slots;                  // [units][T][slot_pitch]: G | P, each gpart wide
  float* dal_part;                       // [units][n_tiles]
  float* sink_k; float* sink_v;          // [units][n_tiles][S][64]
};

// Both rows of an offset stay inside the window: the backward folds it (its
// d-alpha term needs both rows even when w == 0).
__device__ __forceinline__ int fold_bwd(const OffGeo& g, int W) { return g.ok && g.lo + 1 <= W - 1; }

__device__ __forceinline__ int cta_geometry_bwd(const FastBwdArgs& a, int layer, OffGeo* sg,
                                                int* s_fold) {
  int bad = 0;
  if ((int)threadIdx.x < a.n_off) {
    const OffGeo g = offset_geometry(__ldg(a.alpha + layer), a.f[threadIdx.x]);
    sg[threadIdx.x] = g;
    s_fold[threadIdx.x] = fold_bwd(g, a.W);
    bad = !g.ok;
  }
  return __syncthreads_or(bad);
}

// Next offset after k that the backward does not fold (n_off when none).
__device__ __forceinline__ int next_far(const int* s_fold, int k, int n_off) {
  ++k;
  while (k < n_off && s_fold[k]) ++k;
  return k;
}
// Rows a far member needs on the query side for the tile [i0, i0 + M), both
// interpolation rows (the d-alpha term reads row i-lo-1 even when w == 0).
__device__ __forceinline__ int qseg_lo(const OffGeo& g, int i0) { return max(0, i0 - g.lo - 1); }
__device__ __forceinline__ int qseg_hi(const OffGeo& g, int i0, int T) {
  return max(0, min(T, i0 + kFastM - g.lo));
}

// Load this lane's 16 dims of 4 consecutive rows of X (bf16 [T][64]), rows
// clamped to T-1; optionally rotated (RoPE at the row's position) and scaled.
template <bool ROT>
__device__ __forceinline__ void load_lane_rows(const __nv_bfloat16* X, const float2* rope, int r0,
                                               int T, int c, float scale, float (&x)[4][16]) {
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const int row = min(r0 + qq, T - 1);
    const uint4* g = reinterpret_cast<const uint4*>(X + (size_t)row * kD);
    float x1[8], x2[8];
    unpack8(__ldg(g + c), x1);
    unpack8(__ldg(g + c + 4), x2);
    if (ROT) {
      const float4* cs = reinterpret_cast<const float4*>(rope + (size_t)row * 32 + 8 * c);
#pragma unroll
      for (int h = 0; h < 8; h += 2) {
        const float4 t = __ldg(cs + h / 2);
        x[qq][h] = (x1[h] * t.x - x2[h] * t.y) * scale;
        x[qq][h + 8] = (x2[h] * t.x + x1[h] * t.y) * scale;
        x[qq][h + 1] = (x1[h + 1] * t.z - x2[h + 1] * t.w) * scale;
        x[qq][h + 9] = (x2[h + 1] * t.z + x1[h + 1] * t.w) * scale;
      }
    } else {
#pragma unroll
      for (int h = 0; h < 8; ++h) { x[qq][h] = x1[h]; x[qq][h + 8] = x2[h]; }
    }
  }
}

// Window dot products for lags [d0, d0+LC) against the ring (same row walk as
// the forward's window scores); results land in out_row[d0 .. d0+LC).
template <int LC, bool F16>
__device__ __forceinline__ void window_dots(const uint4* ring, int RB, int ig, int d0, int c,
                                            const float (&q)[4][16], float* out_row,
                                            int i_own, float* mx) {
  float acc[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) acc[a][l] = 0.f;
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    const int row = max(ig + 3 - d0 - u, 0);
    float x[16];
    ring_load<F16>(ring, row & (RB - 1), c, x);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int l = a + u - 3;
      if (l >= 0 && l < LC) acc[a][l] += dot16(q[a], x);
    }
  }
  float out[LC];
  reduce_scatter4<LC>(acc, out, c);
#pragma unroll
  for (int l = 0; l < LC; ++l) {
    out_row[d0 + l] = out[l];
    if (mx && i_own - (d0 + l) >= 0) *mx = fmaxf(*mx, out[l]);
  }
}

// o[q] += w[q][lag] * ring row, over lags [d0, d0+LC) (weights per query row).
template <int LC, bool F16>
__device__ __forceinline__ void window_axpy(const uint4* ring, int RB, int ig, int d0, int c,
                                            const float* wrow0, int stride, float (&o)[4][16]) {
  float pw[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) pw[a][l] = wrow0[a * stride + d0 + l];
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    const int row = max(ig + 3 - d0 - u, 0);
    float x[16];
    ring_load<F16>(ring, row & (RB - 1), c, x);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int l = a + u - 3;
      if (l >= 0 && l < LC) axpy16(o[a], pw[a][l], x);
    }
  }
}

#define SA_WINDOW_CHUNKS(W, CALL)                                   \
  {                                                                 \
    int d0 = 0;                                                     \
    while ((W) - d0 >= 8) { CALL(8); d0 += 8; }                     \
    if ((W) - d0 >= 4) { CALL(4); d0 += 4; }                        \
    if ((W) - d0 >= 2) { CALL(2); d0 += 2; }                        \
    if ((W) - d0 >= 1) { CALL(1); d0 += 1; }                        \
  }

// One pass of dot products of the lane's 4 rows `x` with every member
// (window, sinks, far offsets): member value into val_row, and for far
// offsets the row difference (row b minus row a) into diff_row[k].
template <bool ROT>
__device__ __forceinline__ void member_dots(const FastBwdArgs& a, uint4* ring, uint4* sinkb,
                                            const __nv_bfloat16* src, const OffGeo* sg,
                                            const int* s_fold, int i0, int ig, int c, int S_rows,
                                            const float (&x)[4][16], float* val_row,
                                            float* diff_row, int i_own, float* mx) {
  constexpr int M = kFastM;
  const int T = a.T, W = a.W, S = a.S, RB = a.ring_rows;
  const int win_lo = max(0, i0 - W + 1), win_hi = min(T, i0 + M);
  __syncthreads();
  stage_rows<ROT>(ring, RB, src, a.rope, win_lo, win_hi);
  stage_sinks<ROT>(sinkb, S_rows, src, a.rope);
  __syncthreads();
#define SA_CALL(LC) window_dots<LC, ROT>(ring, RB, ig, d0, c, x, val_row, i_own, mx)
  SA_WINDOW_CHUNKS(W, SA_CALL)
#undef SA_CALL
  for (int s0 = 0; s0 < S; s0 += 4) {
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float y[16];
      sink_load<ROT>(sinkb, min(s0 + j, S - 1), c, y);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) acc[qq][j] = dot16(x[qq], y);
    }
    float out[4];
    reduce_scatter4<4>(acc, out, c);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < S) {
        val_row[W + s0 + j] = out[j];
        if (mx && s0 + j <= i_own) *mx = fmaxf(*mx, out[j]);
      }
  }
  // far offsets, staged in batches whose rows span at most RB rows
  int low = win_lo;
  int kb = next_far(s_fold, -1, a.n_off);
  while (kb < a.n_off) {
    const int hi = qseg_hi(sg[kb], i0, T);
    int last = kb, nx = next_far(s_fold, kb, a.n_off);
    while (nx < a.n_off && hi - qseg_lo(sg[nx], i0) <= RB) {
      last = nx;
      nx = next_far(s_fold, nx, a.n_off);
    }
    const int lo_row = qseg_lo(sg[last], i0);
    if (lo_row < low && lo_row < hi) {
      __syncthreads();
      stage_rows<ROT>(ring, RB, src, a.rope, lo_row, min(hi, low));
      low = lo_row;
      __syncthreads();
    }
    for (int kk = kb; kk < nx; kk = next_far(s_fold, kk, a.n_off)) {
    const OffGeo g = sg[kk];
    float pa[4], pb[4];
#pragma unroll
    for (int u = 0; u < 5; ++u) {
      const int row = max(ig - g.lo - 1 + u, 0);
      float y[16];
      ring_load<ROT>(ring, row & (RB - 1), c, y);
      if (u <= 3) pb[u] = dot16(x[u], y);
      if (u >= 1) pa[u - 1] = dot16(x[u - 1], y);
    }
    float part[4][2];
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      part[qq][0] = g.wa * pa[qq] + g.w * pb[qq];
      part[qq][1] = pb[qq] - pa[qq];
    }
    float out[2];
    reduce_scatter4<2>(part, out, c);
    val_row[W + S + kk] = out[0];
    diff_row[kk] = out[1];
    if (mx && i_own - g.c >= 0) *mx = fmaxf(*mx, out[0]);
    }
    kb = nx;
  }
}

__global__ void __launch_bounds__(kFastM) k_bwd_q_fast(const FastBwdArgs a) {
  constexpr int M = kFastM;
  extern __shared__ __align__(16) unsigned char smem[];
  const int T = a.T, W = a.W, S = a.S, n_off = a.n_off, RB = a.ring_rows;
  const int st = a.sc_stride;
  uint4* ring = reinterpret_cast<uint4*>(smem);
  const size_t ring_a = (size_t)RB * 128, ring_b = (size_t)(M / 32) * 2 * S * kD * sizeof(float);
  const size_t ring_bytes = ring_a > ring_b ? ring_a : ring_b;
  uint4* sinkb = reinterpret_cast<uint4*>(smem + ring_bytes);
  float* sc = reinterpret_cast<float*>(sinkb + (size_t)S * kChunks);   // sigma, then g
  float* dpb = sc + (size_t)M * st;                                  // dp, then p
  float* dts = dpb + (size_t)M * st;                                 // [M][n_off] dtau
  float* dps = dts + (size_t)M * n_off;                              // [M][n_off] dpi
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_fold[SA_MAX_OFFSETS];
  __shared__ float s_red[M / 32];

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int i0 = tile * M;
  const int t = threadIdx.x, gid = t >> 2, c = t & 3, lane = t & 31, warp = t >> 5;
  const int ig = i0 + 4 * gid;
  const size_t ub = (size_t)unit * T * kD;
  const __nv_bfloat16* Q = a.q + ub;
  const __nv_bfloat16* K = a.k + ub;
  const __nv_bfloat16* V = a.v + ub;
  const __nv_bfloat16* dO = a.dout + ub;
  const float qnan = __int_as_float(0x7fc00000);

  const int bad = cta_geometry_bwd(a, layer, sg, s_fold);
  if (bad) {  // NaN dQ and d-alpha partial; the key side writes NaN dK, dV
    for (int e = t; e < M * kChunks; e += M) {
      const int i = i0 + e / kChunks;
      if (i < T) {
        float x[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) x[h] = qnan;
        reinterpret_cast<uint4*>(a.dq + ub + (size_t)i * kD)[e % kChunks] = pack8(x);
      }
    }
    if (t == 0) a.dal_part[(size_t)unit * a.n_tiles + tile] = qnan;
    return;
  }
  // zero the ring rows and the sink rows (the sink buffer follows the ring
  // region, which may be larger than the ring when it doubles as reduction space)
  for (int e = t; e < RB * kChunks; e += M) ring[e] = make_uint4(0, 0, 0, 0);
  for (int e = t; e < S * kChunks; e += M) sinkb[e] = make_uint4(0, 0, 0, 0);
  const int S_rows = min(S, T);
  const int lr = 4 * gid + c;
  float* my_sc = sc + (size_t)lr * st;
  float* my_dp = dpb + (size_t)lr * st;
  float* my_dt = dts + (size_t)lr * n_off;
  float* my_dpi = dps + (size_t)lr * n_off;

  float x[4][16];
  // pass 1: scores and row-score differences (K ring)
  load_lane_rows<true>(Q, a.rope, ig, T, c, a.scale * kKeyUnstage, x);
  float mx = -INFINITY;     // running max of this lane's query's valid scores
  member_dots<true>(a, ring, sinkb, K, sg, s_fold, i0, ig, c, S_rows, x, my_sc, my_dt, ig + c, &mx);
  // pass 2: dO . values and value differences (V ring)
  load_lane_rows<false>(dO, a.rope, ig, T, c, 1.f, x);
  member_dots<false>(a, ring, sinkb, V, sg, s_fold, i0, ig, c, S_rows, x, my_dp, my_dpi, ig + c,
                     nullptr);
  __syncthreads();

  // owner lane: probabilities, D_i, dsigma, d-alpha, folded window weights
  float dal = 0.f;
  {
    const int i = ig + c;
    const int n_slot = W + S + n_off;
    __nv_bfloat16* out = a.slots + ((size_t)unit * T + min(i, T - 1)) * a.slot_pitch;
    if (i < T) {
      for (int kk = 0; kk < n_off; ++kk) {
        if (!s_fold[kk]) continue;
        const OffGeo g = sg[kk];
        my_sc[W + S + kk] = g.wa * my_sc[g.lo] + g.w * my_sc[g.lo + 1];
        my_dp[W + S + kk] = g.wa * my_dp[g.lo] + g.w * my_dp[g.lo + 1];
        my_dt[kk] = my_sc[g.lo + 1] - my_sc[g.lo];
        my_dpi[kk] = my_dp[g.lo + 1] - my_dp[g.lo];
      }
      // softmax normalised from these scores (not the forward's LSE), so
      // that sum_m p_m = 1 and sum_m g_m = 0 hold for the values used here
      for (int kk = 0; kk < n_off; ++kk)      // near offsets join the running max
        if (s_fold[kk] && i - sg[kk].c >= 0) mx = fmaxf(mx, my_sc[W + S + kk]);
      float l = 0.f, edp = 0.f;
      for (int m = 0; m < n_slot; ++m) {
        bool valid;
        if (m < W) valid = i - m >= 0;
        else if (m < W + S) valid = m - W <= i;
        else valid = i - sg[m - W - S].c >= 0;
        const float e = valid ? __expf(my_sc[m] - mx) : 0.f;
        my_sc[m] = e;
        l += e;
        edp += e * my_dp[m];
      }
      const float inv = 1.f / l;
      const float Dsum = edp * inv;
      for (int m = 0; m < n_slot; ++m) {
        const float p = my_sc[m] * inv;
        const float g = p * (my_dp[m] - Dsum);
        my_dp[m] = p;                       // dp -> p
        my_sc[m] = g;                       // sc -> g (dsigma)
      }
      for (int kk = 0; kk < n_off; ++kk) {
        const OffGeo g = sg[kk];
        if (i - g.lo - 1 >= 0)
          dal += (float)g.f * (my_sc[W + S + kk] * my_dt[kk] + my_dp[W + S + kk] * my_dpi[kk]);
      }
      for (int kk = 0; kk < n_off; ++kk) {  // fold near offsets into window weights
        if (!s_fold[kk]) continue;
        const OffGeo g = sg[kk];
        const float gg = my_sc[W + S + kk], pp = my_dp[W + S + kk];
        my_sc[g.lo] += g.wa * gg;  my_sc[g.lo + 1] += g.w * gg;
        my_dp[g.lo] += g.wa * pp;  my_dp[g.lo + 1] += g.w * pp;
      }
      // weights for the key side: G = [window W | far g_k], P likewise (bf16)
      for (int m = 0; m < W; ++m) {
        out[m] = __float2bfloat16_rn(my_sc[m]);
        out[a.gpart + m] = __float2bfloat16_rn(my_dp[m]);
      }
      for (int kk = 0; kk < n_off; ++kk) {
        const bool far = !s_fold[kk];
        out[W + kk] = __float2bfloat16_rn(far ? my_sc[W + S + kk] : 0.f);
        out[a.gpart + W + kk] = __float2bfloat16_rn(far ? my_dp[W + S + kk] : 0.f);
      }
    } else {
      for (int m = 0; m < n_slot; ++m) { my_sc[m] = 0.f; my_dp[m] = 0.f; }
    }
  }
  __syncthreads();

  // pass 3: dq_hat = sum_m g_m key_m (K ring again)
  {
    const int win_lo = max(0, i0 - W + 1), win_hi = min(T, i0 + M);
    const float* grp_sc = sc + (size_t)(4 * gid) * st;
    const float dqs = a.scale * kKeyUnstage;   // keys were staged times 1/256
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
      for (int h = 0; h < 16; ++h) x[qq][h] = 0.f;
    stage_rows<true>(ring, RB, K, a.rope, win_lo, win_hi);
    stage_sinks<true>(sinkb, S_rows, K, a.rope);
    __syncthreads();
#define SA_CALL(LC) window_axpy<LC, true>(ring, RB, ig, d0, c, grp_sc, st, x)
    SA_WINDOW_CHUNKS(W, SA_CALL)
#undef SA_CALL
    for (int s = 0; s < S; ++s) {
      float y[16];
      sink_load<true>(sinkb, s, c, y);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) axpy16(x[qq], grp_sc[qq * st + W + s], y);
    }
    int low = win_lo;
    int kb = next_far(s_fold, -1, n_off);
    while (kb < n_off) {
      const int hi = qseg_hi(sg[kb], i0, T);
      int last = kb, nx = next_far(s_fold, kb, n_off);
      while (nx < n_off && hi - qseg_lo(sg[nx], i0) <= RB) {
        last = nx;
        nx = next_far(s_fold, nx, n_off);
      }
      const int lo_row = qseg_lo(sg[last], i0);
      if (lo_row < low && lo_row < hi) {
        __syncthreads();
        stage_rows<true>(ring, RB, K, a.rope, lo_row, min(hi, low));
        low = lo_row;
        __syncthreads();
      }
      for (int kk = kb; kk < nx; kk = next_far(s_fold, kk, n_off)) {
        const OffGeo g = sg[kk];
        const int two = g.w != 0.f;
        float gq[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) gq[qq] = grp_sc[qq * st + W + S + kk];
#pragma unroll
        for (int u = 0; u < 5; ++u) {
          if (u == 0 && !two) continue;
          const int row = max(ig - g.lo - 1 + u, 0);
          float y[16];
          ring_load<true>(ring, row & (RB - 1), c, y);
          if (u <= 3 && two) axpy16(x[u], gq[u] * g.w, y);
          if (u >= 1) axpy16(x[u - 1], gq[u - 1] * g.wa, y);
        }
      }
      kb = nx;
    }
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      const int i = ig + qq;
      if (i < T) {
        const float4* cs = reinterpret_cast<const float4*>(a.rope + (size_t)i * 32 + 8 * c);
        float d1[8], d2[8];
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const float4 tt = __ldg(cs + h / 2);
          d1[h] = (x[qq][h] * tt.x + x[qq][h + 8] * tt.y) * dqs;
          d2[h] = (x[qq][h + 8] * tt.x - x[qq][h] * tt.y) * dqs;
          d1[h + 1] = (x[qq][h + 1] * tt.z + x[qq][h + 9] * tt.w) * dqs;
          d2[h + 1] = (x[qq][h + 9] * tt.z - x[qq][h + 1] * tt.w) * dqs;
        }
        uint4* dst = reinterpret_cast<uint4*>(a.dq + ub + (size_t)i * kD);
        dst[c] = pack8(d1);
        dst[c + 4] = pack8(d2);
      }
    }
  }

  // per-tile sink partials: sum over the tile's queries of g * q_hat and p * dO
  if (S > 0) {
    float* swarp = reinterpret_cast<float*>(smem);       // [warps][2][S][64], over the ring
    const float* grp_sc = sc + (size_t)(4 * gid) * st;
    const float* grp_dp = dpb + (size_t)(4 * gid) * st;
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      if (pass == 0) load_lane_rows<true>(Q, a.rope, ig, T, c, a.scale, x);
      else load_lane_rows<false>(dO, a.rope, ig, T, c, 1.f, x);
      const float* wsrc = pass == 0 ? grp_sc : grp_dp;
      for (int s = 0; s < S; ++s) {
        float acc[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) acc[h] = 0.f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) axpy16(acc, wsrc[qq * st + W + s], x[qq]);
#pragma unroll
        for (int h = 0; h < 16; ++h)
#pragma unroll
          for (int off = 4; off <= 16; off <<= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], off);
        if (lane < 4) {
          float* dst = swarp + (((size_t)warp * 2 + pass) * S + s) * kD;
#pragma unroll
          for (int h = 0; h < 8; ++h) { dst[8 * c + h] = acc[h]; dst[32 + 8 * c + h] = acc[h + 8]; }
        }
      }
    }
    __syncthreads();
    const size_t per = (size_t)S * kD;
    float* gk = a.sink_k + ((size_t)unit * a.n_tiles + tile) * per;
    float* gv = a.sink_v + ((size_t)unit * a.n_tiles + tile) * per;
    for (size_t e = t; e < per; e += M) {
      float ak = 0.f, av = 0.f;
      for (int w = 0; w < M / 32; ++w) {
        ak += swarp[((size_t)w * 2 + 0) * per + e];
        av += swarp[((size_t)w * 2 + 1) * per + e];
      }
      gk[e] = ak;
      gv[e] = av;
    }
  }

  // d-alpha partial of this tile: warp butterfly, then warps in order
#pragma unroll
  for (int off = 16; off >= 1; off >>= 1) dal += __shfl_xor_sync(0xffffffffu, dal, off);
  if (lane == 0) s_red[warp] = dal;
  __syncthreads();
  if (t == 0) {
    float acc = 0.f;
    for (int w = 0; w < M / 32; ++w) acc += s_red[w];
    a.dal_part[(size_t)unit * a.n_tiles + tile] = acc;
  }
}

// ---------------------------------------------------------------------------
// Key side.  Stage query rows [lo_row, hi_row) into the ring (rotated and
// scaled Q for dK, or dO for dV) and their weights (one half of the slot
// store: G or P) into wring as fp32; rows >= T are staged as zeros.
template <bool ROT>
__device__ __forceinline__ void stage_sources(const FastBwdArgs& a, uint4* ring, float* wring,
                                              const __nv_bfloat16* src, const __nv_bfloat16* wsrc,
                                              int lo_row, int hi_row) {
  const int RB = a.ring_rows, T = a.T, NW = a.W + a.n_off;
  const int n = (hi_row - lo_row) * 4;
  for (int task = threadIdx.x; task < n; task += blockDim.x) {
    const int row = lo_row + (task >> 2), p = task & 3;
    uint4 u0 = make_uint4(0, 0, 0, 0), u1 = u0;
    if (row < T) {
      const uint4* g = reinterpret_cast<const uint4*>(src + (size_t)row * kD);
      u0 = __ldg(g + p);
      u1 = __ldg(g + p + 4);
      if (ROT) {
        float x1[8], x2[8];
        unpack8(u0, x1);
        unpack8(u1, x2);
        const float4* cs = reinterpret_cast<const float4*>(a.rope + (size_t)row * 32 + 8 * p);
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const float4 t = __ldg(cs + h / 2);
          float a0 = x1[h], b0 = x2[h], a1 = x1[h + 1], b1 = x2[h + 1];
          x1[h] = (a0 * t.x - b0 * t.y) * a.scale;  x2[h] = (b0 * t.x + a0 * t.y) * a.scale;
          x1[h + 1] = (a1 * t.z - b1 * t.w) * a.scale;  x2[h + 1] = (b1 * t.z + a1 * t.w) * a.scale;
        }
        u0 = pack8(x1);
        u1 = pack8(x2);
      }
    }
    const int slot = row & (RB - 1), s = swz(slot);
    ring[slot * kChunks + (p ^ s)] = u0;
    ring[slot * kChunks + ((p + 4) ^ s)] = u1;
  }
  // weights: 8 lanes per row, one 16-byte chunk (8 bf16) per lane and step
  const int n_ch = (NW + 7) / 8;
  for (int row = lo_row + (int)(threadIdx.x >> 3); row < hi_row; row += blockDim.x >> 3) {
    float* dst = wring + (row & (RB - 1)) * a.wpitch;
    for (int ch = threadIdx.x & 7; ch < n_ch; ch += 8) {
      uint4 u = make_uint4(0, 0, 0, 0);
      if (row < T) u = __ldg(reinterpret_cast<const uint4*>(wsrc + (size_t)row * a.slot_pitch) + ch);
      float w8[8];
      unpack8(u, w8);
#pragma unroll
      for (int e = 0; e < 8; ++e)
        if (ch * 8 + e < NW) dst[ch * 8 + e] = w8[e];
    }
  }
}

template <bool ROT>
__device__ __forceinline__ void key_pass(const FastBwdArgs& a, uint4* ring, float* wring,
                                         const __nv_bfloat16* src, const __nv_bfloat16* wsrc,
                                         const OffGeo* sg, const int* s_fold, int r0, int rg, int c,
                                         float (&d)[4][16]) {
  constexpr int M = kFastM;
  const int W = a.W, RB = a.ring_rows, wp = a.wpitch;
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int h = 0; h < 16; ++h) d[kk][h] = 0.f;
  __syncthreads();
  int high = r0 + M + W - 1;
  stage_sources<ROT>(a, ring, wring, src, wsrc, r0, high);
  __syncthreads();
  // window: key rg+kk takes query row rg+d0+u at lead d0 + u - kk
  int d0 = 0;
  while (d0 < W) {
    const int LCr = W - d0 >= 8 ? 8 : (W - d0 >= 4 ? 4 : (W - d0 >= 2 ? 2 : 1));
#define SA_KEY_WINDOW(LC)                                                        \
    {                                                                            \
      _Pragma("unroll") for (int u = 0; u < LC + 3; ++u) {                       \
        const int slot = (rg + d0 + u) & (RB - 1);                                     \
        float y[16];                                                             \
        ring_load(ring, slot, c, y);                                             \
        _Pragma("unroll") for (int kk = 0; kk < 4; ++kk) {                       \
          const int l = u - kk;                                                  \
          if (l >= 0 && l < LC) axpy16(d[kk], wring[slot * wp + d0 + l], y);     \
        }                                                                        \
      }                                                                          \
    }
    if (LCr == 8) SA_KEY_WINDOW(8)
    else if (LCr == 4) SA_KEY_WINDOW(4)
    else if (LCr == 2) SA_KEY_WINDOW(2)
    else SA_KEY_WINDOW(1)
#undef SA_KEY_WINDOW
    d0 += LCr;
  }
  // far offsets: query rg+lo+u is row a of key rg+u and row b of key rg+u-1.
  // Member kk needs query rows [r0+lo, r0+M+lo+1); consecutive members whose
  // rows span at most RB rows are staged in one round.
  int kb = next_far(s_fold, -1, a.n_off);
  while (kb < a.n_off) {
    const int lo_first = r0 + sg[kb].lo;
    int last = kb, nx = next_far(s_fold, kb, a.n_off);
    while (nx < a.n_off && r0 + M + sg[nx].lo + 1 - lo_first <= RB) {
      last = nx;
      nx = next_far(s_fold, nx, a.n_off);
    }
    const int hi_last = r0 + M + sg[last].lo + 1;
    if (hi_last > high) {
      __syncthreads();
      stage_sources<ROT>(a, ring, wring, src, wsrc, max(lo_first, high), hi_last);
      high = hi_last;
      __syncthreads();
    }
    for (int kk = kb; kk < nx; kk = next_far(s_fold, kk, a.n_off)) {
      const OffGeo g = sg[kk];
#pragma unroll
      for (int u = 0; u < 5; ++u) {
        const int slot = (rg + g.lo + u) & (RB - 1);
        float y[16];
        ring_load(ring, slot, c, y);
        const float gk = wring[slot * wp + W + kk];
        if (u <= 3) axpy16(d[u], g.wa * gk, y);
        if (u >= 1) axpy16(d[u - 1], g.w * gk, y);
      }
    }
    kb = nx;
  }
}

__global__ void __launch_bounds__(kFastM) k_bwd_kv_fast(const FastBwdArgs a) {
  constexpr int M = kFastM;
  extern __shared__ __align__(16) unsigned char smem[];
  const int T = a.T, S = a.S, RB = a.ring_rows;
  uint4* ring = reinterpret_cast<uint4*>(smem);
  float* wring = reinterpret_cast<float*>(ring + (size_t)RB * kChunks);
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_fold[SA_MAX_OFFSETS];

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int r0 = tile * M;
  const int t = threadIdx.x, gid = t >> 2, c = t & 3;
  const int rg = r0 + 4 * gid;
  const size_t ub = (size_t)unit * T * kD;
  const __nv_bfloat16* slots = a.slots + (size_t)unit * T * a.slot_pitch;

  const int bad = cta_geometry_bwd(a, layer, sg, s_fold);
  if (bad) {
    const float qnan = __int_as_float(0x7fc00000);
    for (int e = t; e < M * kChunks; e += M) {
      const int r = r0 + e / kChunks;
      if (r < T) {
        float x[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) x[h] = qnan;
        reinterpret_cast<uint4*>(a.dk + ub + (size_t)r * kD)[e % kChunks] = pack8(x);
        reinterpret_cast<uint4*>(a.dv + ub + (size_t)r * kD)[e % kChunks] = pack8(x);
      }
    }
    return;
  }

  float d[4][16];
  for (int pass = 0; pass < 2; ++pass) {
    if (pass == 0)
      key_pass<true>(a, ring, wring, a.q + ub, slots, sg, s_fold, r0, rg, c, d);
    else
      key_pass<false>(a, ring, wring, a.dout + ub, slots + a.gpart, sg, s_fold, r0, rg, c, d);
    const float* sink = pass == 0 ? a.sink_k : a.sink_v;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int r = rg + kk;
      if (r < T && r < S) {
        const size_t per = (size_t)S * kD;
        const float* src = sink + (size_t)unit * a.n_tiles * per + (size_t)r * kD;
        for (int tt = 0; tt < a.n_tiles; ++tt) {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            d[kk][h] += src[tt * per + 8 * c + h];
            d[kk][h + 8] += src[tt * per + 32 + 8 * c + h];
          }
        }
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int r = rg + kk;
      if (r >= T) continue;
      float d1[8], d2[8];
      if (pass == 0) {
        const float4* cs = reinterpret_cast<const float4*>(a.rope + (size_t)r * 32 + 8 * c);
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const float4 tt = __ldg(cs + h / 2);
          d1[h] = d[kk][h] * tt.x + d[kk][h + 8] * tt.y;
          d2[h] = d[kk][h + 8] * tt.x - d[kk][h] * tt.y;
          d1[h + 1] = d[kk][h + 1] * tt.z + d[kk][h + 9] * tt.w;
          d2[h + 1] = d[kk][h + 9] * tt.z - d[kk][h + 1] * tt.w;
        }
      } else {
#pragma unroll
        for (int h = 0; h < 8; ++h) { d1[h] = d[kk][h]; d2[h] = d[kk][h + 8]; }
      }
      uint4* dst = reinterpret_cast<uint4*>((pass == 0 ? a.dk : a.dv) + ub + (size_t)r * kD);
      dst[c] = pack8(d1);
      dst[c + 4] = pack8(d2);
    }
  }
}

struct FastBwdLayout {
  int ring_rows, sc_stride, gpart, slot_pitch, wpitch, n_tiles;
  size_t q_smem, kv_smem;
  size_t slots_off, dal_off, sink_off, total;
};

FastBwdLayout fast_bwd_layout(const Problem& pb) {
  constexpr int M = kFastM;
  FastBwdLayout L;
  L.ring_rows = 32;   // a power of two: ring slots are row & (ring_rows - 1)
  while (L.ring_rows < std::max(M + pb.W - 1, M + 2)) L.ring_rows *= 2;
  const int n_slot = pb.W + pb.S + pb.n_off;
  L.sc_stride = n_slot | 1;
  const int NW = pb.W + pb.n_off;
  L.gpart = ((NW + 7) / 8) * 8;
  L.slot_pitch = 2 * L.gpart;
  L.wpitch = NW | 1;
  L.n_tiles = (pb.T + M - 1) / M;
  const size_t ring_bytes =
      std::max((size_t)L.ring_rows * 128, (size_t)(M / 32) * 2 * pb.S * kD * sizeof(float));
  L.q_smem = ring_bytes + (size_t)pb.S * 128 + 2 * (size_t)M * L.sc_stride * sizeof(float) +
             2 * (size_t)M * pb.n_off * sizeof(float);
  L.kv_smem = (size_t)L.ring_rows * 128 + (size_t)L.ring_rows * L.wpitch * sizeof(float);
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t units = (size_t)pb.units();
  L.slots_off = 0;
  L.dal_off = up(units * pb.T * L.slot_pitch * sizeof(__nv_bfloat16));
  L.sink_off = L.dal_off + up(units * L.n_tiles * sizeof(float));
  L.total = L.sink_off + up(2 * units * L.n_tiles * (size_t)pb.S * kD * sizeof(float));
  return L;
}

}  // namespace

bool fast_bwd_supported(const Problem& pb) {
  if (pb.dtype != SA_DTYPE_BF16 || pb.D != kD || pb.W > 256) return false;
  const FastBwdLayout L = fast_bwd_layout(pb);
  return L.q_smem <= 200 * 1024 && L.kv_smem <= 200 * 1024;
}

size_t fast_bwd_workspace(const Problem& pb) { return fast_bwd_layout(pb).total; }

cudaError_t launch_bwd_fast(const Problem& pb, const BwdPtrs& p, cudaStream_t st, int* launches) {
  const FastBwdLayout L = fast_bwd_layout(pb);
  FastBwdArgs a = {};
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = L.n_tiles;
  a.ring_rows = L.ring_rows; a.sc_stride = L.sc_stride; a.gpart = L.gpart;
  a.slot_pitch = L.slot_pitch; a.wpitch = L.wpitch;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  std::sort(a.f, a.f + pb.n_off);
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(p.k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(p.v);
  a.dout = reinterpret_cast<const __nv_bfloat16*>(p.dout);
  a.lse = p.lse; a.alpha = p.alpha; a.rope = p.rope;
  a.dq = reinterpret_cast<__nv_bfloat16*>(p.dq);
  a.dk = reinterpret_cast<__nv_bfloat16*>(p.dk);
  a.dv = reinterpret_cast<__nv_bfloat16*>(p.dv);
  char* ws = reinterpret_cast<char*>(p.workspace);
  a.slots = reinterpret_cast<__nv_bfloat16*>(ws + L.slots_off);
  a.dal_part = reinterpret_cast<float*>(ws + L.dal_off);
  a.sink_k = reinterpret_cast<float*>(ws + L.sink_off);
  a.sink_v = a.sink_k + (size_t)pb.units() * L.n_tiles * pb.S * kD;
  cudaError_t e;
  if ((e = cudaFuncSetAttribute(k_bwd_q_fast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)L.q_smem)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(k_bwd_kv_fast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)L.kv_smem)) != cudaSuccess)
    return e;
  const unsigned grid = (unsigned)((long long)pb.units() * L.n_tiles);
  trace_mark("bwd_q_fast", st, true);
  k_bwd_q_fast<<<grid, kFastM, L.q_smem, st>>>(a);
  trace_mark("bwd_q_fast", st, false);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  trace_mark("bwd_kv_fast", st, true);
  k_bwd_kv_fast<<<grid, kFastM, L.kv_smem, st>>>(a);
  trace_mark("bwd_kv_fast", st, false);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_reduce_dalpha(a.dal_part, pb.L, pb.B * pb.H * L.n_tiles, p.dalpha, st)) !=
      cudaSuccess)
    return e;
  *launches += 3;
  return cudaSuccess;
}

}  // namespace sa
