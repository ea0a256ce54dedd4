// Staged backward for bf16 inputs with head dim 64.  Same tiling, lane mapping
// and row ring (bulk-copy staging, sa_stage.cuh) as the staged forward
// (sa_fast.cu).  A RoPE pre-pass writes the rotated keys K^ = fp16(RoPE(K) /
// 256) and the rotated, scaled queries Q^ = fp16(RoPE(Q) * scale / 256).
//
// Query side (k_bwd_q_fast), one CTA per tile of 128 queries, three passes:
//   1. K^ ring: scores sigma_m = q_hat . key_m and, per offset, the row-score
//      difference dtau = q_hat . (K~[i-lo-1] - K~[i-lo]);
//   owner lane: p_m = softmax of its own scores;
//   2. V ring: dp_m = dO . value_m and dpi = dO . (V[i-lo-1] - V[i-lo]);
//      owner lane: D_i = sum_m p_m dp_m, g_m = p_m (dp_m - D_i), and the
//      d-alpha term sum_k f_k (g_k dtau_k + p_k dpi_k), the gradient through
//      w_k = alpha f_k - lo_k ("Implementation" lets gradients reach alpha
//      through the interpolation), accumulated as
//        sum_k f_k p_k (dp_k dtau_k + dpi_k)  -  D_i sum_k f_k p_k dtau_k
//      while pass 2 produces dp_k and dpi_k, so dpi is never stored;
//   3. K^ ring again: dq_hat = sum_m g_m key_m, dQ = scale * RoPE^T(dq_hat).
//   It also writes the weights the key side needs, indexed by KEY: for key j
//   and lag d < W the folded window weight of query j + d (G for dK, P for
//   dV), and per far offset k the row-a weight (1-w_k) g_k of query j + lo_k
//   and the row-b weight w_k g_k of query j + lo_k + 1; plus per-tile d-alpha
//   and sink-row partials.
// Key side (k_bwd_kv_fast), one CTA per tile of 128 keys, no atomics: the
//   source queries of a key tile are staged in increasing lead order (Q^ rows
//   for dK, dO rows for dV) together with the tile's weight block, and every
//   key accumulates its own dK~ / dV in registers:
//     window lead t : query r + t        (weight G[t] / P[t])
//     far offset k  : query r + lo       (row a)
//                     query r + lo + 1   (row b)
//   then dK = RoPE^T(dK~).  Sink rows add the query side's per-tile partials.
#include <algorithm>

#include "sa_stage.cuh"

namespace sa {

namespace {

using namespace fast;
using namespace stage;

struct FastBwdArgs {
  int B, H, T, W, n_off, S, n_tiles;
  int ring_rows, sc_stride, NS;          // NS = W + 2 n_off weight slots per key
  float scale;
  int f[SA_MAX_OFFSETS];                 // ascending
  const __nv_bfloat16* q; const __nv_bfloat16* v; const __nv_bfloat16* dout;
  const void* khat; const void* qhat;    // fp16 rotated keys / rotated scaled queries
  const float* alpha; const float2* rope;
  __nv_bfloat16* dq; __nv_bfloat16* dk; __nv_bfloat16* dv;
  __nv_bfloat16* gblk; __nv_bfloat16* pblk;   // [units][n_tiles][NS][M], key-indexed
  float* dal_part;                       // [units][n_tiles]
  float* sink_k; float* sink_v;          // [units][n_tiles][S][64]
  unsigned* err;
  long long wait_limit;                // bounded waits: SM clocks (0: the default)
  int stall;                           // failure-path test: the first staging round waits in vain
  const float* ctx_p;                    // training context: [units][W+S+n_off][T] probabilities
  const float* ctx_dt;                   // ... and [units][n_off][T] row-score differences
  const float* beta;                     // log-prior on offset members [units][T], or nullptr
  float* dbeta;                          // its gradient [units][T], or nullptr
};

enum : int { kFar = 0, kNear = 1, kDead = 2 };

// Both rows of an offset stay inside the window: the backward folds it (its
// d-alpha term needs both rows even when w == 0).
__device__ __forceinline__ int near_bwd(const OffGeo& g, int W) { return g.ok && g.lo + 1 <= W - 1; }

// Next offset after k of kind kFar (n_off when none).
__device__ __forceinline__ int next_far(const int* s_kind, int k, int n_off) {
  ++k;
  while (k < n_off && s_kind[k] != kFar) ++k;
  return k;
}

// Load this lane's 16 dims of 4 consecutive rows of X (bf16 [T][64]), rows
// clamped to T-1, in the lane's half order (first half = chunk c + 4 par);
// optionally rotated (RoPE at the row's position); times `scale`.
template <bool ROT>
__device__ __forceinline__ void load_lane_rows(const __nv_bfloat16* X, const float2* rope, int r0,
                                               int T, int c, int par, float scale,
                                               float (&x)[4][16]) {
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
        const float a0 = x1[h], b0 = x2[h], a1 = x1[h + 1], b1 = x2[h + 1];
        x1[h] = a0 * t.x - b0 * t.y;  x2[h] = b0 * t.x + a0 * t.y;
        x1[h + 1] = a1 * t.z - b1 * t.w;  x2[h + 1] = b1 * t.z + a1 * t.w;
      }
    }
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      x[qq][h] = (par ? x2[h] : x1[h]) * scale;
      x[qq][h + 8] = (par ? x1[h] : x2[h]) * scale;
    }
  }
}

// Window dot products for lags [d0, d0+LC) (rows ig+3-d0-u, walked upward
// from the lowest); results land in out_row[d0 .. d0+LC).
template <int LC, bool F16>
__device__ __forceinline__ void window_dots(const unsigned char* ring, int RB, int ig, int d0,
                                            int off0, int d1, int c, const float (&q)[4][16],
                                            float* out_row, int i_own, float* mx) {
  float acc[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) acc[a][l] = 0.f;
  const unsigned char* p = ring + (size_t)((ig + 1 - d0 - LC) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    float x[16];
    lane_row<F16>(p + (LC + 2 - u) * kRowBytes, d1, x);
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
__device__ __forceinline__ void window_axpy(const unsigned char* ring, int RB, int ig, int d0,
                                            int off0, int d1, const float* wrow0, int stride,
                                            float (&o)[4][16]) {
  float pw[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) pw[a][l] = wrow0[a * stride + d0 + l];
  const unsigned char* p = ring + (size_t)((ig + 1 - d0 - LC) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    float x[16];
    lane_row<F16>(p + (LC + 2 - u) * kRowBytes, d1, x);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int l = a + u - 3;
      if (l >= 0 && l < LC) axpy16(o[a], pw[a][l], x);
    }
  }
}

// Window lags in blocks of 4: the unrolled body stays small enough for the
// instruction cache (measured on B200: 8-lag blocks ran 5-14% slower).
#define SA_WINDOW_CHUNKS(W, CALL)                                   \
  {                                                                 \
    int d0 = 0;                                                     \
    while ((W) - d0 >= 4) { CALL(4); d0 += 4; }                     \
    if ((W) - d0 >= 2) { CALL(2); d0 += 2; }                        \
    if ((W) - d0 >= 1) { CALL(1); d0 += 1; }                        \
  }

// One pass of dot products of the lane's 4 rows `x` with every member
// (window, sinks, far offsets) of the 16-bit array `src` (F16: rotated keys;
// else V): member value into val_row; for far offsets the row difference
// (row b minus row a) goes to diff_row[k] (the key pass), or, with p_row set
// (the value pass), into this query's d-alpha sum
//   *dal_u += f_k p_k (dp_k dtau_k + dpi_k)      (diff_row then holds dtau).
// Returns nonzero when a staging wait gave up.
template <bool F16>
__device__ __forceinline__ int member_dots(const FastBwdArgs& a, Stager& stg,
                                           unsigned char* ring, unsigned char* sinkb,
                                           const unsigned char* src, const OffGeo* sg,
                                           const int* s_kind, int i0, int ig, int c, int off0,
                                           int d1, const float (&x)[4][16], float* val_row,
                                           float* diff_row, int i_own, float* mx,
                                           const float* p_row, float* dal_u, float bias) {
  constexpr int M = kFastM;
  const int T = a.T, W = a.W, S = a.S, RB = a.ring_rows;
  const int win_lo = i0 - W + 1, win_hi = i0 + M;
  __syncthreads();
  stage_ring(stg, ring, RB, src, T, win_lo, win_hi);
  stage_plain(stg, sinkb, src, min(S, T), S);
  if (stage_commit_wait(stg)) { stage_drain(stg); return 1; }
  dbg_rows(stg, ig - W + 1, ig + 4);
#define SA_CALL(LC) window_dots<LC, F16>(ring, RB, ig, d0, off0, d1, c, x, val_row, i_own, mx)
  SA_WINDOW_CHUNKS(W, SA_CALL)
#undef SA_CALL
  for (int s0 = 0; s0 < S; s0 += 4) {
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float y[16];
      lane_row<F16>(sinkb + (size_t)min(s0 + j, S - 1) * kRowBytes + off0, d1, y);
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
  // far offsets, staged in batches whose rows span at most RB rows; a member
  // reads rows [i0 - lo - 1, i0 + M - lo)
  int low = win_lo;
  int kb = next_far(s_kind, -1, a.n_off);
  while (kb < a.n_off) {
    const int hi = i0 + M - sg[kb].lo;
    int last = kb, nx = next_far(s_kind, kb, a.n_off);
    while (nx < a.n_off && hi - (i0 - sg[nx].lo - 1) <= RB) {
      last = nx;
      nx = next_far(s_kind, nx, a.n_off);
    }
    const int lo_row = i0 - sg[last].lo - 1;
    if (lo_row < low) {
      __syncthreads();
      stage_ring(stg, ring, RB, src, T, lo_row, min(hi, low));
      if (stage_commit_wait(stg)) { stage_drain(stg); return 1; }
      low = lo_row;
    }
    for (int kk = kb; kk < nx; kk = next_far(s_kind, kk, a.n_off)) {
      const OffGeo g = sg[kk];
      dbg_rows(stg, ig - g.lo - 1, ig - g.lo + 4);
      const unsigned char* p = ring + (size_t)((ig - g.lo - 1) & (RB - 1)) * kRowBytes + off0;
      float pa[4], pb[4];
#pragma unroll
      for (int u = 0; u < 5; ++u) {
        float y[16];
        lane_row<F16>(p + u * kRowBytes, d1, y);
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
      out[0] += bias;
      val_row[W + S + kk] = out[0];
      if (p_row) {
        if (i_own - g.lo - 1 >= 0)
          *dal_u += (float)g.f * p_row[W + S + kk] * (out[0] * diff_row[kk] + out[1]);
      } else {
        diff_row[kk] = out[1];
      }
      if (mx && i_own - g.c >= 0) *mx = fmaxf(*mx, out[0]);
    }
    kb = nx;
  }
  return 0;
}

// CTX: the probabilities and row-score differences come from the training
// context the saving forward wrote; the score pass is skipped.
template <bool CTX>
__global__ void __launch_bounds__(kFastM) k_bwd_q_fast(const FastBwdArgs a) {
  constexpr int M = kFastM;
  extern __shared__ __align__(128) unsigned char smem[];
  const int T = a.T, W = a.W, S = a.S, n_off = a.n_off, RB = a.ring_rows;
  const int st = a.sc_stride;
  unsigned char* ring = smem;
  const size_t ring_a = (size_t)(RB + kMirror) * kRowBytes;
  const size_t ring_b = (size_t)(M / 32) * 2 * S * kD * sizeof(float);
  const size_t ring_bytes = ring_a > ring_b ? ring_a : ring_b;
  unsigned char* sinkb = smem + ring_bytes;
  float* sc = reinterpret_cast<float*>(sinkb + (size_t)S * kRowBytes);   // sigma, then g
  float* dpb = sc + (size_t)M * st;                                  // dp, then p
  float* dts = dpb + (size_t)M * st;                                 // [M][n_off] dtau
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_kind[SA_MAX_OFFSETS];
  __shared__ float s_red[M / 32];
  __shared__ uint64_t bar;

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int i0 = tile * M;
  const int t = threadIdx.x, gid = t >> 2, c = t & 3, lane = t & 31, warp = t >> 5;
  const int par = gid & 1;
  const int ig = i0 + 4 * gid;
  const size_t ub = (size_t)unit * T * kD;
  const __nv_bfloat16* Q = a.q + ub;
  const __nv_bfloat16* dO = a.dout + ub;
  const unsigned char* Kh = reinterpret_cast<const unsigned char*>(a.khat) + ub * 2;
  const unsigned char* Vb = reinterpret_cast<const unsigned char*>(a.v + ub);
  const float qnan = __int_as_float(0x7fc00000);

  if (t == 0) { mbar_init(&bar, 1); fence_barrier_init(); }
  int bad = 0;
  if (t < n_off) {
    const OffGeo g = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    sg[t] = g;
    bad = !g.ok;
    const int dead = i0 + M - 1 - g.c < 0;        // no query of the tile has it yet
    s_kind[t] = near_bwd(g, W) ? kNear : (dead ? kDead : kFar);
  }
  bad = __syncthreads_or(bad);
  if (bad) {  // NaN dQ and d-alpha partial; the key side writes NaN dK, dV
    for (int e = t; e < M * kChunks; e += M) {
      const int i = i0 + e / kChunks;
      if (i < T) {
        float x[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) x[h] = qnan;
        reinterpret_cast<uint4*>(a.dq + ub + (size_t)i * kD)[e % kChunks] = pack8(x);
        if (e % kChunks == 0 && a.dbeta) a.dbeta[(size_t)unit * T + i] = qnan;
      }
    }
    if (t == 0) a.dal_part[(size_t)unit * a.n_tiles + tile] = qnan;
    return;
  }
  Stager stg = make_stager(&bar, a.err, a.wait_limit, a.stall);
  const int off0 = half0_off(c, par), d1 = half1_off(c, par) - off0;
  const int lr = 4 * gid + c;
  float* my_sc = sc + (size_t)lr * st;
  float* my_dp = dpb + (size_t)lr * st;
  float* my_dt = dts + (size_t)lr * n_off;

  float x[4][16];
  const int i = ig + c;
  const int n_slot = W + S + n_off;
  // this lane's query's log-prior on the offset members (0 without one)
  const float prior = (!CTX && a.beta && i < T) ? __ldg(a.beta + (size_t)unit * T + i) : 0.f;
  float dal_v = 0.f, dal_u = 0.f;
  if (CTX) {
    // probabilities and row-score differences from the training context:
    // every element an asynchronous 4-byte copy into this lane's rows, one wait
    if (i < T) {
      const float* cp = a.ctx_p + (size_t)unit * n_slot * T + i;
      const float* cd = a.ctx_dt + (size_t)unit * n_off * T + i;
      for (int m = 0; m < n_slot; ++m) cp_async4(my_sc + m, cp + (size_t)m * T);
      for (int kk = 0; kk < n_off; ++kk) cp_async4(my_dt + kk, cd + (size_t)kk * T);
      cp_async_wait_all();
    } else {
      for (int m = 0; m < n_slot; ++m) my_sc[m] = 0.f;
    }
  } else {
    // pass 1: scores and row-score differences (rotated keys)
    load_lane_rows<true>(Q, a.rope, ig, T, c, par, a.scale * kKeyUnstage, x);
    float mx = -INFINITY;   // running max of this lane's query's valid scores
    if (member_dots<true>(a, stg, ring, sinkb, Kh, sg, s_kind, i0, ig, c, off0, d1, x, my_sc,
                          my_dt, ig + c, &mx, nullptr, nullptr, prior))
      return;
    // owner lane: probabilities from these scores (not the forward's LSE, so
    // that sum_m p_m = 1 and sum_m g_m = 0 hold for the values used here)
    if (i < T) {
      for (int kk = 0; kk < n_off; ++kk) {
        if (s_kind[kk] != kNear) continue;
        const OffGeo g = sg[kk];
        my_sc[W + S + kk] = g.wa * my_sc[g.lo] + g.w * my_sc[g.lo + 1] + prior;
        my_dt[kk] = my_sc[g.lo + 1] - my_sc[g.lo];
        if (i - g.c >= 0) mx = fmaxf(mx, my_sc[W + S + kk]);
      }
      float l = 0.f;
      for (int m = 0; m < n_slot; ++m) {
        bool valid;
        if (m < W) valid = i - m >= 0;
        else if (m < W + S) valid = m - W <= i;
        else valid = s_kind[m - W - S] != kDead && i - sg[m - W - S].c >= 0;
        const float e = valid ? __expf(my_sc[m] - mx) : 0.f;
        my_sc[m] = e;
        l += e;
      }
      const float inv = 1.f / l;
      for (int m = 0; m < n_slot; ++m) my_sc[m] *= inv;          // scores -> p
    } else {
      for (int m = 0; m < n_slot; ++m) my_sc[m] = 0.f;
    }
  }
  // the first d-alpha sum  dal_v = sum_k f_k p_k dtau_k
  if (i < T) {
    for (int kk = 0; kk < n_off; ++kk) {
      const OffGeo g = sg[kk];
      if (s_kind[kk] != kDead && i - g.lo - 1 >= 0)
        dal_v += (float)g.f * my_sc[W + S + kk] * my_dt[kk];
    }
  }

  // pass 2: dO . values; far offsets add f_k p_k (dp_k dtau_k + dpi_k) to dal_u
  load_lane_rows<false>(dO, a.rope, ig, T, c, par, 1.f, x);
  if (member_dots<false>(a, stg, ring, sinkb, Vb, sg, s_kind, i0, ig, c, off0, d1, x, my_dp,
                         my_dt, ig + c, nullptr, my_sc, &dal_u, 0.f))
    return;
  __syncthreads();

  // owner lane: D_i, dsigma, d-alpha = dal_u - D_i dal_v, folded window weights
  float dal = 0.f;
  {
    if (i < T) {
      for (int kk = 0; kk < n_off; ++kk) {    // near offsets from two window values
        if (s_kind[kk] != kNear) continue;
        const OffGeo g = sg[kk];
        const float dpk = g.wa * my_dp[g.lo] + g.w * my_dp[g.lo + 1];
        const float dpi = my_dp[g.lo + 1] - my_dp[g.lo];
        my_dp[W + S + kk] = dpk;
        if (i - g.lo - 1 >= 0)
          dal_u += (float)g.f * my_sc[W + S + kk] * (dpk * my_dt[kk] + dpi);
      }
      float Dsum = 0.f;
      for (int m = 0; m < n_slot; ++m) Dsum += my_sc[m] != 0.f ? my_sc[m] * my_dp[m] : 0.f;
      for (int m = 0; m < n_slot; ++m) {
        const float p = my_sc[m];
        const float g = p * (my_dp[m] - Dsum);
        my_dp[m] = p;                       // dp -> p
        my_sc[m] = p != 0.f ? g : 0.f;      // p -> g (dsigma)
      }
      dal = dal_u - Dsum * dal_v;
      if (a.dbeta) {                        // d log-prior: the offset members' g, summed
        float db = 0.f;
        for (int kk = 0; kk < n_off; ++kk) db += my_sc[W + S + kk];
        a.dbeta[(size_t)unit * T + i] = db;
      }
      for (int kk = 0; kk < n_off; ++kk) {  // fold near offsets into window weights
        if (s_kind[kk] != kNear) continue;
        const OffGeo g = sg[kk];
        const float gg = my_sc[W + S + kk], pp = my_dp[W + S + kk];
        my_sc[g.lo] += g.wa * gg;  my_sc[g.lo + 1] += g.w * gg;
        my_dp[g.lo] += g.wa * pp;  my_dp[g.lo + 1] += g.w * pp;
      }
      // key-indexed weights: entry (key j, slot) of key tile j / M at
      // [slot][j % M]; window slot d from query j + d, far slots from queries
      // j + lo (row a) and j + lo + 1 (row b)
      const size_t tile_base = (size_t)unit * a.n_tiles;
      const size_t blk = (size_t)a.NS * M;
      const size_t blk_end = (size_t)gridDim.x * blk;   // weight entries of the launch
      for (int d = 0; d < W; ++d) {
        const int j = i - d;
        if (j < 0) break;
        const size_t off = (tile_base + j / M) * blk + (size_t)d * M + (j % M);
        dbg_check(a.err, off < blk_end);
        a.gblk[off] = __float2bfloat16_rn(my_sc[d]);
        a.pblk[off] = __float2bfloat16_rn(my_dp[d]);
      }
      for (int kk = 0; kk < n_off; ++kk) {
        if (s_kind[kk] == kNear) continue;
        const OffGeo g = sg[kk];
        const float gg = my_sc[W + S + kk], pp = my_dp[W + S + kk];
        const int ja = i - g.lo, jb = i - g.lo - 1;
        if (ja >= 0) {
          const size_t off = (tile_base + ja / M) * blk + (size_t)(W + kk) * M + (ja % M);
          dbg_check(a.err, off < blk_end);
          a.gblk[off] = __float2bfloat16_rn(g.wa * gg);
          a.pblk[off] = __float2bfloat16_rn(g.wa * pp);
        }
        if (jb >= 0) {
          const size_t off = (tile_base + jb / M) * blk + (size_t)(W + n_off + kk) * M + (jb % M);
          dbg_check(a.err, off < blk_end);
          a.gblk[off] = __float2bfloat16_rn(g.w * gg);
          a.pblk[off] = __float2bfloat16_rn(g.w * pp);
        }
      }
    } else {
      for (int m = 0; m < n_slot; ++m) { my_sc[m] = 0.f; my_dp[m] = 0.f; }
    }
    // zero the weight entries of this tile's keys that no query writes
    // (source query at or beyond T; near-offset slots are never read): per
    // slot the keys [max(i0, T - lag), min(i0 + M, T)), one warp per slot
    {
      const size_t base = ((size_t)unit * a.n_tiles + tile) * (size_t)a.NS * M;
      const __nv_bfloat16 zero = __float2bfloat16_rn(0.f);
      for (int slot = warp; slot < a.NS; slot += M / 32) {
        int lag;
        if (slot < W) lag = slot;
        else if (slot < W + n_off) lag = sg[slot - W].lo;
        else lag = sg[slot - W - n_off].lo + 1;
        const int jhi = min(i0 + M, T);
        for (int j = max(i0, T - lag) + lane; j < jhi; j += 32) {
          a.gblk[base + (size_t)slot * M + (j - i0)] = zero;
          a.pblk[base + (size_t)slot * M + (j - i0)] = zero;
        }
      }
    }
  }
  __syncthreads();

  // pass 3: dq_hat = sum_m g_m key_m (rotated keys again)
  {
    const int win_lo = i0 - W + 1, win_hi = i0 + M;
    const float* grp_sc = sc + (size_t)(4 * gid) * st;
    const float dqs = a.scale * kKeyUnstage;   // keys were staged times 1/256
#pragma unroll
    for (int qq = 0; qq < 4; ++qq)
#pragma unroll
      for (int h = 0; h < 16; ++h) x[qq][h] = 0.f;
    stage_ring(stg, ring, RB, Kh, T, win_lo, win_hi);
    stage_plain(stg, sinkb, Kh, min(S, T), S);
    if (stage_commit_wait(stg)) { stage_drain(stg); return; }
    dbg_rows(stg, ig - W + 1, ig + 4);
#define SA_CALL(LC) window_axpy<LC, true>(ring, RB, ig, d0, off0, d1, grp_sc, st, x)
    SA_WINDOW_CHUNKS(W, SA_CALL)
#undef SA_CALL
    for (int s = 0; s < S; ++s) {
      float y[16];
      lane_row<true>(sinkb + (size_t)s * kRowBytes + off0, d1, y);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) axpy16(x[qq], grp_sc[qq * st + W + s], y);
    }
    int low = win_lo;
    int kb = next_far(s_kind, -1, n_off);
    while (kb < n_off) {
      const int hi = i0 + M - sg[kb].lo;
      int last = kb, nx = next_far(s_kind, kb, n_off);
      while (nx < n_off && hi - (i0 - sg[nx].lo - 1) <= RB) {
        last = nx;
        nx = next_far(s_kind, nx, n_off);
      }
      const int lo_row = i0 - sg[last].lo - 1;
      if (lo_row < low) {
        __syncthreads();
        stage_ring(stg, ring, RB, Kh, T, lo_row, min(hi, low));
        if (stage_commit_wait(stg)) { stage_drain(stg); return; }
        low = lo_row;
      }
      for (int kk = kb; kk < nx; kk = next_far(s_kind, kk, n_off)) {
        const OffGeo g = sg[kk];
        const int two = g.w != 0.f;
        float gq[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) gq[qq] = grp_sc[qq * st + W + S + kk];
        dbg_rows(stg, ig - g.lo - 1 + (two ? 0 : 1), ig - g.lo + 4);
        const unsigned char* p = ring + (size_t)((ig - g.lo - 1) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
        for (int u = 0; u < 5; ++u) {
          if (u == 0 && !two) continue;
          float y[16];
          lane_row<true>(p + u * kRowBytes, d1, y);
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
        float o1[8], o2[8];      // chunk c (dims 8c..) and chunk c + 4
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const float4 tt = __ldg(cs + h / 2);
          const float l0 = par ? x[qq][h + 8] : x[qq][h], hv0 = par ? x[qq][h] : x[qq][h + 8];
          const float l1 = par ? x[qq][h + 9] : x[qq][h + 1], hv1 = par ? x[qq][h + 1] : x[qq][h + 9];
          o1[h] = (l0 * tt.x + hv0 * tt.y) * dqs;
          o2[h] = (hv0 * tt.x - l0 * tt.y) * dqs;
          o1[h + 1] = (l1 * tt.z + hv1 * tt.w) * dqs;
          o2[h + 1] = (hv1 * tt.z - l1 * tt.w) * dqs;
        }
        uint4* dst = reinterpret_cast<uint4*>(a.dq + ub + (size_t)i * kD);
        dst[c] = pack8(o1);
        dst[c + 4] = pack8(o2);
      }
    }
  }

  // per-tile sink partials: sum over the tile's queries of g * q_hat and p * dO,
  // stored in natural dim order
  if (S > 0) {
    float* swarp = reinterpret_cast<float*>(smem);       // [warps][2][S][64], over the ring
    const float* grp_sc = sc + (size_t)(4 * gid) * st;
    const float* grp_dp = dpb + (size_t)(4 * gid) * st;
    const int h0 = c + 4 * par, h1 = c + 4 - 4 * par;
    __syncthreads();
    for (int pass = 0; pass < 2; ++pass) {
      if (pass == 0) load_lane_rows<true>(Q, a.rope, ig, T, c, par, a.scale, x);
      else load_lane_rows<false>(dO, a.rope, ig, T, c, par, 1.f, x);
      const float* wsrc = pass == 0 ? grp_sc : grp_dp;
      for (int s = 0; s < S; ++s) {
        float acc[16];
#pragma unroll
        for (int h = 0; h < 16; ++h) acc[h] = 0.f;
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) axpy16(acc, wsrc[qq * st + W + s], x[qq]);
        // sum over the warp's groups of the same parity (same half order)
#pragma unroll
        for (int h = 0; h < 16; ++h)
#pragma unroll
          for (int off = 8; off <= 16; off <<= 1) acc[h] += __shfl_xor_sync(0xffffffffu, acc[h], off);
        float* dst = swarp + (((size_t)warp * 2 + pass) * S + s) * kD;
        if (lane < 4) {         // group 0 (even): first half is chunk c
#pragma unroll
          for (int h = 0; h < 8; ++h) { dst[8 * h0 + h] = acc[h]; dst[8 * h1 + h] = acc[h + 8]; }
        }
        __syncwarp();
        if (lane >= 4 && lane < 8) {   // group 1 (odd): first half is chunk c + 4
#pragma unroll
          for (int h = 0; h < 8; ++h) { dst[8 * h0 + h] += acc[h]; dst[8 * h1 + h] += acc[h + 8]; }
        }
        __syncwarp();
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
// Key side.  One pass accumulates d[kk] = sum over source rows of weight *
// row for the lane's 4 keys rg + kk, from the rows of `src` (F16: rotated
// scaled queries; else dO) and the tile's weight block `wsrc` ([NS][M] bf16).
// Returns nonzero when a staging wait gave up.
template <bool F16>
__device__ __forceinline__ int key_pass(const FastBwdArgs& a, Stager& stg, unsigned char* ring,
                                        unsigned char* wblk, const unsigned char* src,
                                        const __nv_bfloat16* wsrc, const OffGeo* sg,
                                        const int* s_kind, int r0, int rg, int gid, int off0,
                                        int d1, float (&d)[4][16]) {
  constexpr int M = kFastM;
  const int W = a.W, RB = a.ring_rows, T = a.T, n_off = a.n_off;
  const __nv_bfloat16* wb = reinterpret_cast<const __nv_bfloat16*>(wblk);
#pragma unroll
  for (int kk = 0; kk < 4; ++kk)
#pragma unroll
    for (int h = 0; h < 16; ++h) d[kk][h] = 0.f;
  __syncthreads();
  int high = r0 + M + W - 1;
  stage_ring(stg, ring, RB, src, T, r0, high);
  stage_plain(stg, wblk, wsrc, 2 * a.NS, 2 * a.NS);     // NS * M bf16 = 2 NS rows of 128 B
  if (stage_commit_wait(stg)) { stage_drain(stg); return 1; }
  dbg_rows(stg, rg, rg + W + 3);
  // window: key rg+kk takes query row rg+d0+u at lag d0 + u - kk
  int d0 = 0;
  while (d0 < W) {
    const int LCr = W - d0 >= 4 ? 4 : (W - d0 >= 2 ? 2 : 1);
#define SA_KEY_WINDOW(LC)                                                           \
    {                                                                               \
      float wl[LC][4];                                                              \
      _Pragma("unroll") for (int l = 0; l < LC; ++l) {                              \
        const uint2 u2 = *reinterpret_cast<const uint2*>(wb + (size_t)(d0 + l) * M + 4 * gid); \
        wl[l][0] = bf16lo(u2.x); wl[l][1] = bf16hi(u2.x);                           \
        wl[l][2] = bf16lo(u2.y); wl[l][3] = bf16hi(u2.y);                           \
      }                                                                             \
      const unsigned char* p = ring + (size_t)((rg + d0) & (RB - 1)) * kRowBytes + off0; \
      _Pragma("unroll") for (int u = 0; u < LC + 3; ++u) {                          \
        float y[16];                                                                \
        lane_row<F16>(p + u * kRowBytes, d1, y);                                    \
        _Pragma("unroll") for (int kk = 0; kk < 4; ++kk) {                          \
          const int l = u - kk;                                                     \
          if (l >= 0 && l < LC) axpy16(d[kk], wl[l][kk], y);                        \
        }                                                                           \
      }                                                                             \
    }
    if (LCr == 4) SA_KEY_WINDOW(4)
    else if (LCr == 2) SA_KEY_WINDOW(2)
    else SA_KEY_WINDOW(1)
#undef SA_KEY_WINDOW
    d0 += LCr;
  }
  // far offsets: query rg+lo+u is row a of key rg+u and row b of key rg+u-1.
  // Member kk needs query rows [r0+lo, r0+M+lo+1); consecutive members whose
  // rows span at most RB rows are staged in one round.
  int kb = next_far(s_kind, -1, n_off);
  while (kb < n_off) {
    const int lo_first = r0 + sg[kb].lo;
    int last = kb, nx = next_far(s_kind, kb, n_off);
    while (nx < n_off && r0 + M + sg[nx].lo + 1 - lo_first <= RB) {
      last = nx;
      nx = next_far(s_kind, nx, n_off);
    }
    const int hi_last = r0 + M + sg[last].lo + 1;
    if (hi_last > high) {
      __syncthreads();
      stage_ring(stg, ring, RB, src, T, max(lo_first, high), hi_last);
      if (stage_commit_wait(stg)) { stage_drain(stg); return 1; }
      high = hi_last;
    }
    for (int kk = kb; kk < nx; kk = next_far(s_kind, kk, n_off)) {
      const OffGeo g = sg[kk];
      const int two = g.w != 0.f;
      float fa[4], fb[4];
      {
        const uint2 ua = *reinterpret_cast<const uint2*>(wb + (size_t)(W + kk) * M + 4 * gid);
        const uint2 uv = *reinterpret_cast<const uint2*>(wb + (size_t)(W + n_off + kk) * M + 4 * gid);
        fa[0] = bf16lo(ua.x); fa[1] = bf16hi(ua.x); fa[2] = bf16lo(ua.y); fa[3] = bf16hi(ua.y);
        fb[0] = bf16lo(uv.x); fb[1] = bf16hi(uv.x); fb[2] = bf16lo(uv.y); fb[3] = bf16hi(uv.y);
      }
      dbg_rows(stg, rg + g.lo, rg + g.lo + (two ? 5 : 4));
      const unsigned char* p = ring + (size_t)((rg + g.lo) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
      for (int u = 0; u < 5; ++u) {
        if (u == 4 && !two) continue;
        float y[16];
        lane_row<F16>(p + u * kRowBytes, d1, y);
        if (u <= 3) axpy16(d[u], fa[u], y);
        if (u >= 1 && two) axpy16(d[u - 1], fb[u - 1], y);
      }
    }
    kb = nx;
  }
  return 0;
}

__global__ void __launch_bounds__(kFastM, 4) k_bwd_kv_fast(const FastBwdArgs a) {
  constexpr int M = kFastM;
  extern __shared__ __align__(128) unsigned char smem[];
  const int T = a.T, S = a.S, RB = a.ring_rows, n_off = a.n_off;
  unsigned char* ring = smem;
  unsigned char* wblk = smem + (size_t)(RB + kMirror) * kRowBytes;
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_kind[SA_MAX_OFFSETS];
  __shared__ uint64_t bar;

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int r0 = tile * M;
  const int t = threadIdx.x, gid = t >> 2, c = t & 3, par = gid & 1;
  const int rg = r0 + 4 * gid;
  const size_t ub = (size_t)unit * T * kD;

  if (t == 0) { mbar_init(&bar, 1); fence_barrier_init(); }
  int bad = 0;
  if (t < n_off) {
    const OffGeo g = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    sg[t] = g;
    bad = !g.ok;
    const int dead = r0 + g.lo >= T;             // every source query is beyond T
    s_kind[t] = near_bwd(g, a.W) ? kNear : (dead ? kDead : kFar);
  }
  bad = __syncthreads_or(bad);
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
  (void)n_off;
  Stager stg = make_stager(&bar, a.err, a.wait_limit, a.stall);
  const int off0 = half0_off(c, par), d1 = half1_off(c, par) - off0;
  const int h0 = c + 4 * par, h1 = c + 4 - 4 * par;
  const size_t blk = ((size_t)unit * a.n_tiles + tile) * (size_t)a.NS * M;

  float d[4][16];
  for (int pass = 0; pass < 2; ++pass) {
    const int stop =
        pass == 0
            ? key_pass<true>(a, stg, ring, wblk,
                             reinterpret_cast<const unsigned char*>(a.qhat) + ub * 2, a.gblk + blk,
                             sg, s_kind, r0, rg, gid, off0, d1, d)
            : key_pass<false>(a, stg, ring, wblk,
                              reinterpret_cast<const unsigned char*>(a.dout + ub), a.pblk + blk,
                              sg, s_kind, r0, rg, gid, off0, d1, d);
    if (stop) return;
    const float* sink = pass == 0 ? a.sink_k : a.sink_v;
    // Q^ was staged times 1/256: dK~ is rescaled by 256 here, before the sink
    // partials (which carry the true scale, in natural dim order) are added
    const float dks = pass == 0 ? kKeyUnstage : 1.f;
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int r = rg + kk;
#pragma unroll
      for (int h = 0; h < 16; ++h) d[kk][h] *= dks;
      if (r < T && r < S) {
        const size_t per = (size_t)S * kD;
        const float* src = sink + (size_t)unit * a.n_tiles * per + (size_t)r * kD;
        // two tiles' loads in flight (the sum stays in tile order)
#pragma unroll 2
        for (int tt = 0; tt < a.n_tiles; ++tt) {
#pragma unroll
          for (int h = 0; h < 8; ++h) {
            d[kk][h] += src[tt * per + 8 * h0 + h];
            d[kk][h + 8] += src[tt * per + 8 * h1 + h];
          }
        }
      }
    }
#pragma unroll
    for (int kk = 0; kk < 4; ++kk) {
      const int r = rg + kk;
      if (r >= T) continue;
      float o1[8], o2[8];        // chunk c (dims 8c..) and chunk c + 4
      if (pass == 0) {
        const float4* cs = reinterpret_cast<const float4*>(a.rope + (size_t)r * 32 + 8 * c);
#pragma unroll
        for (int h = 0; h < 8; h += 2) {
          const float4 tt = __ldg(cs + h / 2);
          const float l0 = par ? d[kk][h + 8] : d[kk][h], hv0 = par ? d[kk][h] : d[kk][h + 8];
          const float l1 = par ? d[kk][h + 9] : d[kk][h + 1], hv1 = par ? d[kk][h + 1] : d[kk][h + 9];
          o1[h] = l0 * tt.x + hv0 * tt.y;
          o2[h] = hv0 * tt.x - l0 * tt.y;
          o1[h + 1] = l1 * tt.z + hv1 * tt.w;
          o2[h + 1] = hv1 * tt.z - l1 * tt.w;
        }
      } else {
#pragma unroll
        for (int h = 0; h < 8; ++h) {
          o1[h] = par ? d[kk][h + 8] : d[kk][h];
          o2[h] = par ? d[kk][h] : d[kk][h + 8];
        }
      }
      uint4* dst = reinterpret_cast<uint4*>((pass == 0 ? a.dk : a.dv) + ub + (size_t)r * kD);
      dst[c] = pack8(o1);
      dst[c + 4] = pack8(o2);
    }
  }
}

__device__ unsigned g_bwd_err;   // error bits as listed in sa_stage.cuh

struct FastBwdLayout {
  int ring_rows, sc_stride, NS, n_tiles;
  size_t q_smem, kv_smem;
  size_t khat_off, qhat_off, gblk_off, pblk_off, dal_off, sink_off, total;
};

FastBwdLayout fast_bwd_layout(const Problem& pb) {
  constexpr int M = kFastM;
  FastBwdLayout L;
  L.ring_rows = 32;   // a power of two: ring slots are row & (ring_rows - 1)
  while (L.ring_rows < std::max(M + pb.W - 1, M + 2)) L.ring_rows *= 2;
  const int n_slot = pb.W + pb.S + pb.n_off;
  L.sc_stride = n_slot | 1;
  L.NS = pb.W + 2 * pb.n_off;
  L.n_tiles = (pb.T + M - 1) / M;
  const size_t ring_a = (size_t)(L.ring_rows + kMirror) * kRowBytes;
  const size_t ring_b = (size_t)(M / 32) * 2 * pb.S * kD * sizeof(float);
  const size_t ring_bytes = std::max(ring_a, ring_b);
  L.q_smem = ring_bytes + (size_t)pb.S * kRowBytes + 2 * (size_t)M * L.sc_stride * sizeof(float) +
             (size_t)M * pb.n_off * sizeof(float);
  L.kv_smem = ring_a + (size_t)L.NS * M * sizeof(__nv_bfloat16);
  auto up = [](size_t x) { return (x + 255) & ~(size_t)255; };
  const size_t units = (size_t)pb.units();
  const size_t rows = units * pb.T * kD * 2;
  const size_t wblk = units * L.n_tiles * (size_t)L.NS * M * sizeof(__nv_bfloat16);
  L.khat_off = 0;
  L.qhat_off = up(rows);
  L.gblk_off = L.qhat_off + up(rows);
  L.pblk_off = L.gblk_off + up(wblk);
  L.dal_off = L.pblk_off + up(wblk);
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

cudaError_t fast_bwd_read_error(unsigned* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_bwd_err, sizeof(unsigned));
  if (e != cudaSuccess || !clear || *out == 0) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_bwd_err, &zero, sizeof(unsigned));
}

cudaError_t launch_bwd_fast(const Problem& pb, const BwdPtrs& p, cudaStream_t st, int* launches,
                            const void* ctx) {
  const FastBwdLayout L = fast_bwd_layout(pb);
  FastBwdArgs a = {};
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = L.n_tiles;
  a.ring_rows = L.ring_rows; a.sc_stride = L.sc_stride; a.NS = L.NS;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  std::sort(a.f, a.f + pb.n_off);
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.v = reinterpret_cast<const __nv_bfloat16*>(p.v);
  a.dout = reinterpret_cast<const __nv_bfloat16*>(p.dout);
  a.alpha = p.alpha; a.rope = p.rope;
  a.dq = reinterpret_cast<__nv_bfloat16*>(p.dq);
  a.dk = reinterpret_cast<__nv_bfloat16*>(p.dk);
  a.dv = reinterpret_cast<__nv_bfloat16*>(p.dv);
  a.beta = p.beta; a.dbeta = p.dbeta;
  char* ws = reinterpret_cast<char*>(p.workspace);
  const CtxLayout CL = ctx_layout(pb);
  const char* cb = reinterpret_cast<const char*>(ctx);
  void* khat = ctx ? const_cast<char*>(cb + CL.khat_off) : ws + L.khat_off;
  void* qhat = ctx ? const_cast<char*>(cb + CL.qhat_off) : ws + L.qhat_off;
  if (ctx) {
    a.ctx_p = reinterpret_cast<const float*>(cb + CL.p_off);
    a.ctx_dt = reinterpret_cast<const float*>(cb + CL.dt_off);
  }
  a.khat = khat;
  a.qhat = qhat;
  a.gblk = reinterpret_cast<__nv_bfloat16*>(ws + L.gblk_off);
  a.pblk = reinterpret_cast<__nv_bfloat16*>(ws + L.pblk_off);
  a.dal_part = reinterpret_cast<float*>(ws + L.dal_off);
  a.sink_k = reinterpret_cast<float*>(ws + L.sink_off);
  a.sink_v = a.sink_k + (size_t)pb.units() * L.n_tiles * pb.S * kD;
  cudaError_t e;
  if ((e = cudaGetSymbolAddress(reinterpret_cast<void**>(&a.err), g_bwd_err)) != cudaSuccess)
    return e;
  const WaitCfg wc = wait_cfg();
  a.wait_limit = wc.limit;
  a.stall = wc.stall;
  const long long n_rows = pb.units() * pb.T;
  if (!ctx && (e = launch_rope_rows(p.k, p.rope, pb.T, n_rows, kKeyStage, khat, st,
                                    "rope_keys")) != cudaSuccess)
    return e;
  if (!ctx && (e = launch_rope_rows(p.q, p.rope, pb.T, n_rows, pb.scale * kKeyStage, qhat, st,
                                    "rope_queries")) != cudaSuccess)
    return e;
  auto kq = ctx ? k_bwd_q_fast<true> : k_bwd_q_fast<false>;
  if ((e = cudaFuncSetAttribute(kq, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)L.q_smem)) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(k_bwd_kv_fast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)L.kv_smem)) != cudaSuccess)
    return e;
  const unsigned grid = (unsigned)((long long)pb.units() * L.n_tiles);
  trace_mark("bwd_q_fast", st, true);
  kq<<<grid, kFastM, L.q_smem, st>>>(a);
  trace_mark("bwd_q_fast", st, false);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  trace_mark("bwd_kv_fast", st, true);
  k_bwd_kv_fast<<<grid, kFastM, L.kv_smem, st>>>(a);
  trace_mark("bwd_kv_fast", st, false);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  if ((e = launch_reduce_dalpha(a.dal_part, pb.L, pb.B * pb.H * L.n_tiles, p.dalpha, st)) !=
      cudaSuccess)
    return e;
  *launches += ctx ? 3 : 5;
  return cudaSuccess;
}

}  // namespace sa
