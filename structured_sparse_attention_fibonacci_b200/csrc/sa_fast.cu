// Staged forward for bf16 inputs with head dim 64 (the shape of every bf16
// workload of "Depth-Staggered Fibonacci Spacing for Sparse Attention":
// hidden 512 = 8 heads x 64, technical summary, Methodology).
//
// One CTA owns a tile of M consecutive queries of one (layer, batch, head).
//  * Lane mapping: a group of 4 lanes owns 4 consecutive queries; lane c of
//    the group holds 16 of the 64 dims of each, chunks c and c + 4 (a rotate-
//    half RoPE pair stays in one lane), in the group-parity order of the ring
//    reads (sa_stage.cuh).  Every staged row chunk a lane reads is reused for
//    up to 4 queries (window) or 2 queries (an interpolated offset).
//  * Partial dot products of the 4 lanes are combined by a 4-lane transpose
//    reduce-scatter, after which each lane owns one query's full scores.
//  * Staging: the tile's members are visited in increasing lag order (window,
//    then the offsets sorted by f).  Each member needs a contiguous row range;
//    only rows below everything staged so far are fetched, by bulk copies into
//    a ring of shared-memory rows, so every row of the tile's union is read
//    from L2 once per pass.  Keys arrive already rotated (fp16 of RoPE(K) /
//    256, written by the RoPE pre-pass); the allocation-free entry point,
//    which has no room for that, copies raw K rows and rotates them in place.
//  * An offset whose rows lie inside the window ("near") costs nothing: its
//    score is the interpolation of two window scores, and its probability is
//    folded into the two window weights used for PV.  An offset that no query
//    of the tile has yet ("dead") is skipped.
//  * Two passes over the members: scores (key ring), softmax by the owner
//    lane, then PV (value ring).
#include <algorithm>

#include "sa_stage.cuh"

namespace sa {

namespace {

using namespace fast;
using namespace stage;

struct FastArgs {
  int B, H, T, W, n_off, S, n_tiles;
  int ring_rows, sc_stride;
  float scale;
  int f[SA_MAX_OFFSETS];               // ascending
  const __nv_bfloat16* q;
  const void* k;                       // rotated fp16 keys, or raw bf16 K (in-place rotation)
  const __nv_bfloat16* v;
  const float* alpha; const float2* rope;
  __nv_bfloat16* o; float* lse;
  unsigned* err;
  long long wait_limit;                // bounded waits: SM clocks (0: the default)
  int stall;                           // failure-path test: the first staging round waits in vain
  float* save_p;                       // SAVE: [units][W+S+n_off][T] member probabilities
  float* save_dt;                      // SAVE: [units][n_off][T] row-score differences
  __half* save_q;                      // SAVE: [units][T][64] fp16 of RoPE(Q) * scale / 256
  const float* beta;                   // log-prior on offset members [units][T], or nullptr
};

enum : int { kFar = 0, kNear = 1, kDead = 2 };

// Window scores for lags [d0, d0 + LC): rows ig+3-d0-u, u = 0..LC+2, walked
// upward from the lowest; query q (row ig+q) takes row u at lag d0 + q + u - 3.
template <int LC>
__device__ __forceinline__ void window_scores(const unsigned char* ring, int RB, int ig, int d0,
                                              int off0, int d1, int c, const float (&q)[4][16],
                                              float* sc_row, int i_own, float& mx) {
  float acc[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) acc[a][l] = 0.f;
  const unsigned char* p = ring + (size_t)((ig + 1 - d0 - LC) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    float x[16];
    lane_row<true>(p + (LC + 2 - u) * kRowBytes, d1, x);
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
    sc_row[d0 + l] = out[l];
    if (i_own - (d0 + l) >= 0) mx = fmaxf(mx, out[l]);
  }
}

// Window PV for lags [d0, d0 + LC) with weights sc[query][lag].
template <int LC>
__device__ __forceinline__ void window_pv(const unsigned char* ring, int RB, int ig, int d0,
                                          int off0, int d1, const float* sc, int stride,
                                          float (&o)[4][16]) {
  float pw[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) pw[a][l] = sc[a * stride + d0 + l];
  const unsigned char* p = ring + (size_t)((ig + 1 - d0 - LC) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    float x[16];
    lane_row<false>(p + (LC + 2 - u) * kRowBytes, d1, x);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int l = a + u - 3;
      if (l >= 0 && l < LC) axpy16(o[a], pw[a][l], x);
    }
  }
}

// Next offset after k that is neither near nor dead (n_off when none).
__device__ __forceinline__ int next_far(const int* s_kind, int k, int n_off) {
  ++k;
  while (k < n_off && s_kind[k] != kFar) ++k;
  return k;
}

// Rotate, in place, the raw bf16 K rows [a, b) (all inside [0, T)) staged in
// the ring (RB > 0) or in a plain buffer (RB == 0, row r at r * 128), into
// fp16 of RoPE(K) * kKeyStage.  Thread (run j, pair-chunk p) walks a run of
// consecutive rows, stepping the angles by theta_j per row (a run is a few
// rows, so the fp32 recurrence stays within ~1e-6 of the table); odd runs
// touch their two chunks in the opposite order (bank-conflict-free).
__device__ __forceinline__ void rotate_rows(unsigned char* buf, int RB, const float2* rope, int a,
                                            int b, unsigned* err) {
  const int n = b - a;
  if (n <= 0) return;
  const int runs = blockDim.x >> 2;
  const int L = (n + runs - 1) / runs;
  const int j = threadIdx.x >> 2, p = threadIdx.x & 3, par = j & 1;
  const int r0 = a + j * L, r1 = min(r0 + L, b);
  if (r0 >= r1) return;
  float2 cs[8], st[8];
  {
    const float4* g0 = reinterpret_cast<const float4*>(rope + (size_t)r0 * 32 + 8 * p);
    const float4* g1 = reinterpret_cast<const float4*>(rope + 32 + 8 * p);
#pragma unroll
    for (int h = 0; h < 4; ++h) {
      const float4 u = __ldg(g0 + h), w = __ldg(g1 + h);
      cs[2 * h] = make_float2(u.x, u.y); cs[2 * h + 1] = make_float2(u.z, u.w);
      st[2 * h] = make_float2(w.x, w.y); st[2 * h + 1] = make_float2(w.z, w.w);
    }
  }
  const int o0 = half0_off(p, par), o1 = half1_off(p, par);
  for (int row = r0; row < r1; ++row) {
    const int slot = RB ? (row & (RB - 1)) : row;
    uint4* c0 = reinterpret_cast<uint4*>(buf + (size_t)slot * kRowBytes + o0);
    uint4* c1 = reinterpret_cast<uint4*>(buf + (size_t)slot * kRowBytes + o1);
    float y0[8], y1[8];
    unpack8(*c0, y0);
    unpack8(*c1, y1);
    float x1[8], x2[8];
#pragma unroll
    for (int h = 0; h < 8; ++h) {
      const float lo = par ? y1[h] : y0[h], hi = par ? y0[h] : y1[h];
      x1[h] = (lo * cs[h].x - hi * cs[h].y) * kKeyStage;
      x2[h] = (hi * cs[h].x + lo * cs[h].y) * kKeyStage;
      const float c2 = cs[h].x * st[h].x - cs[h].y * st[h].y;
      cs[h].y = cs[h].y * st[h].x + cs[h].x * st[h].y;
      cs[h].x = c2;
    }
    if (half_overflow8(x1) | half_overflow8(x2)) atomicOr(err, kErrRange);
    const uint4 u1 = pack8_h(x1), u2 = pack8_h(x2);
    *c0 = par ? u2 : u1;
    *c1 = par ? u1 : u2;
    if (RB && slot < kMirror) {
      *reinterpret_cast<uint4*>(buf + (size_t)(RB + slot) * kRowBytes + o0) = par ? u2 : u1;
      *reinterpret_cast<uint4*>(buf + (size_t)(RB + slot) * kRowBytes + o1) = par ? u1 : u2;
    }
  }
}

// One staging round of key rows [a, b) into the ring (plus, on the first
// round, the sink rows): copies, wait, and for raw keys the in-place rotation.
// Returns nonzero when a wait gave up (the kernel then returns).
template <bool PRE>
__device__ __forceinline__ int stage_keys(Stager& s, unsigned char* ring, int RB,
                                          unsigned char* sinkb, const FastArgs& a,
                                          const unsigned char* K, int S_stage, int T, int lo,
                                          int hi) {
  stage_ring(s, ring, RB, K, T, lo, hi);
  if (S_stage) stage_plain(s, sinkb, K, min(a.S, T), a.S);
  if (stage_commit_wait(s)) { stage_drain(s); return 1; }
  if (!PRE) {
    rotate_rows(ring, RB, a.rope, max(lo, 0), min(hi, T), a.err);
    if (S_stage) rotate_rows(sinkb, 0, a.rope, 0, min(a.S, T), a.err);
    __syncthreads();
  }
  return 0;
}

// SAVE (training forward): also store, per query, every member's probability
// (window lags unfolded, sinks, offsets) and every offset's row-score
// difference dtau = score(row i-lo-1) - score(row i-lo), the values the
// backward's score pass would recompute.  Offsets are then "near" only when
// both rows lie in the window (lo + 1 <= W - 1), and far offsets always read
// both rows.
template <bool PRE, bool SAVE>
__global__ void __launch_bounds__(kFastM, 4) k_fwd_fast(const FastArgs a) {
  constexpr int M = kFastM;
  extern __shared__ __align__(128) unsigned char smem[];
  const int RB = a.ring_rows;
  unsigned char* ring = smem;
  unsigned char* sinkb = smem + (size_t)(RB + kMirror) * kRowBytes;
  float* sc = reinterpret_cast<float*>(sinkb + (size_t)a.S * kRowBytes);
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_kind[SA_MAX_OFFSETS];
  __shared__ uint64_t bar;

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int T = a.T, W = a.W, S = a.S, n_off = a.n_off;
  const int i0 = tile * M;
  const int t = threadIdx.x, gid = t >> 2, c = t & 3, par = gid & 1;
  const int ig = i0 + 4 * gid;
  const size_t ub = (size_t)unit * T * kD;
  const __nv_bfloat16* Q = a.q + ub;
  const unsigned char* K = reinterpret_cast<const unsigned char*>(a.k) + ub * 2;
  const unsigned char* V = reinterpret_cast<const unsigned char*>(a.v + ub);

  if (t == 0) { mbar_init(&bar, 1); fence_barrier_init(); }
  int bad = 0;
  if (t < n_off) {
    const OffGeo g = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    sg[t] = g;
    bad = !g.ok;
    const int near = g.ok && (g.lo + ((SAVE || g.w != 0.f) ? 1 : 0) <= W - 1);
    const int dead = i0 + M - 1 - g.c < 0;        // no query of the tile has it yet
    s_kind[t] = near ? kNear : (dead ? kDead : kFar);
  }
  bad = __syncthreads_or(bad);
  if (bad) {  // the layer has an offset with no defined row: NaN outputs
    const float qnan = __int_as_float(0x7fc00000);
    for (int e = t; e < M * kChunks; e += M) {
      const int i = i0 + e / kChunks;
      if (i < T) {
        float x[8];
#pragma unroll
        for (int h = 0; h < 8; ++h) x[h] = qnan;
        reinterpret_cast<uint4*>(a.o + ub + (size_t)i * kD)[e % kChunks] = pack8(x);
        if (e % kChunks == 0 && a.lse) a.lse[(size_t)unit * T + i] = qnan;
      }
    }
    return;
  }
  Stager stg = make_stager(&bar, a.err, a.wait_limit, a.stall);

  // This lane's slice of its 4 queries, rotated and scaled (times the inverse
  // of the key staging factor), first half = chunk c + 4 * par.
  const float qs = a.scale * kKeyUnstage;
  float q[4][16];
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const int row = min(ig + qq, T - 1);
    const uint4* g = reinterpret_cast<const uint4*>(Q + (size_t)row * kD);
    float x1[8], x2[8];
    unpack8(__ldg(g + c), x1);
    unpack8(__ldg(g + c + 4), x2);
    const float4* cs = reinterpret_cast<const float4*>(a.rope + (size_t)row * 32 + 8 * c);
#pragma unroll
    for (int h = 0; h < 8; h += 2) {
      const float4 tt = __ldg(cs + h / 2);
      const float r0 = (x1[h] * tt.x - x2[h] * tt.y) * qs;
      const float r1 = (x2[h] * tt.x + x1[h] * tt.y) * qs;
      const float r2 = (x1[h + 1] * tt.z - x2[h + 1] * tt.w) * qs;
      const float r3 = (x2[h + 1] * tt.z + x1[h + 1] * tt.w) * qs;
      q[qq][h] = par ? r1 : r0;
      q[qq][h + 8] = par ? r0 : r1;
      q[qq][h + 1] = par ? r3 : r2;
      q[qq][h + 9] = par ? r2 : r3;
    }
  }
  const int off0 = half0_off(c, par), d1 = half1_off(c, par) - off0;
  if (SAVE) {
    // the backward's rotated, scaled queries: q holds RoPE(Q) * scale * 256
    const int h0 = c + 4 * par, h1 = c + 4 - 4 * par;
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) {
      const int i = ig + qq;
      if (i >= T) continue;
      float y0[8], y1[8];
#pragma unroll
      for (int h = 0; h < 8; ++h) {
        y0[h] = q[qq][h] * (kKeyStage * kKeyStage);
        y1[h] = q[qq][h + 8] * (kKeyStage * kKeyStage);
      }
      if (half_overflow8(y0) | half_overflow8(y1)) atomicOr(a.err, kErrRange);
      uint4* dst = reinterpret_cast<uint4*>(a.save_q + ub + (size_t)i * kD);
      dst[h0] = pack8_h(y0);
      dst[h1] = pack8_h(y1);
    }
  }

  const int lr = 4 * gid + c;                  // this lane's query, tile-local
  const int i_own = ig + c;                    // ... and its position
  // its log-prior on the offset members (0 without one)
  const float prior = (a.beta && i_own < T) ? __ldg(a.beta + (size_t)unit * T + i_own) : 0.f;
  float mx = -INFINITY;                        // running max of its valid scores
  float* my_sc = sc + (size_t)lr * a.sc_stride;
  const int win_lo = i0 - W + 1, win_hi = i0 + M;

  // ---------------- pass 1: scores ----------------
  if (stage_keys<PRE>(stg, ring, RB, sinkb, a, K, 1, T, win_lo, win_hi)) return;
  dbg_rows(stg, ig - W + 1, ig + 4);
  {
    int d0 = 0;
    // lags in blocks of 3 (the loop body's code stays small: measured on B200,
    // unrolled 8-lag blocks ran 9-11% slower from instruction-cache misses)
    while (W - d0 >= 3) { window_scores<3>(ring, RB, ig, d0, off0, d1, c, q, my_sc, i_own, mx); d0 += 3; }
    if (W - d0 >= 2) { window_scores<2>(ring, RB, ig, d0, off0, d1, c, q, my_sc, i_own, mx); d0 += 2; }
    if (W - d0 >= 1) { window_scores<1>(ring, RB, ig, d0, off0, d1, c, q, my_sc, i_own, mx); d0 += 1; }
  }
  for (int s0 = 0; s0 < S; s0 += 4) {
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float x[16];
      lane_row<true>(sinkb + (size_t)min(s0 + j, S - 1) * kRowBytes + off0, d1, x);
#pragma unroll
      for (int qq = 0; qq < 4; ++qq) acc[qq][j] = dot16(q[qq], x);
    }
    float out[4];
    reduce_scatter4<4>(acc, out, c);
#pragma unroll
    for (int j = 0; j < 4; ++j)
      if (s0 + j < S) {
        my_sc[W + s0 + j] = out[j];
        if (s0 + j <= i_own) mx = fmaxf(mx, out[j]);
      }
  }
  // far offsets, staged in batches: consecutive members whose rows span at
  // most RB rows share one staging round and are computed back to back.  A
  // far member reads rows [i0 - lo - 1, i0 + M - lo).
  {
    int low = win_lo;
    int kk = next_far(s_kind, -1, n_off);
    while (kk < n_off) {
      const int hi = i0 + M - sg[kk].lo;
      int last = kk, nx = next_far(s_kind, kk, n_off);
      while (nx < n_off && hi - (i0 - sg[nx].lo - 1) <= RB) {
        last = nx;
        nx = next_far(s_kind, nx, n_off);
      }
      const int lo_row = i0 - sg[last].lo - 1;
      if (lo_row < low) {              // only rows below everything staged are new
        __syncthreads();
        if (stage_keys<PRE>(stg, ring, RB, sinkb, a, K, 0, T, lo_row, min(hi, low))) return;
        low = lo_row;
      }
      for (int m = kk; m < nx; m = next_far(s_kind, m, n_off)) {
        const OffGeo g = sg[m];
        const int two = SAVE || g.w != 0.f;
        dbg_rows(stg, ig - g.lo - 1 + (two ? 0 : 1), ig - g.lo + 4);
        const unsigned char* p = ring + (size_t)((ig - g.lo - 1) & (RB - 1)) * kRowBytes + off0;
        float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 5; ++u) {
          if (u == 0 && !two) continue;
          float x[16];
          lane_row<true>(p + u * kRowBytes, d1, x);
          if (u <= 3) pb[u] = dot16(q[u], x);
          if (u >= 1) pa[u - 1] = dot16(q[u - 1], x);
        }
        constexpr int NV = SAVE ? 2 : 1;
        float part[4][NV];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) {
          part[qq][0] = g.wa * pa[qq] + g.w * pb[qq];
          if (SAVE) part[qq][NV - 1] = pb[qq] - pa[qq];
        }
        float out[NV];
        reduce_scatter4<NV>(part, out, c);
        const float sv = out[0] + prior;
        my_sc[W + S + m] = sv;
        if (SAVE && i_own < T) a.save_dt[((size_t)unit * n_off + m) * T + i_own] = out[NV - 1];
        if (i_own - g.c >= 0) mx = fmaxf(mx, sv);
      }
      kk = nx;
    }
  }
  __syncthreads();

  // ---------------- softmax (owner lane of each query) ----------------
  // The running max was taken as scores were produced; one pass turns scores
  // into unnormalised weights e = exp(score - max); 1/sum is applied to O.
  float inv_l = 0.f;
  {
    const int i = i_own;
    if (i < T) {
      for (int kk = 0; kk < n_off; ++kk) {    // near offsets: from two window scores
        if (SAVE && s_kind[kk] == kDead) a.save_dt[((size_t)unit * n_off + kk) * T + i] = 0.f;
        if (s_kind[kk] != kNear) continue;
        const OffGeo g = sg[kk];
        float sv = g.wa * my_sc[g.lo];
        if (g.w != 0.f) sv += g.w * my_sc[g.lo + 1];
        sv += prior;
        my_sc[W + S + kk] = sv;
        if (SAVE)
          a.save_dt[((size_t)unit * n_off + kk) * T + i] = my_sc[g.lo + 1] - my_sc[g.lo];
        if (i - g.c >= 0) mx = fmaxf(mx, sv);
      }
      float l = 0.f;
      for (int d = 0; d < W; ++d) {
        const float e = (i - d >= 0) ? __expf(my_sc[d] - mx) : 0.f;
        my_sc[d] = e; l += e;
      }
      for (int sk = 0; sk < S; ++sk) {
        const float e = (sk <= i) ? __expf(my_sc[W + sk] - mx) : 0.f;
        my_sc[W + sk] = e; l += e;
      }
      for (int kk = 0; kk < n_off; ++kk) {
        const OffGeo g = sg[kk];
        const float e =
            (s_kind[kk] != kDead && i - g.c >= 0) ? __expf(my_sc[W + S + kk] - mx) : 0.f;
        my_sc[W + S + kk] = e; l += e;
      }
      inv_l = 1.f / l;
      if (SAVE) {                              // probabilities, window lags unfolded
        float* sp = a.save_p + (size_t)unit * (W + S + n_off) * T + i;
        for (int m = 0; m < W + S + n_off; ++m) sp[(size_t)m * T] = my_sc[m] * inv_l;
      }
      for (int kk = 0; kk < n_off; ++kk) {     // fold near offsets into the window weights
        if (s_kind[kk] != kNear) continue;
        const OffGeo g = sg[kk];
        const float e = my_sc[W + S + kk];
        my_sc[g.lo] += g.wa * e;
        if (g.w != 0.f) my_sc[g.lo + 1] += g.w * e;
      }
      if (a.lse) a.lse[(size_t)unit * T + i] = mx + __logf(l);
    } else {
      for (int d = 0; d < W + S + n_off; ++d) my_sc[d] = 0.f;
    }
  }
  __syncthreads();

  // ---------------- pass 2: PV ----------------
  float o[4][16];
#pragma unroll
  for (int qq = 0; qq < 4; ++qq)
#pragma unroll
    for (int h = 0; h < 16; ++h) o[qq][h] = 0.f;
  const float* grp_sc = sc + (size_t)(4 * gid) * a.sc_stride;
  stage_ring(stg, ring, RB, V, T, win_lo, win_hi);
  stage_plain(stg, sinkb, V, min(S, T), S);
  if (stage_commit_wait(stg)) { stage_drain(stg); return; }
  dbg_rows(stg, ig - W + 1, ig + 4);
  {
    int d0 = 0;
    while (W - d0 >= 3) { window_pv<3>(ring, RB, ig, d0, off0, d1, grp_sc, a.sc_stride, o); d0 += 3; }
    if (W - d0 >= 2) { window_pv<2>(ring, RB, ig, d0, off0, d1, grp_sc, a.sc_stride, o); d0 += 2; }
    if (W - d0 >= 1) { window_pv<1>(ring, RB, ig, d0, off0, d1, grp_sc, a.sc_stride, o); d0 += 1; }
  }
  for (int s = 0; s < S; ++s) {
    float x[16];
    lane_row<false>(sinkb + (size_t)s * kRowBytes + off0, d1, x);
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) axpy16(o[qq], grp_sc[qq * a.sc_stride + W + s], x);
  }
  {
    int low = win_lo;
    int kk = next_far(s_kind, -1, n_off);
    while (kk < n_off) {
      const int hi = i0 + M - sg[kk].lo;
      int last = kk, nx = next_far(s_kind, kk, n_off);
      while (nx < n_off && hi - (i0 - sg[nx].lo - 1) <= RB) {
        last = nx;
        nx = next_far(s_kind, nx, n_off);
      }
      const int lo_row = i0 - sg[last].lo - 1;
      if (lo_row < low) {
        __syncthreads();
        stage_ring(stg, ring, RB, V, T, lo_row, min(hi, low));
        if (stage_commit_wait(stg)) { stage_drain(stg); return; }
        low = lo_row;
      }
      for (int m = kk; m < nx; m = next_far(s_kind, m, n_off)) {
        const OffGeo g = sg[m];
        const int two = g.w != 0.f;
        dbg_rows(stg, ig - g.lo - 1 + (two ? 0 : 1), ig - g.lo + 4);
        float p[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) p[qq] = grp_sc[qq * a.sc_stride + W + S + m];
        const unsigned char* rp = ring + (size_t)((ig - g.lo - 1) & (RB - 1)) * kRowBytes + off0;
#pragma unroll
        for (int u = 0; u < 5; ++u) {
          if (u == 0 && !two) continue;
          float x[16];
          lane_row<false>(rp + u * kRowBytes, d1, x);
          if (u <= 3 && two) axpy16(o[u], p[u] * g.w, x);
          if (u >= 1) axpy16(o[u - 1], p[u - 1] * g.wa, x);
        }
      }
      kk = nx;
    }
  }

  // 1 / sum of the weights, from each query's owner lane (lane 4*gid + qq)
  float inv[4];
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) inv[qq] = __shfl_sync(0xffffffffu, inv_l, (t & 28) + qq);
  const int h0 = c + 4 * par, h1 = c + 4 - 4 * par;
#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const int i = ig + qq;
#pragma unroll
    for (int h = 0; h < 16; ++h) o[qq][h] *= inv[qq];
    if (i < T) {
      uint4* dst = reinterpret_cast<uint4*>(a.o + ub + (size_t)i * kD);
      dst[h0] = pack8(o[qq]);
      dst[h1] = pack8(o[qq] + 8);
    }
  }
}

__device__ unsigned g_fwd_err;   // error bits as listed in sa_stage.cuh

int ring_rows_for(const Problem& pb) {
  int rr = 32;   // a power of two: ring slots are row & (rr - 1)
  while (rr < std::max(kFastM + pb.W - 1, kFastM + 2)) rr *= 2;
  return rr;
}

}  // namespace

bool fast_fwd_supported(const Problem& pb) {
  return pb.dtype == SA_DTYPE_BF16 && pb.D == kD && pb.W <= 256;
}

size_t fast_fwd_smem(const Problem& pb, int* ring_rows, int* sc_stride) {
  const int rr = ring_rows_for(pb);
  // odd stride: the 8 lane groups of a warp read rows 4 apart, and the 32
  // owner lanes read 32 consecutive rows, without shared-memory bank conflicts
  const int n_slot = pb.W + pb.S + pb.n_off;
  const int st = n_slot | 1;
  if (ring_rows) *ring_rows = rr;
  if (sc_stride) *sc_stride = st;
  return (size_t)(rr + kMirror) * kRowBytes + (size_t)pb.S * kRowBytes +
         (size_t)kFastM * st * sizeof(float);
}

size_t fast_fwd_workspace(const Problem& pb) {
  return fast_fwd_supported(pb) ? (size_t)pb.units() * pb.T * kD * 2 : 0;
}

cudaError_t launch_fwd_fast(const Problem& pb, const FwdPtrs& p, void* keys_ws, cudaStream_t st,
                            int* launches, float* save_p, float* save_dt, void* save_q) {
  FastArgs a = {};
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = (pb.T + kFastM - 1) / kFastM;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  std::sort(a.f, a.f + pb.n_off);
  const size_t smem = fast_fwd_smem(pb, &a.ring_rows, &a.sc_stride);
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.v = reinterpret_cast<const __nv_bfloat16*>(p.v);
  a.alpha = p.alpha; a.rope = p.rope;
  a.o = reinterpret_cast<__nv_bfloat16*>(p.o); a.lse = p.lse;
  a.save_p = save_p; a.save_dt = save_dt; a.save_q = reinterpret_cast<__half*>(save_q);
  a.beta = p.beta;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&a.err), g_fwd_err);
  const WaitCfg wc = wait_cfg();
  a.wait_limit = wc.limit;
  a.stall = wc.stall;
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((long long)pb.units() * a.n_tiles);
  auto launch = [&](auto kernel) -> cudaError_t {
    cudaError_t r = cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         (int)smem);
    if (r != cudaSuccess) return r;
    trace_mark("fwd_fast", st, true);
    kernel<<<grid, kFastM, smem, st>>>(a);
    trace_mark("fwd_fast", st, false);
    return cudaGetLastError();
  };
  if (keys_ws) {
    // rotated keys, fp16 of RoPE(K) / 256, then the staged kernel
    if ((e = launch_rope_rows(p.k, p.rope, pb.T, pb.units() * pb.T, kKeyStage, keys_ws, st,
                              "rope_keys")) != cudaSuccess)
      return e;
    *launches += 1;
    a.k = keys_ws;
    e = (save_p && save_dt && save_q) ? launch(k_fwd_fast<true, true>)
                                      : launch(k_fwd_fast<true, false>);
  } else {
    a.k = p.k;
    e = launch(k_fwd_fast<false, false>);
  }
  if (e == cudaSuccess) *launches += 1;
  return e;
}

cudaError_t fast_fwd_read_error(unsigned* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_fwd_err, sizeof(unsigned));
  if (e != cudaSuccess || !clear || *out == 0) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_fwd_err, &zero, sizeof(unsigned));
}

}  // namespace sa
