// Staged forward for bf16 inputs with head dim 64 (the shape of every bf16
// workload of "Depth-Staggered Fibonacci Spacing for Sparse Attention":
// hidden 512 = 8 heads x 64, technical summary, Methodology).
//
// One CTA owns a tile of M consecutive queries of one (layer, batch, head).
//  * Lane mapping: a group of 4 lanes owns 4 consecutive queries; lane c of
//    the group holds dims [8c, 8c+8) and [32+8c, 32+8c+8) of each (a rotate-
//    half RoPE pair stays in one lane).  Every staged row chunk a lane reads
//    is reused for up to 4 queries (window) or 2 queries (an interpolated
//    offset), which keeps shared-memory traffic near one byte per FMA.
//  * Partial dot products of the 4 lanes are combined by a 4-lane transpose
//    reduce-scatter, after which each lane owns one query's full scores.
//  * Staging: the tile's members are visited in increasing lag order (window,
//    then the offsets sorted by f).  Each member needs a contiguous row range;
//    only rows below everything staged so far are fetched, into a ring of
//    shared-memory rows, so every row of the tile's union is read from L2 once
//    per pass.  K rows are rotated (RoPE) on the way in and kept as scaled
//    fp16, V rows as bf16, with a 16-byte-chunk XOR swizzle.
//  * An offset whose rows lie inside the window ("near") costs nothing: its
//    score is the interpolation of two window scores, and its probability is
//    folded into the two window weights used for PV.
//  * Two passes over the members: scores (K ring), softmax by the owner lane,
//    then PV (V ring).
#include <algorithm>

#include "sa_fast_common.cuh"

namespace sa {

namespace {

using namespace fast;

struct FastArgs {
  int B, H, T, W, n_off, S, n_tiles;
  int ring_rows, sc_stride;
  float scale;
  int f[SA_MAX_OFFSETS];               // ascending
  const __nv_bfloat16* q; const __nv_bfloat16* k; const __nv_bfloat16* v;
  const float* alpha; const float2* rope;
  __nv_bfloat16* o; float* lse;
};

// Window scores for lags [d0, d0 + LC): rows ig+3-d0-u, u = 0..LC+2; query q
// (row ig+q) takes row u at lag d0 + (q + u - 3).
template <int LC>
__device__ __forceinline__ void window_scores(const uint4* ring, int ring_rows, int ig, int d0,
                                              int c, const float (&q)[4][16], float* sc_row,
                                              int i_own, float& mx) {
  float acc[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) acc[a][l] = 0.f;
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    const int row = max(ig + 3 - d0 - u, 0);
    float x[16];
    ring_load<true>(ring, row & (ring_rows - 1), c, x);
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
__device__ __forceinline__ void window_pv(const uint4* ring, int ring_rows, int ig, int d0, int c,
                                          const float* sc, int stride, float (&o)[4][16]) {
  float pw[4][LC];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int l = 0; l < LC; ++l) pw[a][l] = sc[a * stride + d0 + l];
#pragma unroll
  for (int u = 0; u < LC + 3; ++u) {
    const int row = max(ig + 3 - d0 - u, 0);
    float x[16];
    ring_load(ring, row & (ring_rows - 1), c, x);
#pragma unroll
    for (int a = 0; a < 4; ++a) {
      const int l = a + u - 3;
      if (l >= 0 && l < LC) axpy16(o[a], pw[a][l], x);
    }
  }
}

// Rows a far offset's member needs for the tile [i0, i0 + M): [lo, hi).
__device__ __forceinline__ int far_seg_lo(const OffGeo& g, int i0) {
  return max(0, i0 - g.lo - (g.w != 0.f ? 1 : 0));
}
__device__ __forceinline__ int far_seg_hi(const OffGeo& g, int i0, int T) {
  return max(0, min(T, i0 + kFastM - g.lo));
}
// Next offset after k that is not folded into the window (n_off when none).
__device__ __forceinline__ int next_far(const int* s_fold, int k, int n_off) {
  ++k;
  while (k < n_off && s_fold[k]) ++k;
  return k;
}

__global__ void __launch_bounds__(kFastM, 4) k_fwd_fast(const FastArgs a) {
  constexpr int M = kFastM;
  extern __shared__ __align__(16) unsigned char smem[];
  uint4* ring = reinterpret_cast<uint4*>(smem);
  uint4* sinkb = ring + (size_t)a.ring_rows * kChunks;
  float* sc = reinterpret_cast<float*>(sinkb + (size_t)a.S * kChunks);
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_fold[SA_MAX_OFFSETS];

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int T = a.T, W = a.W, S = a.S, n_off = a.n_off;
  const int i0 = tile * M;
  const int t = threadIdx.x, gid = t >> 2, c = t & 3;
  const int ig = i0 + 4 * gid;
  const size_t ub = (size_t)unit * T * kD;
  const __nv_bfloat16* Q = a.q + ub;
  const __nv_bfloat16* K = a.k + ub;
  const __nv_bfloat16* V = a.v + ub;

  int bad = 0;
  if (t < n_off) {
    const OffGeo g = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    sg[t] = g;
    bad = !g.ok;
    s_fold[t] = g.ok && (g.lo + (g.w != 0.f ? 1 : 0) <= W - 1);
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

  // zero the ring and the sink rows so unstaged slots always hold finite values
  // (sink rows s >= T are never attended and never staged)
  for (int e = t; e < (a.ring_rows + S) * kChunks; e += M) ring[e] = make_uint4(0, 0, 0, 0);
  const int S_rows = min(S, T);

  // this lane's slice of its 4 queries, rotated and scaled (times the inverse
  // of the key staging factor)
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
      q[qq][h] = (x1[h] * tt.x - x2[h] * tt.y) * qs;
      q[qq][h + 8] = (x2[h] * tt.x + x1[h] * tt.y) * qs;
      q[qq][h + 1] = (x1[h + 1] * tt.z - x2[h + 1] * tt.w) * qs;
      q[qq][h + 9] = (x2[h + 1] * tt.z + x1[h + 1] * tt.w) * qs;
    }
  }

  const int lr = 4 * gid + c;                  // this lane's query, tile-local
  const int i_own = ig + c;                    // ... and its position
  float mx = -INFINITY;                        // running max of its valid scores
  float* my_sc = sc + (size_t)lr * a.sc_stride;
  const int win_lo = max(0, i0 - W + 1), win_hi = min(T, i0 + M);
  const int RB = a.ring_rows;

  // ---------------- pass 1: scores ----------------
  __syncthreads();
  stage_rotate<true>(ring, RB, K, a.rope, win_lo, win_hi, kKeyStage);
  stage_sinks<true>(sinkb, S_rows, K, a.rope);
  __syncthreads();
  {
    int d0 = 0;
    while (W - d0 >= 8) { window_scores<8>(ring, RB, ig, d0, c, q, my_sc, i_own, mx); d0 += 8; }
    if (W - d0 >= 4) { window_scores<4>(ring, RB, ig, d0, c, q, my_sc, i_own, mx); d0 += 4; }
    if (W - d0 >= 2) { window_scores<2>(ring, RB, ig, d0, c, q, my_sc, i_own, mx); d0 += 2; }
    if (W - d0 >= 1) { window_scores<1>(ring, RB, ig, d0, c, q, my_sc, i_own, mx); d0 += 1; }
  }
  for (int s0 = 0; s0 < S; s0 += 4) {
    float acc[4][4];
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      float x[16];
      sink_load<true>(sinkb, min(s0 + j, S - 1), c, x);
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
  // most RB rows share one staging round and are computed back to back
  {
    int low = win_lo;
    int kk = next_far(s_fold, -1, n_off);
    while (kk < n_off) {
      const int hi = far_seg_hi(sg[kk], i0, T);
      int last = kk, nx = next_far(s_fold, kk, n_off);
      while (nx < n_off && hi - far_seg_lo(sg[nx], i0) <= RB) {
        last = nx;
        nx = next_far(s_fold, nx, n_off);
      }
      // rows the batch needs: [lo_row, hi); only those below `low` are new
      const int lo_row = far_seg_lo(sg[last], i0);
      if (lo_row < low && lo_row < hi) {
        __syncthreads();
        stage_rotate<true>(ring, RB, K, a.rope, lo_row, min(hi, low), kKeyStage);
        low = lo_row;
        __syncthreads();
      }
      for (int m = kk; m < nx; m = next_far(s_fold, m, n_off)) {
        const OffGeo g = sg[m];
        const int two = g.w != 0.f;
        float pa[4] = {0.f, 0.f, 0.f, 0.f}, pb[4] = {0.f, 0.f, 0.f, 0.f};
#pragma unroll
        for (int u = 0; u < 5; ++u) {
          if (u == 0 && !two) continue;
          const int row = max(ig - g.lo - 1 + u, 0);
          float x[16];
          ring_load<true>(ring, row & (RB - 1), c, x);
          if (u <= 3) pb[u] = dot16(q[u], x);
          if (u >= 1) pa[u - 1] = dot16(q[u - 1], x);
        }
        float part[4][1];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) part[qq][0] = g.wa * pa[qq] + g.w * pb[qq];
        float out[1];
        reduce_scatter4<1>(part, out, c);
        my_sc[W + S + m] = out[0];
        if (i_own - g.c >= 0) mx = fmaxf(mx, out[0]);
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
        if (!s_fold[kk]) continue;
        const OffGeo g = sg[kk];
        float sv = g.wa * my_sc[g.lo];
        if (g.w != 0.f) sv += g.w * my_sc[g.lo + 1];
        my_sc[W + S + kk] = sv;
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
        const float e = (i - g.c >= 0) ? __expf(my_sc[W + S + kk] - mx) : 0.f;
        my_sc[W + S + kk] = e; l += e;
        if (s_fold[kk]) {                      // fold into the two window weights
          my_sc[g.lo] += g.wa * e;
          if (g.w != 0.f) my_sc[g.lo + 1] += g.w * e;
        }
      }
      inv_l = 1.f / l;
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
  stage_copy(ring, RB, V, win_lo, win_hi);
  stage_sinks<false>(sinkb, S_rows, V, a.rope);
  __syncthreads();
  {
    int d0 = 0;
    while (W - d0 >= 8) { window_pv<8>(ring, RB, ig, d0, c, grp_sc, a.sc_stride, o); d0 += 8; }
    if (W - d0 >= 4) { window_pv<4>(ring, RB, ig, d0, c, grp_sc, a.sc_stride, o); d0 += 4; }
    if (W - d0 >= 2) { window_pv<2>(ring, RB, ig, d0, c, grp_sc, a.sc_stride, o); d0 += 2; }
    if (W - d0 >= 1) { window_pv<1>(ring, RB, ig, d0, c, grp_sc, a.sc_stride, o); d0 += 1; }
  }
  for (int s = 0; s < S; ++s) {
    float x[16];
    sink_load(sinkb, s, c, x);
#pragma unroll
    for (int qq = 0; qq < 4; ++qq) axpy16(o[qq], grp_sc[qq * a.sc_stride + W + s], x);
  }
  {
    int low = win_lo;
    int kk = next_far(s_fold, -1, n_off);
    while (kk < n_off) {
      const int hi = far_seg_hi(sg[kk], i0, T);
      int last = kk, nx = next_far(s_fold, kk, n_off);
      while (nx < n_off && hi - far_seg_lo(sg[nx], i0) <= RB) {
        last = nx;
        nx = next_far(s_fold, nx, n_off);
      }
      const int lo_row = far_seg_lo(sg[last], i0);
      if (lo_row < low && lo_row < hi) {
        __syncthreads();
        stage_copy(ring, RB, V, lo_row, min(hi, low));
        low = lo_row;
        __syncthreads();
      }
      for (int m = kk; m < nx; m = next_far(s_fold, m, n_off)) {
        const OffGeo g = sg[m];
        const int two = g.w != 0.f;
        float p[4];
#pragma unroll
        for (int qq = 0; qq < 4; ++qq) p[qq] = grp_sc[qq * a.sc_stride + W + S + m];
#pragma unroll
        for (int u = 0; u < 5; ++u) {
          if (u == 0 && !two) continue;
          const int row = max(ig - g.lo - 1 + u, 0);
          float x[16];
          ring_load(ring, row & (RB - 1), c, x);
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
#pragma unroll
  for (int qq = 0; qq < 4; ++qq)
#pragma unroll
    for (int h = 0; h < 16; ++h) o[qq][h] *= inv[qq];

#pragma unroll
  for (int qq = 0; qq < 4; ++qq) {
    const int i = ig + qq;
    if (i < T) {
      uint4* dst = reinterpret_cast<uint4*>(a.o + ub + (size_t)i * kD);
      dst[c] = pack8(o[qq]);
      dst[c + 4] = pack8(o[qq] + 8);
    }
  }
}

}  // namespace

bool fast_fwd_supported(const Problem& pb) {
  return pb.dtype == SA_DTYPE_BF16 && pb.D == kD && pb.W <= 256;
}

size_t fast_fwd_smem(const Problem& pb, int* ring_rows, int* sc_stride) {
  int rr = 32;   // a power of two: ring slots are row & (rr - 1)
  while (rr < std::max(kFastM + pb.W - 1, kFastM + 2)) rr *= 2;
  // odd stride: the 8 lane groups of a warp read rows 4 apart, and the 32
  // owner lanes read 32 consecutive rows, without shared-memory bank conflicts
  const int n_slot = pb.W + pb.S + pb.n_off;
  const int st = n_slot | 1;
  if (ring_rows) *ring_rows = rr;
  if (sc_stride) *sc_stride = st;
  return (size_t)rr * 128 + (size_t)pb.S * 128 + (size_t)kFastM * st * sizeof(float);
}

cudaError_t launch_fwd_fast(const Problem& pb, const FwdPtrs& p, cudaStream_t st, int* launches) {
  FastArgs a = {};
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = (pb.T + kFastM - 1) / kFastM;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  std::sort(a.f, a.f + pb.n_off);
  const size_t smem = fast_fwd_smem(pb, &a.ring_rows, &a.sc_stride);
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.k = reinterpret_cast<const __nv_bfloat16*>(p.k);
  a.v = reinterpret_cast<const __nv_bfloat16*>(p.v);
  a.alpha = p.alpha; a.rope = p.rope;
  a.o = reinterpret_cast<__nv_bfloat16*>(p.o); a.lse = p.lse;
  cudaError_t e = cudaFuncSetAttribute(k_fwd_fast, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                       (int)smem);
  if (e != cudaSuccess) return e;
  const unsigned grid = (unsigned)((long long)pb.units() * a.n_tiles);
  trace_mark("fwd_fast", st, true);
  k_fwd_fast<<<grid, kFastM, smem, st>>>(a);
  trace_mark("fwd_fast", st, false);
  e = cudaGetLastError();
  if (e == cudaSuccess) *launches += 1;
  return e;
}

}  // namespace sa
