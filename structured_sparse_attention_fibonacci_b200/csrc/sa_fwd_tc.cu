// Tensor-core forward for bf16 inputs with head dim 64 (the shape of every
// bf16 workload of "Depth-Staggered Fibonacci Spacing for Sparse Attention":
// hidden 512 = 8 heads x 64, technical summary, Methodology).
//
// One CTA owns a tile of 128 consecutive queries of one (layer, batch, head);
// each warp owns 32 of them as two m16 tiles and does all its dot products
// with warp-level mma.sync (fp32 accumulate):
//  * scores, Q^ . K^ (fp16 operands; the RoPE pre-pass stores K^ = RoPE(K) /
//    256, the query fragments carry RoPE(q) * scale):
//      window band: the 16 queries of a tile against the key rows
//        [floor16(q0 - W + 1), q0 + 16), band entries (lag < W) kept;
//      sinks: against the sink rows;
//      far offset k: against the 24 rows [q0 - lo - 1, q0 - lo + 23); query r
//        takes columns r (row b = i - lo - 1) and r + 1 (row a = i - lo),
//        interpolated with weights (w, 1 - w);
//  * softmax by an owner thread per query (scores in shared memory);
//  * output, P . V (bf16 operands): the band of window weights, the sink
//    weights, and per far offset the bidiagonal weights (p w, p (1 - w)) on
//    the same 24 rows (a 16-row and an 8-row k step).
// Near offsets (both rows inside the window) are scored from two window
// scores and folded into the window weights; offsets that no query of the
// tile has yet are skipped.
// Rows are staged by 8-row tensor copies into a 128-byte-swizzled ring
// (sa_tc.cuh): the window first, then the far offsets in increasing lag
// order, consecutive offsets sharing a staging round while their rows span
// at most the ring; only rows below everything staged so far are fetched.
#include <algorithm>
#include <cstring>

#include "sa_tc.cuh"

namespace sa {

namespace {

using namespace fast;
using namespace stage;
using namespace tc;

struct TcFwdArgs {
  CUtensorMap tmK;                     // rotated keys, fp16 [units][T][64]
  CUtensorMap tmV;                     // V, bf16 [units][T][64]
  int B, H, T, W, n_off, S, n_tiles, ring_rows, sc_stride;
  float scale;
  int f[SA_MAX_OFFSETS];               // ascending
  const __nv_bfloat16* q;
  const float* alpha; const float2* rope;
  __nv_bfloat16* o; float* lse;
  unsigned* err;
  long long wait_limit;                // bounded waits: SM clocks (0: the default)
  int stall;                           // failure-path test: the first staging round waits in vain
  const float* beta;                   // log-prior on offset members [units][T], or nullptr
};

enum : int { kFar = 0, kNear = 1, kDead = 2 };

__device__ __forceinline__ int next_far(const int* s_kind, int k, int n_off) {
  ++k;
  while (k < n_off && s_kind[k] != kFar) ++k;
  return k;
}

// A fragments of RoPE(q) * scale (fp16) for the m16 tile of queries qb..qb+15:
// aq[ks] holds k step ks (dims 16 ks .. 16 ks + 15).  A dim d < 32 and its
// rotate-half partner d + 32 sit in k steps ks and ks + 2 of the same lane.
__device__ __forceinline__ void q_frags(const TcFwdArgs& a, const __nv_bfloat16* Q, int qb,
                                        int lane, uint32_t (&aq)[4][4]) {
  const int g = lane >> 2, t = lane & 3;
  bool over = false;                            // a value beyond fp16's range
#pragma unroll
  for (int h = 0; h < 2; ++h) {                 // row g (regs 0, 2) and g + 8 (regs 1, 3)
    const int row = min(qb + g + 8 * h, a.T - 1);
    const __nv_bfloat16* qr = Q + (size_t)row * kD;
    const float2* cs = a.rope + (size_t)row * 32;
#pragma unroll
    for (int ks = 0; ks < 2; ++ks)
#pragma unroll
      for (int p = 0; p < 2; ++p) {
        const int d = 16 * ks + 2 * t + 8 * p;  // dims d, d + 1 (< 32) and d + 32, d + 33
        const uint32_t lo2 = __ldg(reinterpret_cast<const unsigned*>(qr + d));
        const uint32_t hi2 = __ldg(reinterpret_cast<const unsigned*>(qr + d + 32));
        const float4 c = __ldg(reinterpret_cast<const float4*>(cs + d));
        const float x0 = bf16lo(lo2), x1 = bf16hi(lo2), y0 = bf16lo(hi2), y1 = bf16hi(hi2);
        float r[8] = {(x0 * c.x - y0 * c.y) * a.scale, (x1 * c.z - y1 * c.w) * a.scale,
                      (y0 * c.x + x0 * c.y) * a.scale, (y1 * c.z + x1 * c.w) * a.scale,
                      0.f, 0.f, 0.f, 0.f};
        over |= half_overflow8(r);
        aq[ks][h + 2 * p] = pack_h2(r[0], r[1]);
        aq[ks + 2][h + 2 * p] = pack_h2(r[2], r[3]);
      }
  }
  if (over) atomicOr(a.err, kErrRange);
}

__device__ __forceinline__ void qk_mma(const uint32_t (&aq)[4][4], const uint32_t (&b)[2][4],
                                       float (&c)[4]) {
  mma_f16(c, aq[0], b[0][0], b[0][1]);
  mma_f16(c, aq[1], b[0][2], b[0][3]);
  mma_f16(c, aq[2], b[1][0], b[1][1]);
  mma_f16(c, aq[3], b[1][2], b[1][3]);
}

// acc[0..7] (8 n tiles = 64 dims) += (A + Alo)(16 x 16 key rows) . V rows
// kb .. kb + 15 (the weights as the bf16 pair split_bf16x2 makes); all eight B
// fragments are loaded before the (independent) mma.
template <bool POW2>
__device__ __forceinline__ void pv_k16(const Ring& ring, int kb, int lane,
                                       const uint32_t (&A)[4], const uint32_t (&Alo)[4],
                                       float (&acc)[8][4]) {
  int slot = ring_slot<POW2>(ring, kb) + (lane & 15);
  if (slot >= ring.rows) slot -= ring.rows;
  const uint32_t base = ring.base + (uint32_t)slot * 128u;
  const int x = slot & 7, m = lane >> 4;
  uint32_t b[4][4];
#pragma unroll
  for (int np = 0; np < 4; ++np) ldsm_x4_t(base + (uint32_t)(((2 * np + m) ^ x) << 4), b[np]);
#pragma unroll
  for (int np = 0; np < 4; ++np) {
    mma_bf16(acc[2 * np], A, b[np][0], b[np][1]);
    mma_bf16(acc[2 * np + 1], A, b[np][2], b[np][3]);
    mma_bf16(acc[2 * np], Alo, b[np][0], b[np][1]);
    mma_bf16(acc[2 * np + 1], Alo, b[np][2], b[np][3]);
  }
}

// POW2: the ring's rows are a power of two (slots by a mask).
template <bool POW2>
__global__ void __launch_bounds__(kFastM, 4) k_fwd_tc(const __grid_constant__ TcFwdArgs a) {
  constexpr int M = kFastM;
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  const int RB = a.ring_rows, st = a.sc_stride;
  const Ring ring = make_ring(smem_u32(smem), RB);
  const Ring sinkr = make_ring(ring.base + (uint32_t)RB * 128u, 16);   // own swizzle atoms
  float* sc = reinterpret_cast<float*>(smem + (size_t)RB * 128 + 2048);
  float* inv_l = sc + (size_t)M * st;
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_kind[SA_MAX_OFFSETS];
  __shared__ uint64_t bar;

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int T = a.T, W = a.W, S = a.S, n_off = a.n_off;
  const int i0 = tile * M;
  const int t = threadIdx.x, warp = t >> 5, lane = t & 31, g = lane >> 2, tq = lane & 3;
  const size_t ub = (size_t)unit * T * kD;

  if (t == 0) { mbar_init(&bar, 1); fence_barrier_init(); }
  int bad = 0;
  if (t < n_off) {
    const OffGeo og = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    sg[t] = og;
    bad = !og.ok;
    const int near = og.ok && (og.lo + (og.w != 0.f ? 1 : 0) <= W - 1);
    const int dead = i0 + M - 1 - og.c < 0;        // no query of the tile has it yet
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

  uint32_t aq[2][4][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) q_frags(a, a.q + ub, i0 + 32 * warp + 16 * mt, lane, aq[mt]);

  const int win_lo = floor16(i0 - W + 1);

  // ---------------- pass 1: scores ----------------
  stage_tiles<POW2>(stg, ring, &a.tmK, unit, win_lo, i0 + M);
  if (S > 0) stage_tiles<true>(stg, sinkr, &a.tmK, unit, 0, 16);
  if (stage_commit_wait(stg)) { stage_drain(stg); return; }
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int qb = i0 + 32 * warp + 16 * mt, ql = 32 * warp + 16 * mt;
    const int kr0 = floor16(qb - W + 1);
    const int n_nt = (qb + 16 - kr0) >> 3;
    for (int nt = 0; nt < n_nt; nt += 2) {      // n_nt is even
      uint32_t b0[2][4], b1[2][4];
      qk_load<POW2>(ring, kr0 + 8 * nt, lane, b0);
      qk_load<POW2>(ring, kr0 + 8 * nt + 8, lane, b1);
      float c[2][4] = {{0.f, 0.f, 0.f, 0.f}, {0.f, 0.f, 0.f, 0.f}};
      qk_mma(aq[mt], b0, c[0]);
      qk_mma(aq[mt], b1, c[1]);
#pragma unroll
      for (int j = 0; j < 2; ++j)
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const int r = g + 8 * (e >> 1);
          const int lag = qb + r - (kr0 + 8 * (nt + j) + 2 * tq + (e & 1));
          if (lag >= 0 && lag < W) sc[(ql + r) * st + lag] = kKeyUnstage * c[j][e];
        }
    }
    for (int nt = 0; nt < ((S + 7) >> 3); ++nt) {
      float c[4] = {0.f, 0.f, 0.f, 0.f};
      uint32_t b[2][4];
      qk_load<true>(sinkr, 8 * nt, lane, b);
      qk_mma(aq[mt], b, c);
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const int r = g + 8 * (e >> 1), s = 8 * nt + 2 * tq + (e & 1);
        if (s < S) sc[(ql + r) * st + W + s] = kKeyUnstage * c[e];
      }
    }
  }
  // far offsets, staged in batches; a far member reads rows
  // [i0 - lo - 1, i0 + M - lo + 7)
  {
    int low = win_lo;
    int kk = next_far(s_kind, -1, n_off);
    while (kk < n_off) {
      const int hi = ceil8(i0 + M - sg[kk].lo + 7);
      int last = kk, nx = next_far(s_kind, kk, n_off);
      while (nx < n_off && hi - floor8(i0 - sg[nx].lo - 1) <= RB) {
        last = nx;
        nx = next_far(s_kind, nx, n_off);
      }
      const int lo_row = floor8(i0 - sg[last].lo - 1);
      if (lo_row < low) {
        __syncthreads();
        stage_tiles<POW2>(stg, ring, &a.tmK, unit, lo_row, min(hi, low));
        if (stage_commit_wait(stg)) { stage_drain(stg); return; }
        low = lo_row;
      }
      for (int m = kk; m < nx; m = next_far(s_kind, m, n_off)) {
        const OffGeo og = sg[m];
        const bool two = og.w != 0.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int qb = i0 + 32 * warp + 16 * mt, ql = 32 * warp + 16 * mt;
          const int rb = qb - og.lo - (two ? 1 : 0);
          // three n tiles (24 rows) when w != 0, two when w == 0; loads
          // first, then the accumulator chains interleaved
          uint32_t b[3][2][4];
          float cc[3][4];
#pragma unroll
          for (int nt = 0; nt < 3; ++nt)
#pragma unroll
            for (int e = 0; e < 4; ++e) cc[nt][e] = 0.f;
          if (two) {
#pragma unroll
            for (int nt = 0; nt < 3; ++nt) qk_load<POW2>(ring, rb + 8 * nt, lane, b[nt]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
              for (int nt = 0; nt < 3; ++nt)
                mma_f16(cc[nt], aq[mt][ks], b[nt][ks >> 1][2 * (ks & 1)],
                        b[nt][ks >> 1][2 * (ks & 1) + 1]);
          } else {                               // w == 0: row a only, two n tiles
#pragma unroll
            for (int nt = 0; nt < 2; ++nt) qk_load<POW2>(ring, rb + 8 * nt, lane, b[nt]);
#pragma unroll
            for (int ks = 0; ks < 4; ++ks)
#pragma unroll
              for (int nt = 0; nt < 2; ++nt)
                mma_f16(cc[nt], aq[mt][ks], b[nt][ks >> 1][2 * (ks & 1)],
                        b[nt][ks >> 1][2 * (ks & 1) + 1]);
          }
          const float (&c0)[4] = cc[0];
          const float (&c1)[4] = cc[1];
          const float (&c2)[4] = cc[2];
          // query r needs column r (two: row b) and column r + 1 (row a);
          // rows g and g + 8 of this lane's row group
          const int odd = g & 1;
          const int src_d = 4 * g + (g >> 1);                     // holds column g
          const int src_n = g == 7 ? 28 : 4 * g + ((g + 1) >> 1);   // holds column g + 1
          const float cd_lo = odd ? c0[1] : c0[0], cd_hi = odd ? c1[3] : c1[2];
          const float cn_lo = g == 7 ? c1[0] : (odd ? c0[0] : c0[1]);
          const float cn_hi = g == 7 ? c2[2] : (odd ? c1[2] : c1[3]);
          const float d_lo = __shfl_sync(0xffffffffu, cd_lo, src_d);
          const float d_hi = __shfl_sync(0xffffffffu, cd_hi, src_d);
          const float n_lo = __shfl_sync(0xffffffffu, cn_lo, src_n);
          const float n_hi = __shfl_sync(0xffffffffu, cn_hi, src_n);
          if (tq == 0) {
            const float s_lo = two ? og.wa * n_lo + og.w * d_lo : d_lo;
            const float s_hi = two ? og.wa * n_hi + og.w * d_hi : d_hi;
            sc[(ql + g) * st + W + S + m] = kKeyUnstage * s_lo;
            sc[(ql + g + 8) * st + W + S + m] = kKeyUnstage * s_hi;
          }
        }
      }
      kk = nx;
    }
  }
  __syncthreads();

  // ---------------- softmax (owner thread of each query) ----------------
  {
    const int i = i0 + t;
    float* my = sc + (size_t)t * st;
    if (i < T) {
      // near offsets from two window scores; every offset member gets the
      // query's log-prior (0 without one)
      const float prior = a.beta ? __ldg(a.beta + (size_t)unit * T + i) : 0.f;
      for (int k = 0; k < n_off; ++k) {
        if (s_kind[k] == kNear) {
          const OffGeo og = sg[k];
          float sv = og.wa * my[og.lo];
          if (og.w != 0.f) sv += og.w * my[og.lo + 1];
          my[W + S + k] = sv + prior;
        } else if (s_kind[k] == kFar) {
          my[W + S + k] += prior;
        }
      }
      float mx = -INFINITY;
      for (int d = 0; d < W; ++d)
        if (i - d >= 0) mx = fmaxf(mx, my[d]);
      for (int s = 0; s < S; ++s)
        if (s <= i) mx = fmaxf(mx, my[W + s]);
      for (int k = 0; k < n_off; ++k)
        if (s_kind[k] != kDead && i - sg[k].c >= 0) mx = fmaxf(mx, my[W + S + k]);
      float l = 0.f;
      for (int d = 0; d < W; ++d) {
        const float e = (i - d >= 0) ? __expf(my[d] - mx) : 0.f;
        my[d] = e; l += e;
      }
      for (int s = 0; s < S; ++s) {
        const float e = (s <= i) ? __expf(my[W + s] - mx) : 0.f;
        my[W + s] = e; l += e;
      }
      for (int k = 0; k < n_off; ++k) {
        const OffGeo og = sg[k];
        const float e =
            (s_kind[k] != kDead && i - og.c >= 0) ? __expf(my[W + S + k] - mx) : 0.f;
        my[W + S + k] = e; l += e;
        if (s_kind[k] == kNear) {              // fold into the two window weights
          my[og.lo] += og.wa * e;
          if (og.w != 0.f) my[og.lo + 1] += og.w * e;
        }
      }
      inv_l[t] = 1.f / l;
      if (a.lse) a.lse[(size_t)unit * T + i] = mx + __logf(l);
    } else {
      for (int d = 0; d < W + S + n_off; ++d) my[d] = 0.f;
      inv_l[t] = 0.f;
    }
  }
  __syncthreads();

  // ---------------- pass 2: P . V ----------------
  // Bidiagonal A fragments (far offsets): in a row block, query g puts its
  // column-g weight and its column-(g+1) weight; register 0 of lane (g, tq)
  // covers columns 2tq, 2tq+1, register 2 columns 2tq+8, 2tq+9.  Code 1: both
  // columns (g even, tq = g/2); code 2: column g in the high half (g odd,
  // tq = (g-1)/2); code 3: column g+1 in the low half (g odd, tq = (g+1)/2);
  // register 2 carries column 8 for g = 7, tq = 0.  The same codes hold for
  // rows g + 8 in register 3 (the column-16 entry of query 15 goes to the
  // 8-row k step).
  const bool bd_lo_c1 = !(g & 1) && tq == (g >> 1);
  const bool bd_c2 = (g & 1) && tq == (g >> 1);
  const bool bd_c3 = (g & 1) && g < 7 && tq == ((g + 1) >> 1);
  const bool bd_a2 = g == 7 && tq == 0;
  stage_tiles<POW2>(stg, ring, &a.tmV, unit, win_lo, i0 + M);
  if (S > 0) stage_tiles<true>(stg, sinkr, &a.tmV, unit, 0, 16);
  if (stage_commit_wait(stg)) { stage_drain(stg); return; }
  float acc[2][8][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int nt = 0; nt < 8; ++nt)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][nt][e] = 0.f;
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int qb = i0 + 32 * warp + 16 * mt, ql = 32 * warp + 16 * mt;
    const float* e_lo = sc + (size_t)(ql + g) * st;
    const float* e_hi = sc + (size_t)(ql + g + 8) * st;
    const int kr0 = floor16(qb - W + 1);
    const int n_k = (qb + 16 - kr0) >> 4;
    for (int ks = 0; ks < n_k; ++ks) {
      const int kb = kr0 + 16 * ks;
      uint32_t A[4], Al[4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const float* er = h ? e_hi : e_lo;
          const int lag0 = qb + g + 8 * h - (kb + 2 * tq + 8 * p);   // lag of the first column
          const float v0 = (lag0 >= 0 && lag0 < W) ? er[lag0] : 0.f;
          const float v1 = (lag0 - 1 >= 0 && lag0 - 1 < W) ? er[lag0 - 1] : 0.f;
          split_bf16x2(v0, v1, A[h + 2 * p], Al[h + 2 * p]);
        }
      pv_k16<POW2>(ring, kb, lane, A, Al, acc[mt]);
    }
    if (S > 0) {
      uint32_t A[4], Al[4];
#pragma unroll
      for (int h = 0; h < 2; ++h)
#pragma unroll
        for (int p = 0; p < 2; ++p) {
          const float* er = h ? e_hi : e_lo;
          const int s0 = 2 * tq + 8 * p;
          split_bf16x2(s0 < S ? er[W + s0] : 0.f, s0 + 1 < S ? er[W + s0 + 1] : 0.f, A[h + 2 * p],
                       Al[h + 2 * p]);
        }
      pv_k16<true>(sinkr, 0, lane, A, Al, acc[mt]);
    }
  }
  {
    int low = win_lo;
    int kk = next_far(s_kind, -1, n_off);
    while (kk < n_off) {
      const int hi = ceil8(i0 + M - sg[kk].lo + 7);
      int last = kk, nx = next_far(s_kind, kk, n_off);
      while (nx < n_off && hi - floor8(i0 - sg[nx].lo - 1) <= RB) {
        last = nx;
        nx = next_far(s_kind, nx, n_off);
      }
      const int lo_row = floor8(i0 - sg[last].lo - 1);
      if (lo_row < low) {
        __syncthreads();
        stage_tiles<POW2>(stg, ring, &a.tmV, unit, lo_row, min(hi, low));
        if (stage_commit_wait(stg)) { stage_drain(stg); return; }
        low = lo_row;
      }
      for (int m = kk; m < nx; m = next_far(s_kind, m, n_off)) {
        const OffGeo og = sg[m];
        const bool two = og.w != 0.f;
#pragma unroll
        for (int mt = 0; mt < 2; ++mt) {
          const int qb = i0 + 32 * warp + 16 * mt, ql = 32 * warp + 16 * mt;
          const float p_lo = sc[(size_t)(ql + g) * st + W + S + m];
          const float p_hi = sc[(size_t)(ql + g + 8) * st + W + S + m];
          // query r weighs column r by kd (row b, or row a when w == 0) and
          // column r + 1 by ks (row a, when w != 0)
          const float kd = two ? og.w : 1.f, ksu = two ? og.wa : 0.f;
          const float dl = p_lo * kd, sl = p_lo * ksu, dh = p_hi * kd, sh = p_hi * ksu;
          const int kb = qb - og.lo - (two ? 1 : 0);
          uint32_t A[4], Al[4];
          split_bf16x2(bd_lo_c1 ? dl : (bd_c3 ? sl : 0.f), bd_lo_c1 ? sl : (bd_c2 ? dl : 0.f), A[0],
                       Al[0]);
          A[1] = Al[1] = 0u;
          split_bf16x2(bd_a2 ? sl : 0.f, 0.f, A[2], Al[2]);
          split_bf16x2(bd_lo_c1 ? dh : (bd_c3 ? sh : 0.f), bd_lo_c1 ? sh : (bd_c2 ? dh : 0.f), A[3],
                       Al[3]);
          pv_k16<POW2>(ring, kb, lane, A, Al, acc[mt]);
          if (two) {
            // the 17th row (row a of query 15) as an 8-row k step
            uint32_t a1, a1l;
            split_bf16x2(bd_a2 ? sh : 0.f, 0.f, a1, a1l);
            const int row = kb + 16 + (lane & 7);
#pragma unroll
            for (int hh = 0; hh < 2; ++hh) {
              uint32_t b[4];
              ldsm_x4_t(swz_addr<POW2>(ring, row, 4 * hh + (lane >> 3)), b);
#pragma unroll
              for (int i = 0; i < 4; ++i) {
                mma_bf16_k8(acc[mt][4 * hh + i], 0u, a1, b[i]);
                mma_bf16_k8(acc[mt][4 * hh + i], 0u, a1l, b[i]);
              }
            }
          }
        }
      }
      kk = nx;
    }
  }

  // scale by 1 / sum of the weights and store
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int qb = i0 + 32 * warp + 16 * mt, ql = 32 * warp + 16 * mt;
#pragma unroll
    for (int h = 0; h < 2; ++h) {
      const int i = qb + g + 8 * h;
      const float inv = inv_l[ql + g + 8 * h];
      if (i < T) {
        __nv_bfloat16* dst = a.o + ub + (size_t)i * kD + 2 * tq;
#pragma unroll
        for (int nt = 0; nt < 8; ++nt)
          *reinterpret_cast<uint32_t*>(dst + 8 * nt) =
              pack_bf16x2(acc[mt][nt][2 * h] * inv, acc[mt][nt][2 * h + 1] * inv);
      }
    }
  }
}

__device__ unsigned g_fwd_tc_err;   // error bits as listed in sa_stage.cuh

// CTAs of `smem` dynamic bytes that share one SM's 228 KB (1 KB reserved per
// CTA plus about 1 KB of static shared memory), at most the 4 of the
// launch bounds.
int ctas_per_sm(size_t smem) {
  const size_t per = smem + 2048;
  return (int)std::min<size_t>(4, (size_t)(228 * 1024) / per);
}

size_t tc_smem_bytes(const Problem& pb, int rr, int st) {
  return 1024 + (size_t)rr * 128 + 2048 + (size_t)kFastM * st * sizeof(float) +
         kFastM * sizeof(float);
}

// Ring rows: at least the window round (M + W - 1 rows from a 16-aligned
// start, so M + W + 15).  A power of two (slots by a mask) unless a multiple
// of 16 fits more CTAs per SM; that ring then grows while the CTA count
// holds (more far offsets per staging round).  Measured on B200 (B=1 H=16
// T=32768, 4 sinks): W = 64 gains 16 % (3 CTAs per SM instead of 2) and
// W = 128 38 % (2 instead of 1); where the count is the same the
// power-of-two ring is 5-9 % faster than one indexed by a modulo.
int tc_ring_rows(const Problem& pb) {
  const int st = (pb.W + pb.S + pb.n_off) | 1;
  const int need = std::max(kFastM + pb.W + 15, kFastM + 24);
  int p2 = 32;
  while (p2 < need) p2 *= 2;
  int rr = (need + 15) & ~15;
  const int ctas = ctas_per_sm(tc_smem_bytes(pb, rr, st));
  if (ctas_per_sm(tc_smem_bytes(pb, p2, st)) >= ctas) return p2;
  while (rr + 16 <= 512 && ctas_per_sm(tc_smem_bytes(pb, rr + 16, st)) == ctas) rr += 16;
  return rr;
}

}  // namespace

size_t tc_fwd_smem(const Problem& pb, int* ring_rows, int* sc_stride) {
  const int rr = tc_ring_rows(pb);
  const int st = (pb.W + pb.S + pb.n_off) | 1;
  if (ring_rows) *ring_rows = rr;
  if (sc_stride) *sc_stride = st;
  return tc_smem_bytes(pb, rr, st);
}

bool tc_fwd_supported(const Problem& pb) {
  return pb.dtype == SA_DTYPE_BF16 && pb.D == kD && pb.W <= 256 && pb.S <= 16 &&
         tc_fwd_smem(pb, nullptr, nullptr) <= 200 * 1024;
}

// Measured on B200 (B=1 H=16 T=32768 d=64, 4 sinks, alpha = 1 and 1.1234,
// windows 16..128): the CUDA-core forward is faster up to W = 40 (by 3-14 %),
// this one from W = 48 (by 1-8 % at 48..56, 14-26 % at 64..128).  Where its
// shared memory would leave it one CTA per SM while the CUDA-core forward
// keeps two (W >= 160 with 15 offsets), it is not taken.
bool tc_fwd_preferred(const Problem& pb) {
  if (!tc_fwd_supported(pb) || pb.W < 48) return false;
  const int tc = ctas_per_sm(tc_fwd_smem(pb, nullptr, nullptr));
  const int cc = fast_fwd_supported(pb) ? ctas_per_sm(fast_fwd_smem(pb, nullptr, nullptr)) : 0;
  return !(tc == 1 && cc >= 2);
}

cudaError_t launch_fwd_tc(const Problem& pb, const FwdPtrs& p, void* keys_ws, cudaStream_t st,
                          int* launches) {
  TcFwdArgs a;
  memset(&a, 0, sizeof(a));
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = (pb.T + kFastM - 1) / kFastM;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  std::sort(a.f, a.f + pb.n_off);
  const size_t smem = tc_fwd_smem(pb, &a.ring_rows, &a.sc_stride);
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.alpha = p.alpha; a.beta = p.beta; a.rope = p.rope;
  a.o = reinterpret_cast<__nv_bfloat16*>(p.o); a.lse = p.lse;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&a.err), g_fwd_tc_err);
  const WaitCfg wc = wait_cfg();
  a.wait_limit = wc.limit;
  a.stall = wc.stall;
  if (e != cudaSuccess) return e;
  if ((e = make_rows_map(&a.tmK, keys_ws, pb.T, pb.units())) != cudaSuccess) return e;
  if ((e = make_rows_map(&a.tmV, p.v, pb.T, pb.units())) != cudaSuccess) return e;
  if ((e = launch_rope_rows(p.k, p.rope, pb.T, pb.units() * pb.T, kKeyStage, keys_ws, st,
                            "rope_keys")) != cudaSuccess)
    return e;
  const bool pow2 = (a.ring_rows & (a.ring_rows - 1)) == 0;
  if ((e = cudaFuncSetAttribute(pow2 ? k_fwd_tc<true> : k_fwd_tc<false>,
                                cudaFuncAttributeMaxDynamicSharedMemorySize, (int)smem)) !=
      cudaSuccess)
    return e;
  const unsigned grid = (unsigned)((long long)pb.units() * a.n_tiles);
  trace_mark("fwd_tc", st, true);
  if (pow2) k_fwd_tc<true><<<grid, kFastM, smem, st>>>(a);
  else k_fwd_tc<false><<<grid, kFastM, smem, st>>>(a);
  trace_mark("fwd_tc", st, false);
  e = cudaGetLastError();
  if (e == cudaSuccess) *launches += 2;
  return e;
}

cudaError_t fast_fwd_tc_read_error(unsigned* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_fwd_tc_err, sizeof(unsigned));
  if (e != cudaSuccess || !clear || *out == 0) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_fwd_tc_err, &zero, sizeof(unsigned));
}

}  // namespace sa
