// Forward on the fifth-generation tensor cores (tcgen05, accumulators in
// tensor memory) for bf16 inputs with head dim 64: the dense part of each
// query's member set (the window band and the sinks) as two tile GEMMs, the
// Fibonacci offset members on the CUDA cores.  The operation is the one of
// "Depth-Staggered Fibonacci Spacing for Sparse Attention", Methodology:
// one softmax over window, sinks and interpolated offset keys, the same
// interpolation weights on the values.
//
// One CTA owns 128 consecutive queries of one (layer, batch, head); thread t
// owns query i = i0 + t, which is also row t of both accumulators in tensor
// memory.  Per tile:
//  1. Tensor copies (128-byte swizzle) stage the band of rotated keys
//     K^ = fp16(RoPE(K) / 256) over rows [kb0, i0 + 128), kb0 = i0 - 16
//     ceil((W - 1) / 16), followed by 16 sink rows when S > 0, and the same
//     rows of V.  Each thread writes its query's RoPE(q) * scale, rounded to
//     fp16, as row t of the A operand.
//  2. One thread issues S = Q^ . K^band^T (M = 128, N = band + sinks, K = 64)
//     into tensor memory.  Meanwhile each thread scores its offset members
//     (rows i - lo and i - lo - 1, interpolated) with fp32 dot products, from
//     the band when both rows lie in it and otherwise from rows staged one
//     round at a time.
//  3. Softmax per thread: the band entries of row t whose lag i - key lies in
//     [0, W) (and the sinks s <= i) from tensor memory, the offset scores from
//     shared memory.  The unnormalised weights of the band and the sinks are
//     written, in fp16, as row t of the A operand of the second GEMM.
//  4. One thread issues O = P . V^band (N = 64) into tensor memory, V staged
//     as fp16(V / 256) (converted in place after its copy); each thread adds
//     its offset members' weighted value rows on the CUDA cores, reads its O
//     row back and stores O_i and LSE_i.
// Precision: products of fp16 operands are exact in the fp32 accumulators;
// the rounding left is that of the staged operands (K^ and q^ to fp16 as in
// the other staged kernels, the weights e^(s - max) in [0, 1] to fp16,
// 2^-11 relative).  Range: |RoPE(K)|, |V| below 256 * 65504 and |RoPE(q) *
// scale| below 65504, else the error word's range bit is set.
#include <algorithm>
#include <cstring>

#include "sa_tc.cuh"
#include "sa_umma.cuh"

namespace sa {

namespace {

using namespace fast;
using namespace stage;

constexpr int kM = kFastM;            // queries per CTA = threads per CTA
constexpr int kFarRows = 136;         // rows of one far staging round (17 boxes of 8)
constexpr int kMinSmem = 80 * 1024;   // at most two CTAs per SM: 2 x 256 TMEM columns

struct UmmaFwdArgs {
  CUtensorMap tmK;                     // rotated keys / 256, fp16 [units][T][64]
  CUtensorMap tmV;                     // V, bf16 [units][T][64]
  int B, H, T, W, n_off, S, n_tiles;
  int NB, N, tmem_cols, sc_stride;     // band rows, GEMM columns, TMEM columns
  unsigned off_kb, off_far, off_vb, off_sc;   // byte offsets in the aligned shared memory
  float scale;
  int f[SA_MAX_OFFSETS];               // ascending
  const __nv_bfloat16* q;
  const float* alpha; const float2* rope;
  __nv_bfloat16* o; float* lse;
  unsigned* err;
  long long wait_limit;                // bounded waits: SM clocks (0: the default)
  int stall;                           // failure-path test: the key band expects 16 more bytes
  const float* beta;                   // log-prior on offset members [units][T], or nullptr
};

enum : int { kInband = 0, kFarOff = 1, kDeadOff = 2 };
enum : int { kBarK = 0, kBarV = 1, kBarFar = 2, kBarS = 3, kBarO = 4, kNumBars = 5 };

__device__ __forceinline__ int next_of(const int* s_kind, int k, int n_off, int kind) {
  ++k;
  while (k < n_off && s_kind[k] != kind) ++k;
  return k;
}

// Byte offset of 16-byte chunk c of the row at position p of a buffer filled
// by 8-row tensor copies with 128-byte swizzling (1024-aligned boxes).
__device__ __forceinline__ int swz(int p, int c) { return p * 128 + ((c ^ (p & 7)) << 4); }

// q . (fp16 row at position p)
__device__ __forceinline__ float dot_row(const float (&q)[64], const unsigned char* buf, int p) {
  float2 a0 = make_float2(0.f, 0.f), a1 = make_float2(0.f, 0.f);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float y[8];
    unpack8_h(*reinterpret_cast<const uint4*>(buf + swz(p, c)), y);
    a0 = __ffma2_rn(make_float2(q[8 * c], q[8 * c + 1]), make_float2(y[0], y[1]), a0);
    a1 = __ffma2_rn(make_float2(q[8 * c + 2], q[8 * c + 3]), make_float2(y[2], y[3]), a1);
    a0 = __ffma2_rn(make_float2(q[8 * c + 4], q[8 * c + 5]), make_float2(y[4], y[5]), a0);
    a1 = __ffma2_rn(make_float2(q[8 * c + 6], q[8 * c + 7]), make_float2(y[6], y[7]), a1);
  }
  return (a0.x + a0.y) + (a1.x + a1.y);
}

// o += w * (16-bit row at position p: fp16 when F16, else bf16)
template <bool F16>
__device__ __forceinline__ void axpy_row(float (&o)[64], float w, const unsigned char* buf, int p) {
  const float2 ww = make_float2(w, w);
#pragma unroll
  for (int c = 0; c < 8; ++c) {
    float y[8];
    unpack8x<F16>(*reinterpret_cast<const uint4*>(buf + swz(p, c)), y);
#pragma unroll
    for (int e = 0; e < 8; e += 2) {
      const float2 r = __ffma2_rn(ww, make_float2(y[e], y[e + 1]),
                                  make_float2(o[8 * c + e], o[8 * c + e + 1]));
      o[8 * c + e] = r.x;
      o[8 * c + e + 1] = r.y;
    }
  }
}

// Bounded wait (every thread polls); true when the phase completed.
__device__ __forceinline__ bool wait_bar(uint64_t* bar, uint32_t parity, long long limit) {
  const long long t0 = clock64();
  while (!mbar_try_wait(bar, parity))
    if (clock64() - t0 > limit) return false;
  return true;
}

// Staging and MMA bookkeeping, identical in every thread.
struct Sync {
  uint64_t* bars;
  unsigned pend;        // bit b: barrier b has a phase armed and not yet waited for
  uint32_t far_phase;
  long long limit;
  unsigned* err;
};

// Wait for barrier b's armed phase; false in every thread when any gave up.
__device__ __forceinline__ bool sync_wait(Sync& s, int b) {
  const uint32_t parity = b == kBarFar ? s.far_phase : 0u;
  const bool ok = wait_bar(s.bars + b, parity, s.limit);
  const int bad = __syncthreads_or(!ok);
  if (bad) {
    if (threadIdx.x == 0) atomicOr(s.err, kErrWait);
    return false;
  }
  s.pend &= ~(1u << b);
  if (b == kBarFar) s.far_phase ^= 1u;
  return true;
}

// One far staging round of `map` rows [lo_row, lo_row + 8 nbox) into the far
// buffer (thread 0 issues; completes on the far barrier).
__device__ __forceinline__ void far_issue(Sync& s, uint32_t far_u32, const CUtensorMap* map,
                                          int unit, int lo_row, int nbox) {
  if (threadIdx.x == 0) {
    mbar_expect_tx(s.bars + kBarFar, (uint32_t)nbox * 1024u);
    for (int b = 0; b < nbox; ++b)
      tc::tma_rows8(far_u32 + (uint32_t)b * 1024u, map, lo_row + 8 * b, unit, s.bars + kBarFar);
    mbar_arrive(s.bars + kBarFar);
  }
  s.pend |= 1u << kBarFar;
}

// Consecutive far members [kk, nx) whose rows [i0 - lo - 1, i0 + M - lo) fit
// one round; their rows start at lo_row.
__device__ __forceinline__ void far_batch(const OffGeo* sg, const int* s_kind, int n_off, int kk,
                                          int i0, int& nx, int& lo_row, int& nbox) {
  const int hi = i0 + kM - sg[kk].lo;
  int last = kk;
  nx = next_of(s_kind, kk, n_off, kFarOff);
  while (nx < n_off && hi - (i0 - sg[nx].lo - 1) <= kFarRows) {
    last = nx;
    nx = next_of(s_kind, nx, n_off, kFarOff);
  }
  lo_row = i0 - sg[last].lo - 1;
  nbox = (hi - lo_row + 7) >> 3;
}

// The tile's work after the tensor memory is allocated; false when a bounded
// wait gave up (the caller drains what is in flight).
__device__ __forceinline__ bool fwd_tile(const UmmaFwdArgs& a, Sync& sy, unsigned char* smem,
                                         const OffGeo* sg, const int* s_kind, uint32_t tmem,
                                         int unit, int i0) {
  const int T = a.T, W = a.W, S = a.S, n_off = a.n_off, NB = a.NB, N = a.N;
  const int kb0 = i0 + kM - NB, C = NB - kM;
  const int t = threadIdx.x, warp = t >> 5;
  const int i = i0 + t;
  const bool live = i < T;
  const size_t ub = (size_t)unit * T * kD;
  const uint32_t s_u32 = smem_u32(smem);
  unsigned char* kb = smem + a.off_kb;
  unsigned char* far = smem + a.off_far;
  unsigned char* vb = smem + a.off_vb;
  float* my = reinterpret_cast<float*>(smem + a.off_sc) + (size_t)t * a.sc_stride;

  // ---- 1. band copies, and this query's row of the A operand --------------
  if (t == 0) {
    const uint32_t bytes = (uint32_t)N * 128u;
    for (int m = 0; m < 2; ++m) {
      uint64_t* bar = sy.bars + (m ? kBarV : kBarK);
      const CUtensorMap* map = m ? &a.tmV : &a.tmK;
      const uint32_t dst = s_u32 + (m ? a.off_vb : a.off_kb);
      mbar_expect_tx(bar, bytes + (!m && a.stall ? 16u : 0u));
      for (int r = 0; r < NB; r += 8) tc::tma_rows8(dst + (uint32_t)r * 128u, map, kb0 + r, unit, bar);
      if (N > NB)
        for (int r = 0; r < 16; r += 8)
          tc::tma_rows8(dst + (uint32_t)(NB + r) * 128u, map, r, unit, bar);
      mbar_arrive(bar);
    }
  }
  sy.pend |= (1u << kBarK) | (1u << kBarV);

  float q[64];
  {
    bool over = false;
    const uint4* qr = reinterpret_cast<const uint4*>(a.q + ub + (size_t)min(i, T - 1) * kD);
    const float4* cs = reinterpret_cast<const float4*>(a.rope + (size_t)min(i, T - 1) * 32);
#pragma unroll
    for (int c = 0; c < 4; ++c) {            // dims 8c.. (x) and their partners 8c + 32.. (y)
      float x[8], y[8];
      unpack8(__ldg(qr + c), x);
      unpack8(__ldg(qr + c + 4), y);
#pragma unroll
      for (int e = 0; e < 8; e += 2) {
        const float4 r = __ldg(cs + (8 * c + e) / 2);      // (cos, sin) of pairs 8c+e, 8c+e+1
        q[8 * c + e] = (x[e] * r.x - y[e] * r.y) * a.scale;
        q[8 * c + e + 32] = (y[e] * r.x + x[e] * r.y) * a.scale;
        q[8 * c + e + 1] = (x[e + 1] * r.z - y[e + 1] * r.w) * a.scale;
        q[8 * c + e + 33] = (y[e + 1] * r.z + x[e + 1] * r.w) * a.scale;
      }
    }
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      float* qc = q + 8 * c;
      if (!live) {
#pragma unroll
        for (int e = 0; e < 8; ++e) qc[e] = 0.f;
      }
      over |= half_overflow8(qc);
      const uint4 u = pack8_h(qc);
      *reinterpret_cast<uint4*>(smem + swz(t, c)) = u;    // row t of the A operand
      unpack8_h(u, qc);                                    // the fp16 values the GEMM sees
    }
    if (over) atomicOr(a.err, kErrRange);
  }
  fence_proxy_async();

  // ---- 2. S = Q^ . K^band^T, and the offset scores -------------------------
  if (!sync_wait(sy, kBarK)) return false;     // (its CTA barrier also orders the A rows)
  if (t == 0) {
    umma::fence_after_sync();
    const uint32_t id = umma::idesc_f16(kM, N, false);
#pragma unroll
    for (int s = 0; s < 4; ++s)
      umma::mma_f16(tmem,
                    umma::sdesc(s_u32 + 32u * s, 16u, 1024u, umma::kSwizzle128),
                    umma::sdesc(s_u32 + a.off_kb + 32u * s, 16u, 1024u, umma::kSwizzle128), id,
                    s > 0);
    umma::commit(sy.bars + kBarS);
  }
  sy.pend |= 1u << kBarS;

  const float prior = (a.beta && live) ? __ldg(a.beta + (size_t)unit * T + i) : 0.f;
  float m_off = -INFINITY;
  for (int k = next_of(s_kind, -1, n_off, kInband); k < n_off;
       k = next_of(s_kind, k, n_off, kInband)) {
    const OffGeo g = sg[k];
    if (live && i - g.c >= 0) {
      const int p = i - g.lo - kb0;
      dbg_check(a.err, p >= (g.w != 0.f ? 1 : 0) && p < NB);
      float d = g.wa * dot_row(q, kb, p);
      if (g.w != 0.f) d += g.w * dot_row(q, kb, p - 1);
      my[k] = d * kKeyUnstage + prior;
      m_off = fmaxf(m_off, my[k]);
    }
  }
  for (int kk = next_of(s_kind, -1, n_off, kFarOff); kk < n_off;) {
    int nx, lo_row, nbox;
    far_batch(sg, s_kind, n_off, kk, i0, nx, lo_row, nbox);
    far_issue(sy, s_u32 + a.off_far, &a.tmK, unit, lo_row, nbox);
    if (!sync_wait(sy, kBarFar)) return false;
    for (int k = kk; k < nx; k = next_of(s_kind, k, n_off, kFarOff)) {
      const OffGeo g = sg[k];
      if (live && i - g.c >= 0) {
        const int p = i - g.lo - lo_row;
        dbg_check(a.err, p >= 1 && p < 8 * nbox);
        float d = g.wa * dot_row(q, far, p);
        if (g.w != 0.f) d += g.w * dot_row(q, far, p - 1);
        my[k] = d * kKeyUnstage + prior;
        m_off = fmaxf(m_off, my[k]);
      }
    }
    __syncthreads();                        // every thread is done with the far buffer
    kk = nx;
  }

  // V band -> fp16(V / 256), in place (the operand type of the second GEMM)
  if (!sync_wait(sy, kBarV)) return false;
  {
    bool over = false;
    for (int e = t; e < N * kChunks; e += kM) {
      uint4* p = reinterpret_cast<uint4*>(vb) + e;
      float x[8];
      unpack8(*p, x);
#pragma unroll
      for (int h = 0; h < 8; ++h) x[h] *= kKeyStage;
      over |= half_overflow8(x);
      *p = pack8_h(x);
    }
    if (over) atomicOr(a.err, kErrRange);
  }
  fence_proxy_async();

  // ---- 3. softmax ----------------------------------------------------------
  if (!sync_wait(sy, kBarS)) return false;
  umma::fence_after_sync();
  const uint32_t trow = tmem + ((uint32_t)(32 * warp) << 16);
  // band columns this warp's rows can use: lags [0, W) of queries 32w .. 32w+31
  const int jw0 = (32 * warp + C - W + 1) & ~15, jw1 = 32 * warp + C + 32;
  float mx = m_off;
  for (int j0 = jw0; j0 < jw1; j0 += 16) {
    float v[16];
    umma::ld16(trow + (uint32_t)j0, v);
#pragma unroll
    for (int e = 0; e < 16; ++e) {
      const int d = t + C - (j0 + e);
      if ((unsigned)d < (unsigned)W && kb0 + j0 + e >= 0) mx = fmaxf(mx, v[e] * kKeyUnstage);
    }
  }
  if (S > 0) {
    float v[16];
    umma::ld16(trow + (uint32_t)NB, v);
#pragma unroll
    for (int s = 0; s < 16; ++s)
      if (s < S && s <= i) mx = fmaxf(mx, v[s] * kKeyUnstage);
  }
  __syncthreads();          // P overwrites the q^ rows, the key band and the far buffer
  float l = 0.f;
  {
    unsigned char* prow = smem + (t >> 3) * 128 + (t & 7) * 16;   // row t, core-matrix layout
    const uint4 zero = make_uint4(0u, 0u, 0u, 0u);
    for (int cb = 0; cb < NB / 8; ++cb)
      if (cb < jw0 / 8 || cb >= jw1 / 8) *reinterpret_cast<uint4*>(prow + cb * 2048) = zero;
    for (int j0 = jw0; j0 < jw1; j0 += 16) {
      float v[16];
      umma::ld16(trow + (uint32_t)j0, v);
#pragma unroll
      for (int e = 0; e < 16; ++e) {
        const int d = t + C - (j0 + e);
        const bool ok = live && (unsigned)d < (unsigned)W && kb0 + j0 + e >= 0;
        v[e] = ok ? __expf(v[e] * kKeyUnstage - mx) : 0.f;
        l += v[e];
      }
      *reinterpret_cast<uint4*>(prow + (j0 / 8) * 2048) = pack8_h(v);
      *reinterpret_cast<uint4*>(prow + (j0 / 8 + 1) * 2048) = pack8_h(v + 8);
    }
    if (S > 0) {
      float v[16];
      umma::ld16(trow + (uint32_t)NB, v);
#pragma unroll
      for (int s = 0; s < 16; ++s) {
        v[s] = (live && s < S && s <= i) ? __expf(v[s] * kKeyUnstage - mx) : 0.f;
        l += v[s];
      }
      *reinterpret_cast<uint4*>(prow + (NB / 8) * 2048) = pack8_h(v);
      *reinterpret_cast<uint4*>(prow + (NB / 8 + 1) * 2048) = pack8_h(v + 8);
    }
  }
  for (int k = 0; k < n_off; ++k) {
    const OffGeo g = sg[k];
    if (live && s_kind[k] != kDeadOff && i - g.c >= 0) {
      my[k] = __expf(my[k] - mx);
      l += my[k];
    }
  }
  fence_proxy_async();
  umma::fence_before_sync();
  __syncthreads();

  // ---- 4. O = P . V^band, and the offset members' values -------------------
  if (t == 0) {
    umma::fence_after_sync();
    const uint32_t id = umma::idesc_f16(kM, kD, true);
    for (int s = 0; s < N / 16; ++s)
      umma::mma_f16(tmem,
                    umma::sdesc(s_u32 + 4096u * s, 2048u, 128u, umma::kSwizzleNone),
                    umma::sdesc(s_u32 + a.off_vb + 2048u * s, 16u, 1024u, umma::kSwizzle128), id,
                    s > 0);
    umma::commit(sy.bars + kBarO);
  }
  sy.pend |= 1u << kBarO;

  float o[64];
#pragma unroll
  for (int h = 0; h < 64; ++h) o[h] = 0.f;
  for (int k = next_of(s_kind, -1, n_off, kInband); k < n_off;
       k = next_of(s_kind, k, n_off, kInband)) {
    const OffGeo g = sg[k];
    if (live && i - g.c >= 0) {
      const int p = i - g.lo - kb0;
      const float e = my[k] * kKeyUnstage;     // the band holds V / 256
      axpy_row<true>(o, e * g.wa, vb, p);
      if (g.w != 0.f) axpy_row<true>(o, e * g.w, vb, p - 1);
    }
  }
  if (!sync_wait(sy, kBarO)) return false;    // the far buffer lies under P
  for (int kk = next_of(s_kind, -1, n_off, kFarOff); kk < n_off;) {
    int nx, lo_row, nbox;
    far_batch(sg, s_kind, n_off, kk, i0, nx, lo_row, nbox);
    far_issue(sy, s_u32 + a.off_far, &a.tmV, unit, lo_row, nbox);
    if (!sync_wait(sy, kBarFar)) return false;
    for (int k = kk; k < nx; k = next_of(s_kind, k, n_off, kFarOff)) {
      const OffGeo g = sg[k];
      if (live && i - g.c >= 0) {
        const int p = i - g.lo - lo_row;
        dbg_check(a.err, p >= 1 && p < 8 * nbox);
        axpy_row<false>(o, my[k] * g.wa, far, p);
        if (g.w != 0.f) axpy_row<false>(o, my[k] * g.w, far, p - 1);
      }
    }
    __syncthreads();
    kk = nx;
  }

  umma::fence_after_sync();
  const float inv = live ? 1.f / l : 0.f;
  __nv_bfloat16* dst = a.o + ub + (size_t)i * kD;
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    float v[16];
    umma::ld16(trow + (uint32_t)(16 * c), v);
#pragma unroll
    for (int e = 0; e < 16; ++e) v[e] = (v[e] * kKeyUnstage + o[16 * c + e]) * inv;
    if (live) {
      reinterpret_cast<uint4*>(dst)[2 * c] = pack8(v);
      reinterpret_cast<uint4*>(dst)[2 * c + 1] = pack8(v + 8);
    }
  }
  if (live && a.lse) a.lse[(size_t)unit * T + i] = mx + __logf(l);
  return true;
}

__global__ void __launch_bounds__(kM, 2) k_fwd_umma(const __grid_constant__ UmmaFwdArgs a) {
  extern __shared__ unsigned char smem_raw[];
  unsigned char* smem = smem_raw + ((1024u - (smem_u32(smem_raw) & 1023u)) & 1023u);
  __shared__ OffGeo sg[SA_MAX_OFFSETS];
  __shared__ int s_kind[SA_MAX_OFFSETS];
  __shared__ __align__(8) uint64_t bars[kNumBars];
  __shared__ uint32_t s_tmem;

  const int unit = blockIdx.x / a.n_tiles, tile = blockIdx.x % a.n_tiles;
  const int layer = unit / (a.B * a.H);
  const int T = a.T, n_off = a.n_off;
  const int i0 = tile * kM;
  const int t = threadIdx.x, warp = t >> 5;
  const int C = a.NB - kM;

  if (t == 0) {
    for (int b = 0; b < kNumBars; ++b) mbar_init(&bars[b], 1);
    fence_barrier_init();
  }
  int bad = 0;
  if (t < n_off) {
    const OffGeo g = offset_geometry(__ldg(a.alpha + layer), a.f[t]);
    sg[t] = g;
    bad = !g.ok;
    const int dead = i0 + kM - 1 - g.c < 0;          // no query of the tile has it yet
    const int inband = g.lo + (g.w != 0.f ? 1 : 0) <= C;
    s_kind[t] = dead ? kDeadOff : (inband ? kInband : kFarOff);
  }
  bad = __syncthreads_or(bad);
  if (bad) {  // the layer has an offset with no defined row: NaN outputs
    const float qnan = __int_as_float(0x7fc00000);
    const size_t ub = (size_t)unit * T * kD;
    for (int e = t; e < kM * kChunks; e += kM) {
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

  if (warp == 0) umma::tmem_alloc(smem_u32(&s_tmem), (uint32_t)a.tmem_cols);
  umma::fence_before_sync();
  __syncthreads();
  umma::fence_after_sync();
  const uint32_t tmem = s_tmem;

  Sync sy;
  sy.bars = bars;
  sy.pend = 0u;
  sy.far_phase = 0u;
  sy.limit = a.wait_limit > 0 ? a.wait_limit : kWaitClocks;
  sy.err = a.err;
  if (!fwd_tile(a, sy, smem, sg, s_kind, tmem, unit, i0)) {
    // a wait gave up: wait (bounded) for the copies and products still in
    // flight, so that none lands after the CTA has left
    for (int b = 0; b < kNumBars; ++b)
      if (sy.pend & (1u << b)) wait_bar(&bars[b], b == kBarFar ? sy.far_phase : 0u, sy.limit);
  }
  umma::fence_before_sync();
  __syncthreads();
  if (warp == 0) {
    umma::fence_after_sync();
    umma::tmem_dealloc(tmem, (uint32_t)a.tmem_cols);
  }
}

__device__ unsigned g_fwd_umma_err;   // error bits as listed in sa_stage.cuh

struct UmmaLayout {
  int NB, N, tmem_cols, sc_stride;
  unsigned off_kb, off_far, off_vb, off_sc;
  size_t smem;                         // dynamic bytes, alignment slack included
};

UmmaLayout umma_layout(const Problem& pb) {
  UmmaLayout L;
  L.NB = kM + 16 * ((pb.W - 1 + 15) / 16);
  L.N = L.NB + (pb.S > 0 ? 16 : 0);
  L.tmem_cols = L.N <= 128 ? 128 : 256;
  L.sc_stride = std::max(pb.n_off, 1) | 1;
  L.off_kb = kM * 128;                                   // after the q^ rows
  L.off_far = L.off_kb + (unsigned)L.N * 128u;
  L.off_vb = L.off_far + (unsigned)kFarRows * 128u;
  L.off_sc = L.off_vb + (unsigned)L.N * 128u;
  const size_t total = L.off_sc + (size_t)kM * L.sc_stride * sizeof(float);
  L.smem = std::max<size_t>(total + 1024, kMinSmem);
  return L;
}

}  // namespace

bool umma_fwd_supported(const Problem& pb) {
  if (pb.dtype != SA_DTYPE_BF16 || pb.D != kD || pb.S > 16 || pb.W < 1) return false;
  const UmmaLayout L = umma_layout(pb);
  // the GEMM's N (band plus sinks) is at most 256; P (N x 256 bytes) fits
  // over the q^ rows, the key band and the far buffer
  return L.N <= 256 && (size_t)L.N * 256 <= L.off_vb && L.smem <= 200 * 1024;
}

cudaError_t launch_fwd_umma(const Problem& pb, const FwdPtrs& p, void* keys_ws, cudaStream_t st,
                            int* launches) {
  const UmmaLayout L = umma_layout(pb);
  UmmaFwdArgs a;
  memset(&a, 0, sizeof(a));
  a.B = pb.B; a.H = pb.H; a.T = pb.T; a.W = pb.W; a.n_off = pb.n_off; a.S = pb.S;
  a.n_tiles = (pb.T + kM - 1) / kM;
  a.NB = L.NB; a.N = L.N; a.tmem_cols = L.tmem_cols; a.sc_stride = L.sc_stride;
  a.off_kb = L.off_kb; a.off_far = L.off_far; a.off_vb = L.off_vb; a.off_sc = L.off_sc;
  a.scale = pb.scale;
  for (int k = 0; k < pb.n_off; ++k) a.f[k] = pb.f[k];
  std::sort(a.f, a.f + pb.n_off);
  a.q = reinterpret_cast<const __nv_bfloat16*>(p.q);
  a.alpha = p.alpha; a.beta = p.beta; a.rope = p.rope;
  a.o = reinterpret_cast<__nv_bfloat16*>(p.o); a.lse = p.lse;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&a.err), g_fwd_umma_err);
  const WaitCfg wc = wait_cfg();
  a.wait_limit = wc.limit;
  a.stall = wc.stall;
  if (e != cudaSuccess) return e;
  if ((e = make_rows_map(&a.tmK, keys_ws, pb.T, pb.units())) != cudaSuccess) return e;
  if ((e = make_rows_map(&a.tmV, p.v, pb.T, pb.units())) != cudaSuccess) return e;
  if ((e = launch_rope_rows(p.k, p.rope, pb.T, pb.units() * pb.T, kKeyStage, keys_ws, st,
                            "rope_keys")) != cudaSuccess)
    return e;
  if ((e = cudaFuncSetAttribute(k_fwd_umma, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                (int)L.smem)) != cudaSuccess)
    return e;
  const unsigned grid = (unsigned)((long long)pb.units() * a.n_tiles);
  trace_mark("fwd_umma", st, true);
  k_fwd_umma<<<grid, kM, L.smem, st>>>(a);
  trace_mark("fwd_umma", st, false);
  e = cudaGetLastError();
  if (e == cudaSuccess) *launches += 2;
  return e;
}

cudaError_t fwd_umma_read_error(unsigned* out, bool clear) {
  cudaError_t e = cudaMemcpyFromSymbol(out, g_fwd_umma_err, sizeof(unsigned));
  if (e != cudaSuccess || !clear || *out == 0) return e;
  const unsigned zero = 0;
  return cudaMemcpyToSymbol(g_fwd_umma_err, &zero, sizeof(unsigned));
}

}  // namespace sa
