// Row staging for the bf16 / head-dim-64 kernels: bulk copies (the Tensor
// Memory Accelerator's 1-D global -> shared form) into a ring of 128-byte rows
// in shared memory, completion tracked by an mbarrier.
//
// Ring layout.  Row r of a [T][64] 16-bit array lives in slot r & (RB - 1)
// (RB a power of two) at byte offset slot * 128, unswizzled; slots
// [RB, RB + kMirror) repeat slots [0, kMirror).  A lane walks a run of up to
// kMirror consecutive rows from any starting slot at constant offsets
// (slot + u) * 128, with no wrap test.
//
// Bank conflicts.  A lane group (4 lanes) reads 16-byte chunks c and c + 4 of
// one row; the two groups that share a quarter-warp read rows 4 apart, which
// map to the same banks.  Odd groups therefore read the two chunks in the
// opposite order (chunk c + 4 first): in each of the two loads one group
// touches banks 0-15 and the other banks 16-31.  The "first half" a lane
// holds is chunk c + 4 * parity, the second chunk c + 4 * (1 - parity).
//
// Rows outside [0, T) are zero-filled by the threads (the first and last tile
// of a sequence), so every slot a lane reads holds finite data.
//
// Device error word bits (shared by every staged kernel):
//   bit 0 (kErrWait)   a bounded wait for a staging round gave up;
//   bit 1 (kErrBounds) a row index outside the rows staged, or a staging round
//                      larger than the ring (checked only in builds with
//                      SA_DEBUG_BOUNDS; the access is then skipped or clamped);
//   bit 2 (kErrRange)  a finite input whose 16-bit staged form overflows
//                      (|RoPE(K)| / 256 or a scaled query beyond fp16's 65504).
#pragma once

#include "sa_fast_common.cuh"

namespace sa {
namespace stage {

using fast::kChunks;
using fast::kD;

constexpr int kMirror = 12;          // mirrored slots after the ring (longest run: 11 rows)
constexpr int kRowBytes = 128;       // 64 x 16-bit
// Bounded waits: by default a wait that has not completed after this many SM
// clocks (about half a second) gives up and reports through the device error
// word; the host can lower the limit (sparse_attn_set_wait_limit).
constexpr long long kWaitClocks = 1000000000LL;
constexpr unsigned kErrWait = 1u, kErrBounds = 2u, kErrRange = 4u;

__device__ __forceinline__ uint32_t smem_u32(const void* p) {
  return (uint32_t)__cvta_generic_to_shared(p);
}

__device__ __forceinline__ void mbar_init(uint64_t* bar, uint32_t count) {
  asm volatile("mbarrier.init.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)), "r"(count)
               : "memory");
}

// Make the barrier's initialisation visible to the asynchronous proxy.
__device__ __forceinline__ void fence_barrier_init() {
  asm volatile("fence.mbarrier_init.release.cluster;\n" ::: "memory");
}

// Order this thread's generic-proxy shared-memory accesses before later
// asynchronous-proxy (bulk copy) accesses to the same bytes.
__device__ __forceinline__ void fence_proxy_async() {
  asm volatile("fence.proxy.async.shared::cta;\n" ::: "memory");
}

// Raise the barrier's expected transaction bytes (no arrival).
__device__ __forceinline__ void mbar_expect_tx(uint64_t* bar, uint32_t bytes) {
  asm volatile("mbarrier.expect_tx.relaxed.cta.shared::cta.b64 [%0], %1;\n" ::"r"(smem_u32(bar)),
               "r"(bytes)
               : "memory");
}

__device__ __forceinline__ void mbar_arrive(uint64_t* bar) {
  asm volatile("mbarrier.arrive.shared::cta.b64 _, [%0];\n" ::"r"(smem_u32(bar)) : "memory");
}

__device__ __forceinline__ bool mbar_try_wait(uint64_t* bar, uint32_t parity) {
  uint32_t done;
  asm volatile(
      "{\n"
      ".reg .pred p;\n"
      "mbarrier.try_wait.parity.shared::cta.b64 p, [%1], %2;\n"
      "selp.u32 %0, 1, 0, p;\n"
      "}\n"
      : "=r"(done)
      : "r"(smem_u32(bar)), "r"(parity)
      : "memory");
  return done != 0;
}

// Global -> shared bulk copy of `bytes` (a multiple of 16, both addresses
// 16-byte aligned), completing on `bar`.
__device__ __forceinline__ void bulk_copy(void* dst, const void* src, uint32_t bytes,
                                          uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];\n" ::
          "r"(smem_u32(dst)),
      "l"(src), "r"(bytes), "r"(smem_u32(bar))
      : "memory");
}

// Staging state of one CTA: the barrier and its phase bit (identical in every
// thread), the device error word, the wait limit in SM clocks and the planted
// stall of the failure-path test (sparse_attn_plant_stall: the first round
// expects 16 bytes that no copy delivers, so its wait must give up).  In
// SA_DEBUG_BOUNDS builds it also tracks the rows [vlo, vhi) the ring holds.
struct Stager {
  uint64_t* bar;
  uint32_t phase;
  unsigned* err;
  long long limit;
  int stall;
#ifdef SA_DEBUG_BOUNDS
  int vlo, vhi;
#endif
};

__device__ __forceinline__ Stager make_stager(uint64_t* bar, unsigned* err, long long limit,
                                              int stall) {
  Stager s;
  s.bar = bar;
  s.phase = 0u;
  s.err = err;
  s.limit = limit > 0 ? limit : kWaitClocks;
  s.stall = stall;
#ifdef SA_DEBUG_BOUNDS
  s.vlo = s.vhi = 0;
#endif
  return s;
}

// SA_DEBUG_BOUNDS: record a bounds error (bit 1) when rows [r0, r1) are not
// all among the rows the ring holds; other builds: nothing.
__device__ __forceinline__ void dbg_rows(const Stager& s, int r0, int r1) {
#ifdef SA_DEBUG_BOUNDS
  if (r0 < s.vlo || r1 > s.vhi) atomicOr(s.err, kErrBounds);
#else
  (void)s; (void)r0; (void)r1;
#endif
}

// SA_DEBUG_BOUNDS: record a bounds error when cond is false.
__device__ __forceinline__ void dbg_check(unsigned* err, bool cond) {
#ifdef SA_DEBUG_BOUNDS
  if (!cond) atomicOr(err, kErrBounds);
#else
  (void)err; (void)cond;
#endif
}

// SA_DEBUG_BOUNDS: the ring now also holds rows [a, b): extend the tracked
// range when the round is adjacent to it (rows below, or above, what it
// held), keeping the RB rows nearest the new ones; else restart from [a, b).
__device__ __forceinline__ void dbg_staged(Stager& s, int RB, int a, int b) {
#ifdef SA_DEBUG_BOUNDS
  if (b == s.vlo && s.vlo < s.vhi) { s.vlo = a; s.vhi = min(s.vhi, a + RB); }
  else if (a == s.vhi && s.vlo < s.vhi) { s.vhi = b; s.vlo = max(s.vlo, b - RB); }
  else { s.vlo = a; s.vhi = b; }
#else
  (void)s; (void)RB; (void)a; (void)b;
#endif
}

// One staging round: any number of stage_ring / stage_plain calls (thread 0
// registers their bytes and issues their copies; every thread zero-fills),
// then stage_commit_wait.  Thread 0 arrives only after every copy of the round
// is registered, so the phase cannot complete early; a round without copies
// completes at the arrival.

// Arrive (thread 0) and wait for the round, at most s.limit clocks; ends with a
// CTA barrier, so the zero-fills are visible too.  Returns nonzero in every
// thread when any thread gave up (the error word gets bit 0); the caller then
// calls stage_drain and returns.
__device__ __forceinline__ int stage_commit_wait(Stager& s) {
  if (threadIdx.x == 0) {
    if (s.stall) mbar_expect_tx(s.bar, 16u);   // planted: bytes no copy delivers
    mbar_arrive(s.bar);
  }
  s.stall = 0;
  const long long t0 = clock64();
  bool ok;
  while (!(ok = mbar_try_wait(s.bar, s.phase)))
    if (clock64() - t0 > s.limit) break;
  s.phase ^= 1u;
  const int bad = __syncthreads_or(!ok);
  if (bad && threadIdx.x == 0) atomicOr(s.err, kErrWait);
  return bad;
}

// After a wait gave up: wait once more (bounded) for copies still in flight,
// so that none lands in shared memory after the CTA has left.
__device__ __forceinline__ void stage_drain(Stager& s) {
  const long long t0 = clock64();
  while (!mbar_try_wait(s.bar, s.phase ^ 1u))
    if (clock64() - t0 > s.limit) break;
}

// Stage rows [a, b) (b - a <= RB) of `src` (a 16-bit [T][64] array) into the
// ring: bulk copies for the rows inside [0, T) (and their mirror slots), zero
// fill for the rows outside.  The caller has synchronised the CTA since the
// last reads of the slots involved.
__device__ __forceinline__ void stage_ring(Stager& s, unsigned char* ring, int RB, const void* src,
                                           int T, int a, int b) {
#ifdef SA_DEBUG_BOUNDS
  if (b - a > RB) {                   // more rows than slots: record and stage none
    if (threadIdx.x == 0) atomicOr(s.err, kErrBounds);
    return;
  }
#endif
  dbg_staged(s, RB, a, b);
  const int ca = max(a, 0), cb = min(b, T);
  {
    const int n_lo = max(0, min(b, 0) - a);          // rows a .. min(b, 0) - 1
    const int z_hi0 = max(a, T);
    const int n_hi = max(0, b - z_hi0);              // rows max(a, T) .. b - 1
    const int nz = (n_lo + n_hi) * kChunks;
    for (int e = threadIdx.x; e < nz; e += blockDim.x) {
      const int k = e / kChunks, ch = e % kChunks;
      const int row = k < n_lo ? a + k : z_hi0 + (k - n_lo);
      const int slot = row & (RB - 1);
      uint4* d = reinterpret_cast<uint4*>(ring + (size_t)slot * kRowBytes) + ch;
      *d = make_uint4(0, 0, 0, 0);
      if (slot < kMirror) *(d + (size_t)RB * kChunks) = make_uint4(0, 0, 0, 0);
    }
    if (nz) fence_proxy_async();
  }
  if (ca >= cb || threadIdx.x != 0) return;
  const unsigned char* g = reinterpret_cast<const unsigned char*>(src);
  // up to two contiguous slot segments (the ring wraps at most once)
  const int s0 = ca & (RB - 1);
  const int n1 = min(cb - ca, RB - s0);
  const int n2 = (cb - ca) - n1;
  const int m1 = s0 < kMirror ? min(n1, kMirror - s0) : 0;   // mirror rows of segment 1
  const int m2 = min(n2, kMirror);                           // segment 2 starts at slot 0
  mbar_expect_tx(s.bar, (uint32_t)(n1 + n2 + m1 + m2) * kRowBytes);
  bulk_copy(ring + (size_t)s0 * kRowBytes, g + (size_t)ca * kRowBytes, (uint32_t)n1 * kRowBytes,
            s.bar);
  if (m1)
    bulk_copy(ring + (size_t)(RB + s0) * kRowBytes, g + (size_t)ca * kRowBytes,
              (uint32_t)m1 * kRowBytes, s.bar);
  if (n2) bulk_copy(ring, g + (size_t)(ca + n1) * kRowBytes, (uint32_t)n2 * kRowBytes, s.bar);
  if (m2)
    bulk_copy(ring + (size_t)RB * kRowBytes, g + (size_t)(ca + n1) * kRowBytes,
              (uint32_t)m2 * kRowBytes, s.bar);
}

// Stage rows [0, n) of src into a plain buffer (row r at r * 128); rows
// [n_valid, n) are zero-filled.
__device__ __forceinline__ void stage_plain(Stager& s, unsigned char* buf, const void* src,
                                            int n_valid, int n) {
  n_valid = max(0, min(n_valid, n));
  for (int e = threadIdx.x + n_valid * kChunks; e < n * kChunks; e += blockDim.x)
    reinterpret_cast<uint4*>(buf)[e] = make_uint4(0, 0, 0, 0);
  if (n_valid < n) fence_proxy_async();
  if (n_valid == 0 || threadIdx.x != 0) return;
  mbar_expect_tx(s.bar, (uint32_t)n_valid * kRowBytes);
  bulk_copy(buf, src, (uint32_t)n_valid * kRowBytes, s.bar);
}

// Asynchronous 4-byte global -> shared copy (completes at cp_async_wait_all).
__device__ __forceinline__ void cp_async4(void* smem_dst, const void* gsrc) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 4;\n" ::"r"(smem_u32(smem_dst)), "l"(gsrc)
               : "memory");
}
__device__ __forceinline__ void cp_async_wait_all() {
  asm volatile("cp.async.wait_all;\n" ::: "memory");
}

// ---- lane access ------------------------------------------------------------
// Byte offsets, within a row, of the two 16-byte chunks lane (group parity
// `par`, lane-in-group c) holds: first half, second half.
__device__ __forceinline__ int half0_off(int c, int par) { return (c + 4 * par) * 16; }
__device__ __forceinline__ int half1_off(int c, int par) { return (c + 4 - 4 * par) * 16; }

// Unpack 8 packed 16-bit values (fp16 when F16, else bf16) to fp32.
template <bool F16>
__device__ __forceinline__ void unpack8x(const uint4 u, float* x) {
  if (F16) fast::unpack8_h(u, x);
  else fast::unpack8(u, x);
}

// This lane's 16 values of the row at byte address `p` (the row's slot base
// plus the lane's first-half offset); `d1` = second-half offset minus
// first-half offset (+64 or -64).
template <bool F16>
__device__ __forceinline__ void lane_row(const unsigned char* p, int d1, float (&x)[16]) {
  unpack8x<F16>(*reinterpret_cast<const uint4*>(p), x);
  unpack8x<F16>(*reinterpret_cast<const uint4*>(p + d1), x + 8);
}

}  // namespace stage
}  // namespace sa
