// rmm_select.cuh — the exact top-k selection shared by the top-k kernels and
// the fused decode product (Reduced Matrix Multiplication technical summary,
// Metodología › Estrategia de Selección: keep the k indices with the highest
// scores; the tie rule, lowest index first, and the ascending order are this
// library's reading).
//
// Scores are mapped to order-preserving uint32 keys; keys staged in shared
// memory are searched by histogram rounds: the key range [min, max] is cut
// into 2048 bins, the bin holding the k-th largest key becomes the new range,
// and the search stops when the range is a single key (at most three rounds
// for 32-bit keys) or when the keys at or above the range's start are exactly
// k.  Each round costs three block barriers.  The selected indices are then
// produced in ascending order in one sweep: each warp owns a contiguous block
// of indices, one barrier exchanges the warps' counts, and ballots place each
// index.  Integer work only: the result is the unique set defined by the rule.
#pragma once

#include <cstdint>

namespace rmm {

constexpr int kSelectBins = 2048;

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                       // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // monotone in the float order
}

// Histogram search on keys staged in shared memory.  Invariant of the
// search: count(key >= hi) = `above` < k <= count(key >= lo).  The caller has
// written keys[0..d) and passes each thread's minimum and maximum key and a
// shared-memory array of kSelectBins words (`hist`, 16-byte aligned, any
// contents); every thread of the block calls this once.  emit(pos, j) is
// called once for each selected index j, with pos its place in the ascending
// list (0 .. k-1).
template <int NT, typename Emit>
__device__ __forceinline__ void select_staged_keys(const uint32_t* keys, int d, uint32_t k, uint32_t kmin,
                                                   uint32_t kmax, uint32_t* hist, Emit&& emit) {
  constexpr int NW = NT / 32;
  constexpr int BPT = kSelectBins / NT;  // bins per thread, contiguous
  static_assert(BPT == 2 || BPT == 8, "bin vectors are 2 or 8 words");
  __shared__ uint32_t wred[NW][2];  // per-warp min/max, then per-warp bin totals
  __shared__ uint32_t wcnt[NW][2];  // per-warp (above, in-range) counts for the emission
  __shared__ uint32_t sh_bin, sh_above, sh_done;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint32_t lt_mask = (1u << lane) - 1u;
  for (int b = tid; b < kSelectBins; b += NT) hist[b] = 0u;
  kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
  kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
  if (lane == 0) {
    wred[warp][0] = kmin;
    wred[warp][1] = kmax;
  }
  __syncthreads();
  uint64_t lo = __reduce_min_sync(0xFFFFFFFFu, lane < NW ? wred[lane][0] : 0xFFFFFFFFu);
  uint64_t hi = static_cast<uint64_t>(__reduce_max_sync(0xFFFFFFFFu, lane < NW ? wred[lane][1] : 0u)) + 1u;
  uint32_t above = 0u;
  bool done = false;

  // each round shrinks the range at least 2048-fold (or to one key), so four
  // rounds always suffice for 32-bit keys; the bound is only a guard
  for (int round = 0; round < 8 && hi - lo > 1u && !done; ++round) {
    const uint64_t range = hi - lo;
    const int nbits = 64 - __clzll(static_cast<long long>(range - 1u));  // ceil(log2(range))
    const int shift = nbits > 11 ? nbits - 11 : 0;
    for (int j = tid; j < d; j += NT) {
      const uint32_t key = keys[j];
      if (key >= lo && key < hi) atomicAdd(&hist[static_cast<uint32_t>((key - lo) >> shift)], 1u);
    }
    __syncthreads();
    // this thread's bins [tid*BPT, tid*BPT + BPT), read and cleared for the next round
    uint32_t c[BPT];
    if constexpr (BPT == 2) {
      const uint2 v = reinterpret_cast<const uint2*>(hist)[tid];
      c[0] = v.x;
      c[1] = v.y;
      reinterpret_cast<uint2*>(hist)[tid] = make_uint2(0u, 0u);
    } else {
      const uint4 v0 = reinterpret_cast<const uint4*>(hist)[2 * tid];
      const uint4 v1 = reinterpret_cast<const uint4*>(hist)[2 * tid + 1];
      c[0] = v0.x; c[1] = v0.y; c[2] = v0.z; c[3] = v0.w;
      c[4] = v1.x; c[5] = v1.y; c[6] = v1.z; c[7] = v1.w;
      reinterpret_cast<uint4*>(hist)[2 * tid] = make_uint4(0u, 0u, 0u, 0u);
      reinterpret_cast<uint4*>(hist)[2 * tid + 1] = make_uint4(0u, 0u, 0u, 0u);
    }
    uint32_t local = 0u;
#pragma unroll
    for (int i = 0; i < BPT; ++i) local += c[i];
    uint32_t incl = local;  // keys in the bins of lanes >= this lane (this warp)
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_down_sync(0xFFFFFFFFu, incl, o);
      if (lane + o < 32) incl += n;
    }
    if (lane == 0) wred[warp][0] = incl;
    __syncthreads();
    const uint32_t wt = lane < NW ? wred[lane][0] : 0u;
    uint32_t wincl = wt;  // keys in the bins of warps >= lane
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_down_sync(0xFFFFFFFFu, wincl, o);
      if (lane + o < 32) wincl += n;
    }
    const uint32_t after_warp = __shfl_sync(0xFFFFFFFFu, wincl - wt, warp);
    // walk this thread's bins from the top: exactly one bin in the block has
    // above + (keys in higher bins) < k <= above + (keys in it and higher bins)
    uint32_t higher = above + after_warp + (incl - local);
#pragma unroll
    for (int i = BPT - 1; i >= 0; --i) {
      const uint32_t ge = higher + c[i];
      if (higher < k && ge >= k) {
        sh_bin = static_cast<uint32_t>(tid * BPT + i);
        sh_above = higher;
        sh_done = ge == k ? 1u : 0u;
      }
      higher = ge;
    }
    __syncthreads();
    const uint64_t nlo = lo + (static_cast<uint64_t>(sh_bin) << shift);
    const uint64_t nhi = nlo + (1ull << shift);
    hi = nhi < hi ? nhi : hi;
    lo = nlo;
    above = sh_above;
    done = sh_done != 0u;
  }

  // Selected: every key >= hi (`above` of them) and, lowest index first,
  // need = k - above of the keys in [lo, hi).  When the search stopped with
  // exactly k keys at or above lo, that is all of them; otherwise [lo, hi)
  // is the single key T of the k-th largest score.
  const uint32_t need = k - above;
  const int C = ((d + 32 * NW - 1) / (32 * NW)) * 32;  // indices per warp
  const int j0 = warp * C, j1 = min(d, j0 + C);
  uint32_t ngt = 0u, neq = 0u;
  for (int base = j0; base < j1; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < j1 ? keys[j] : 0u;
    ngt += __popc(__ballot_sync(0xFFFFFFFFu, j < j1 && key >= hi));
    neq += __popc(__ballot_sync(0xFFFFFFFFu, j < j1 && key >= lo && key < hi));
  }
  if (lane == 0) {
    wcnt[warp][0] = ngt;
    wcnt[warp][1] = neq;
  }
  __syncthreads();
  const uint32_t g = lane < NW ? wcnt[lane][0] : 0u, e = lane < NW ? wcnt[lane][1] : 0u;
  uint32_t gi = g, ei = e;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t gn = __shfl_up_sync(0xFFFFFFFFu, gi, o);
    const uint32_t en = __shfl_up_sync(0xFFFFFFFFu, ei, o);
    if (lane >= o) {
      gi += gn;
      ei += en;
    }
  }
  const uint32_t gt_before = __shfl_sync(0xFFFFFFFFu, gi - g, warp);
  uint32_t eq_run = __shfl_sync(0xFFFFFFFFu, ei - e, warp);
  uint32_t pos = gt_before + min(eq_run, need);
  for (int base = j0; base < j1; base += 32) {
    const int j = base + lane;
    const uint32_t key = j < j1 ? keys[j] : 0u;
    const bool gt = j < j1 && key >= hi;
    const bool eq = j < j1 && key >= lo && key < hi;
    const uint32_t eb = __ballot_sync(0xFFFFFFFFu, eq);
    const bool sel = gt || (eq && eq_run + __popc(eb & lt_mask) < need);
    const uint32_t sb = __ballot_sync(0xFFFFFFFFu, sel);
    if (sel) emit(pos + __popc(sb & lt_mask), j);
    pos += __popc(sb);
    eq_run += __popc(eb);
  }
}

}  // namespace rmm
