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
// produced in ascending order: each thread owns a contiguous run of at most
// 128 keys and marks its keys above and at the threshold in bit masks (16-byte
// key loads), one block scan gives every thread its first output position and
// the number of equal keys before it, the selected indices are compacted in
// place over the staged keys, and the sink receives them in position order.
// (A ballot sweep over every index, twice, cost about 30 instructions per key
// and took half of a 32768-key selection.)  Integer work only: the result is
// the unique set defined by the rule.
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
// list (0 .. k-1), by thread pos % NT.  keys must be 16-byte aligned and
// d <= 128 * NT; the keys are overwritten.
template <int NT, typename Emit>
__device__ __forceinline__ void select_staged_keys(uint32_t* keys, int d, uint32_t k, uint32_t kmin,
                                                   uint32_t kmax, uint32_t* hist, Emit&& emit) {
  constexpr int NW = NT / 32;
  constexpr int BPT = kSelectBins / NT;  // bins per thread, contiguous
  static_assert(BPT == 2 || BPT == 8, "bin vectors are 2 or 8 words");
  __shared__ uint32_t wred[NW][2];  // per-warp min/max, then per-warp bin totals
  __shared__ uint32_t wcnt[NW][2];  // per-warp (above, in-range) counts for the emission
  __shared__ uint32_t sh_bin, sh_above, sh_done;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
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
    // key - lo < range, in 32 bits: range - 1 fits (the range is at most 2^32)
    const uint32_t lo32 = static_cast<uint32_t>(lo), span = static_cast<uint32_t>(range - 1u);
    const int dv = d >> 2;
    for (int v = tid; v < dv; v += NT) {
      const uint4 q = reinterpret_cast<const uint4*>(keys)[v];
      const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t off = kq[e] - lo32;  // wraps for keys below lo
        if (off <= span) atomicAdd(&hist[off >> shift], 1u);
      }
    }
    for (int j = 4 * dv + tid; j < d; j += NT) {
      const uint32_t off = keys[j] - lo32;
      if (off <= span) atomicAdd(&hist[off >> shift], 1u);
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
  // this thread's run [j0, j0 + R): bit masks of its keys at or above hi and
  // of its keys in [lo, hi)
  // (word and bit positions are compile-time: a runtime index would put the
  // masks in local memory)
  constexpr int kWords = 4;  // up to 128 keys per thread
  const int R = (((d + NT - 1) / NT) + 3) & ~3;
  const int j0 = tid * R;
  const bool hi_in = hi <= 0xFFFFFFFFull;  // hi = 2^32: no key lies at or above it
  const uint32_t lo32 = static_cast<uint32_t>(lo), hi32 = static_cast<uint32_t>(hi);
  uint32_t gtm[kWords] = {0u, 0u, 0u, 0u}, eqm[kWords] = {0u, 0u, 0u, 0u};
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int q = 32 * w + 4 * u;  // this vector's first key in the run
      const int j = j0 + q;
      if (q < R && j < d) {
        uint32_t kq[4];
        if (j + 4 <= d) {
          const uint4 v = reinterpret_cast<const uint4*>(keys)[j >> 2];
          kq[0] = v.x; kq[1] = v.y; kq[2] = v.z; kq[3] = v.w;
        } else {
#pragma unroll
          for (int e = 0; e < 4; ++e) kq[e] = j + e < d ? keys[j + e] : 0u;
        }
#pragma unroll
        for (int e = 0; e < 4; ++e) {
          const bool valid = j + e < d;
          const bool ge_hi = hi_in && kq[e] >= hi32;
          gtm[w] |= static_cast<uint32_t>(valid && ge_hi) << (4 * u + e);
          eqm[w] |= static_cast<uint32_t>(valid && kq[e] >= lo32 && !ge_hi) << (4 * u + e);
        }
      }
    }
  }
  uint32_t ngt = 0u, neq = 0u;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    ngt += __popc(gtm[w]);
    neq += __popc(eqm[w]);
  }
  // block exclusive scan of (ngt, neq) in thread order
  uint32_t gi = ngt, ei = neq;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t gn = __shfl_up_sync(0xFFFFFFFFu, gi, o);
    const uint32_t en = __shfl_up_sync(0xFFFFFFFFu, ei, o);
    if (lane >= o) {
      gi += gn;
      ei += en;
    }
  }
  if (lane == 31) {
    wcnt[warp][0] = gi;
    wcnt[warp][1] = ei;
  }
  __syncthreads();  // every key has been read; warp totals are in wcnt
  const uint32_t wg = lane < NW ? wcnt[lane][0] : 0u, we = lane < NW ? wcnt[lane][1] : 0u;
  uint32_t wgi = wg, wei = we;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t gn = __shfl_up_sync(0xFFFFFFFFu, wgi, o);
    const uint32_t en = __shfl_up_sync(0xFFFFFFFFu, wei, o);
    if (lane >= o) {
      wgi += gn;
      wei += en;
    }
  }
  const uint32_t gt_before = __shfl_sync(0xFFFFFFFFu, wgi - wg, warp) + (gi - ngt);
  const uint32_t eq_before = __shfl_sync(0xFFFFFFFFu, wei - we, warp) + (ei - neq);
  // of this thread's equal keys, the first `take` (lowest indices) are kept
  uint32_t take = eq_before < need ? min(neq, need - eq_before) : 0u;
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    uint32_t m = eqm[w], keep = 0u;
    while (m && take) {
      const uint32_t low = m & (~m + 1u);
      keep |= low;
      m ^= low;
      --take;
    }
    gtm[w] |= keep;
  }
  // compact the selected indices, ascending, over the keys
  uint32_t pos = gt_before + min(eq_before, need);
#pragma unroll
  for (int w = 0; w < kWords; ++w) {
    uint32_t m = gtm[w];
    while (m) {
      const int bit = __ffs(m) - 1;
      keys[pos++] = static_cast<uint32_t>(j0 + 32 * w + bit);
      m &= m - 1u;
    }
  }
  __syncthreads();
  for (int q = tid; q < static_cast<int>(k); q += NT) emit(static_cast<uint32_t>(q), static_cast<int>(keys[q]));
}

}  // namespace rmm
