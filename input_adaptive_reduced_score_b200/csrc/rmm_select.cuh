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
//
// A row too long for one CTA to search quickly is split over a thread-block
// cluster: CTA r of C stages the r-th consecutive slice, each round's
// histogram is the sum of the C CTAs' bins read through distributed shared
// memory (two bin buffers, so one cluster barrier per round suffices), every
// CTA takes the same decision from the same sums, and one more exchange of
// the CTAs' counts places each slice's selections in the row's list.
#pragma once

#include <cstdint>

#include "rmm_device.cuh"

namespace rmm {

constexpr int kSelectBins = 2048;

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                       // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // monotone in the float order
}

// Stage the keys of scores s[0 .. d) in shared memory and return this
// thread's smallest and largest key.  16-byte loads when s is 16-byte
// aligned, four in flight per thread (one memory round trip per batch).
template <int NT>
__device__ __forceinline__ void stage_score_keys(const float* __restrict__ s, int d, uint32_t* keys, uint32_t& kmin,
                                                 uint32_t& kmax) {
  const int tid = threadIdx.x;
  kmin = 0xFFFFFFFFu;
  kmax = 0u;
  const int nv = (reinterpret_cast<uintptr_t>(s) & 15u) == 0 ? d >> 2 : 0;
  const float4* s4 = reinterpret_cast<const float4*>(s);
  for (int v0 = tid; v0 < nv; v0 += 4 * NT) {
    float4 f[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * NT;
      f[u] = v < nv ? __ldg(s4 + v) : make_float4(0.f, 0.f, 0.f, 0.f);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int v = v0 + u * NT;
      if (v < nv) {
        const uint4 q = make_uint4(score_key(f[u].x), score_key(f[u].y), score_key(f[u].z), score_key(f[u].w));
        reinterpret_cast<uint4*>(keys)[v] = q;
        kmin = min(kmin, min(min(q.x, q.y), min(q.z, q.w)));
        kmax = max(kmax, max(max(q.x, q.y), max(q.z, q.w)));
      }
    }
  }
  for (int j0 = 4 * nv + tid; j0 < d; j0 += 8 * NT) {
    float f[8];
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * NT;
      f[u] = j < d ? __ldg(s + j) : 0.f;
    }
#pragma unroll
    for (int u = 0; u < 8; ++u) {
      const int j = j0 + u * NT;
      if (j < d) {
        const uint32_t key = score_key(f[u]);
        keys[j] = key;
        kmin = min(kmin, key);
        kmax = max(kmax, key);
      }
    }
  }
}

// Where a CTA's selections go: its slice's selected indices (slice-local,
// ascending) are in keys[0 .. count), and they take places base .. base +
// count - 1 of the row's ascending list.
struct StagedSelection {
  uint32_t base, count;
};

// The outcome of the search, the same in every CTA of a cluster: the
// selected keys are every key >= hi and, lowest index first, `need` of the
// keys in [lo, hi).  `split` is false when those are all of the keys in
// [lo, hi) (then the selection is simply key >= lo); when true, [lo, hi) is
// the single key of the k-th largest score and some of its copies are left.
struct SelectThreshold {
  uint64_t lo, hi;
  uint32_t need;
  bool split;
};

// Histogram search on keys staged in shared memory.  Invariant of the
// search: count(key >= hi) = `above` < k <= count(key >= lo), counted over
// the whole row.  The caller has written this CTA's keys[0..d) and passes
// each thread's minimum and maximum key (unused when C > 1); every thread of
// the block (of every block of the cluster, C > 1) calls this once.  hist: kSelectBins words
// (2 kSelectBins when C > 1) of shared memory, 16-byte aligned, any contents.
// keys must be 16-byte aligned and d <= 128 * NT; 1 <= k <= the row's length.
// With C > 1 the row is the concatenation of the slices of cluster ranks
// 0 .. C-1 (launched as a cluster along x), and the other CTAs may still
// read this CTA's bins until all pass the next cluster barrier: the caller
// must not write hist, nor exit, before one (select_compact has one).
template <int NT, int C>
__device__ __forceinline__ SelectThreshold select_threshold(const uint32_t* keys, int d, uint32_t k, uint32_t kmin,
                                                            uint32_t kmax, uint32_t* hist) {
  constexpr int NW = NT / 32;
  constexpr int BPT = kSelectBins / NT;  // bins per thread, contiguous
  static_assert(BPT == 2 || BPT == 4 || BPT == 8, "bin vectors are 2, 4 or 8 words");
  static_assert(C == 1 || C == 2 || C == 4 || C == 8 || C == 16, "cluster of 1, 2, 4, 8 or 16 CTAs");
  constexpr int NBUF = C > 1 ? 2 : 1;
  __shared__ uint32_t wred[NW][2];  // per-warp min/max, then per-warp bin totals
  __shared__ uint32_t sh_bin, sh_above, sh_done, sh_count;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  for (int b = tid; b < NBUF * kSelectBins; b += NT) hist[b] = 0u;
  uint64_t lo, hi;
  if constexpr (C > 1) {
    // a cluster starts from the whole key range: exchanging the CTAs'
    // extremes costs a cluster barrier and a remote read, and saves a round
    // only when every key of the row lies within 2^22 of the others
    __syncthreads();  // the bins are cleared before any thread counts
    lo = 0u;
    hi = 1ull << 32;
  } else {
    kmin = __reduce_min_sync(0xFFFFFFFFu, kmin);
    kmax = __reduce_max_sync(0xFFFFFFFFu, kmax);
    if (lane == 0) {
      wred[warp][0] = kmin;
      wred[warp][1] = kmax;
    }
    __syncthreads();
    lo = __reduce_min_sync(0xFFFFFFFFu, lane < NW ? wred[lane][0] : 0xFFFFFFFFu);
    hi = static_cast<uint64_t>(__reduce_max_sync(0xFFFFFFFFu, lane < NW ? wred[lane][1] : 0u)) + 1u;
  }
  uint32_t above = 0u;
  uint32_t in_range = 0xFFFFFFFFu;  // keys in [lo, hi) over the row (unknown before the first round)
  bool done = false;

  // each round shrinks the range at least 2048-fold (or to one key), so four
  // rounds always suffice for 32-bit keys; the bound is only a guard
  for (int round = 0; round < 8 && hi - lo > 1u && !done; ++round) {
    const uint64_t range = hi - lo;
    const int nbits = 64 - __clzll(static_cast<long long>(range - 1u));  // ceil(log2(range))
    const int shift = nbits > 11 ? nbits - 11 : 0;
    // key - lo < range, in 32 bits: range - 1 fits (the range is at most 2^32)
    const uint32_t lo32 = static_cast<uint32_t>(lo), span = static_cast<uint32_t>(range - 1u);
    uint32_t* h = hist + (NBUF > 1 ? (round & 1) * kSelectBins : 0);
    const int dv = d >> 2;
    for (int v = tid; v < dv; v += NT) {
      const uint4 q = reinterpret_cast<const uint4*>(keys)[v];
      const uint32_t kq[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        const uint32_t off = kq[e] - lo32;  // wraps for keys below lo
        if (off <= span) atomicAdd(&h[off >> shift], 1u);
      }
    }
    for (int j = 4 * dv + tid; j < d; j += NT) {
      const uint32_t off = keys[j] - lo32;
      if (off <= span) atomicAdd(&h[off >> shift], 1u);
    }
    // this thread's bins [tid*BPT, tid*BPT + BPT), summed over the cluster
    uint32_t c[BPT];
    if constexpr (C == 1) {
      __syncthreads();
      // read and cleared for the next round
      if constexpr (BPT == 2) {
        const uint2 v = reinterpret_cast<const uint2*>(h)[tid];
        c[0] = v.x;
        c[1] = v.y;
        reinterpret_cast<uint2*>(h)[tid] = make_uint2(0u, 0u);
      } else if constexpr (BPT == 4) {
        const uint4 v = reinterpret_cast<const uint4*>(h)[tid];
        c[0] = v.x; c[1] = v.y; c[2] = v.z; c[3] = v.w;
        reinterpret_cast<uint4*>(h)[tid] = make_uint4(0u, 0u, 0u, 0u);
      } else {
        const uint4 v0 = reinterpret_cast<const uint4*>(h)[2 * tid];
        const uint4 v1 = reinterpret_cast<const uint4*>(h)[2 * tid + 1];
        c[0] = v0.x; c[1] = v0.y; c[2] = v0.z; c[3] = v0.w;
        c[4] = v1.x; c[5] = v1.y; c[6] = v1.z; c[7] = v1.w;
        reinterpret_cast<uint4*>(h)[2 * tid] = make_uint4(0u, 0u, 0u, 0u);
        reinterpret_cast<uint4*>(h)[2 * tid + 1] = make_uint4(0u, 0u, 0u, 0u);
      }
    } else {
      cluster_sync();  // every CTA's bins of this round are complete
#pragma unroll
      for (int i = 0; i < BPT; ++i) c[i] = 0u;
      const uint32_t mine = smem_u32(h) + static_cast<uint32_t>(tid * BPT * 4);
#pragma unroll
      for (int r = 0; r < C; ++r) {
        const uint32_t a = mapa_shared(mine, static_cast<uint32_t>(r));
        if constexpr (BPT == 2) {
          const uint2 v = ld_dsmem_v2(a);
          c[0] += v.x;
          c[1] += v.y;
        } else if constexpr (BPT == 4) {
          const uint4 v = ld_dsmem_v4(a);
          c[0] += v.x; c[1] += v.y; c[2] += v.z; c[3] += v.w;
        } else {
          const uint4 v0 = ld_dsmem_v4(a), v1 = ld_dsmem_v4(a + 16u);
          c[0] += v0.x; c[1] += v0.y; c[2] += v0.z; c[3] += v0.w;
          c[4] += v1.x; c[5] += v1.y; c[6] += v1.z; c[7] += v1.w;
        }
      }
      // the other buffer was last read (by every CTA, last round) before
      // this round's barrier: clear this thread's bins of it for next round
      uint32_t* o = hist + ((round + 1) & 1) * kSelectBins + tid * BPT;
#pragma unroll
      for (int i = 0; i < BPT; ++i) o[i] = 0u;
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
        sh_count = c[i];
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
    in_range = sh_count;
    done = sh_done != 0u;
  }
  // When the search stopped with exactly k keys at or above lo, all keys in
  // [lo, hi) are taken; otherwise [lo, hi) is the single key T of the k-th
  // largest score, of which need = k - above copies are taken.
  const uint32_t need = k - above;
  return SelectThreshold{lo, hi, need, need < in_range};
}

// The selected indices of this CTA's slice compacted, ascending, over its
// keys (every thread of the block, of every block of the cluster, calls this
// once, after select_threshold on the same keys).  With C > 1, on return this
// thread has arrived on the cluster barrier after its last access to another
// CTA's shared memory: the caller must call cluster_wait() before it exits
// and must not use the cluster barrier in between.
template <int NT, int C>
__device__ __forceinline__ StagedSelection select_compact(uint32_t* keys, int d, const SelectThreshold& thr) {
  constexpr int NW = NT / 32;
  __shared__ uint32_t wcnt[NW][2];  // per-warp (above, in-range) counts
  __shared__ uint32_t xch[2];       // read by the cluster's CTAs: block counts
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const uint64_t lo = thr.lo, hi = thr.hi;
  const uint32_t need = thr.need;
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
  for (int v4 = 0; v4 < 8 * kWords; ++v4) {
    const int q = 4 * v4;  // this vector's first key in the run
    const int j = j0 + q;
    if (q >= R || j >= d) break;  // runs are short for small rows: leave the unrolled sweep early
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
      gtm[v4 >> 3] |= static_cast<uint32_t>(valid && ge_hi) << (4 * (v4 & 7) + e);
      eqm[v4 >> 3] |= static_cast<uint32_t>(valid && kq[e] >= lo32 && !ge_hi) << (4 * (v4 & 7) + e);
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
  uint32_t gt_before = __shfl_sync(0xFFFFFFFFu, wgi - wg, warp) + (gi - ngt);
  uint32_t eq_before = __shfl_sync(0xFFFFFFFFu, wei - we, warp) + (ei - neq);
  // this CTA's totals, and the totals of the cluster's lower ranks
  const uint32_t cta_gt = __shfl_sync(0xFFFFFFFFu, wgi, 31), cta_eq = __shfl_sync(0xFFFFFFFFu, wei, 31);
  uint32_t gt_pre = 0u, eq_pre = 0u;
  if constexpr (C > 1) {
    if (tid == 0) {
      xch[0] = cta_gt;
      xch[1] = cta_eq;
    }
    cluster_sync();
    const int rank = static_cast<int>(cluster_ctarank());
    uint32_t g0 = 0u, e0 = 0u;
    if (lane < rank) {
      const uint32_t a = mapa_shared(smem_u32(xch), static_cast<uint32_t>(lane));
      g0 = ld_dsmem_u32(a);
      e0 = ld_dsmem_u32(a + 4u);
    }
    gt_pre = __reduce_add_sync(0xFFFFFFFFu, g0);
    eq_pre = __reduce_add_sync(0xFFFFFFFFu, e0);
    cluster_arrive();  // no further access to another CTA's shared memory
    gt_before += gt_pre;
    eq_before += eq_pre;
  }
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
  // compact the selected indices, ascending, over the keys (slice-local
  // places: minus this CTA's first place in the row's list)
  const uint32_t base = gt_pre + min(eq_pre, need);
  const uint32_t count = cta_gt + (eq_pre < need ? min(cta_eq, need - eq_pre) : 0u);
  uint32_t pos = gt_before + min(eq_before, need) - base;
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
  return StagedSelection{base, count};
}

// Search and compaction (the contract of select_compact).
template <int NT, int C>
__device__ __forceinline__ StagedSelection select_staged_compact(uint32_t* keys, int d, uint32_t k, uint32_t kmin,
                                                                 uint32_t kmax, uint32_t* hist) {
  const SelectThreshold thr = select_threshold<NT, C>(keys, d, k, kmin, kmax, hist);
  return select_compact<NT, C>(keys, d, thr);
}

// The one-CTA search (C = 1) followed by the emission: emit(pos, j) is called
// once for each selected index j, with pos its place in the ascending list
// (0 .. k-1), by thread pos % NT.
template <int NT, typename Emit>
__device__ __forceinline__ void select_staged_keys(uint32_t* keys, int d, uint32_t k, uint32_t kmin,
                                                   uint32_t kmax, uint32_t* hist, Emit&& emit) {
  select_staged_compact<NT, 1>(keys, d, k, kmin, kmax, hist);
  for (int q = threadIdx.x; q < static_cast<int>(k); q += NT) emit(static_cast<uint32_t>(q), static_cast<int>(keys[q]));
}

}  // namespace rmm
