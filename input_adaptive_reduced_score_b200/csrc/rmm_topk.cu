// rmm_topk.cu — deterministic top-k index selection (Reduced Matrix
// Multiplication technical summary, Metodología › Estrategia de Selección:
// keep the k indices with the highest scores).  The tie rule (lowest index
// first) and the ascending output order are this library's reading.
//
// One 1024-thread CTA per score row; scores are mapped to order-preserving
// uint32 keys.  The exact key T of the k-th largest score is found either by
// a register-resident 4-ary search over the key range (rows of up to 16384)
// or by a 4-pass MSB-first radix select (8-bit digits, shared-memory
// histograms; keys staged once in shared memory when the row fits in 200 KB).
// A final ordered sweep emits, in ascending index order, every index with
// key > T and the first `need` indices with key == T, using warp ballots and
// a block-wide scan for output positions.
// Integer work only: the result is the unique set defined by the rule.
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

constexpr int kTopkThreads = 1024;

__device__ __forceinline__ uint32_t score_key(float f) {
  uint32_t u = __float_as_uint(f);
  if (u == 0x80000000u) u = 0u;                       // -0.0 ranks as +0.0
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);  // monotone in the float order
}

// Block-wide exclusive scan of one flag per thread; returns this thread's
// exclusive count, and the block total in *total.  Uses `warp_cnt` (32 words).
__device__ __forceinline__ uint32_t block_flag_scan(bool flag, uint32_t* warp_cnt, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  const uint32_t ballot = __ballot_sync(0xFFFFFFFFu, flag);
  const uint32_t below = __popc(ballot & ((1u << lane) - 1u));
  if (lane == 0) warp_cnt[warp] = __popc(ballot);
  __syncthreads();
  if (warp == 0) {
    const uint32_t c = warp_cnt[lane];
    uint32_t incl = c;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
      if (lane >= o) incl += n;
    }
    warp_cnt[lane] = incl - c;           // exclusive prefix of warp counts
    if (lane == 31) warp_cnt[32] = incl;  // total
  }
  __syncthreads();
  const uint32_t r = warp_cnt[warp] + below;
  *total = warp_cnt[32];
  __syncthreads();  // warp_cnt is reused by the next call
  return r;
}

// Keys of the row: staged in dynamic shared memory when it fits (one parallel
// load, then every pass reads shared memory), else re-read from global memory.
template <bool kStaged>
__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int64_t d,
                                                             int64_t ld_s, int64_t k, int32_t* __restrict__ idx,
                                                             int64_t ld_idx) {
  extern __shared__ uint32_t staged[];
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_cnt[33];
  __shared__ uint32_t sh_prefix, sh_need;
  const float* s = scores + static_cast<int64_t>(blockIdx.x) * ld_s;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.x) * ld_idx;
  const int tid = threadIdx.x, lane = tid & 31;
  pdl_wait();
  pdl_trigger();

  if (kStaged) {
    for (int64_t j = tid; j < d; j += kTopkThreads) staged[j] = score_key(__ldg(s + j));
  }
  auto key_at = [&](int64_t j) -> uint32_t { return kStaged ? staged[j] : score_key(__ldg(s + j)); };

  uint32_t prefix = 0u, mask = 0u, need = static_cast<uint32_t>(k);
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    for (int64_t j = tid; j < d; j += kTopkThreads) {
      const uint32_t key = key_at(j);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & 255u], 1u);
    }
    __syncthreads();
    if (tid < 32) {
      // lane l owns buckets 255-8l ... 248-8l (descending key order)
      uint32_t c[8], sum = 0u;
#pragma unroll
      for (int i = 0; i < 8; ++i) {
        c[i] = hist[255 - 8 * lane - i];
        sum += c[i];
      }
      uint32_t incl = sum;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t n = __shfl_up_sync(0xFFFFFFFFu, incl, o);
        if (lane >= o) incl += n;
      }
      uint32_t before = incl - sum;  // keys in buckets above this lane's
      if (before < need && need <= incl) {
#pragma unroll
        for (int i = 0; i < 8; ++i) {
          if (before < need && need <= before + c[i]) {
            sh_prefix = prefix | (static_cast<uint32_t>(255 - 8 * lane - i) << shift);
            sh_need = need - before;
          }
          before += c[i];
        }
      }
    }
    __syncthreads();
    prefix = sh_prefix;
    need = sh_need;
    mask |= 255u << shift;
    __syncthreads();
  }

  // prefix is now the exact key T of the k-th largest score; `need` keys equal
  // to T are kept, lowest index first.
  const uint32_t T = prefix;
  uint32_t eq_seen = 0u, written = 0u;
  for (int64_t base = 0; base < d; base += kTopkThreads) {
    const int64_t j = base + tid;
    const bool in = j < d;
    const uint32_t key = in ? key_at(j) : 0u;
    const bool eq = in && key == T;
    uint32_t eq_total;
    const uint32_t eq_rank = eq_seen + block_flag_scan(eq, warp_cnt, &eq_total);
    const bool sel = in && (key > T || (eq && eq_rank < need));
    uint32_t sel_total;
    const uint32_t pos = written + block_flag_scan(sel, warp_cnt, &sel_total);
    if (sel) out[pos] = static_cast<int32_t>(j);
    eq_seen += eq_total;
    written += sel_total;
  }
}

// Register-resident variant for d <= 1024 * KPT: thread t holds the keys of
// indices t, t + 1024, ...  The threshold T (the k-th largest key) is found by
// a 4-ary search over the 32-bit key range: each step counts, block-wide, the
// keys at or above three probes (warp redux + one barrier, double-buffered
// counts), keeping count(>= lo) >= k > count(>= hi).  Sixteen steps reach
// hi = lo + 1, so T = lo exactly.  No atomics.
template <int KPT>
__global__ void __launch_bounds__(kTopkThreads, 1) topk_search_kernel(const float* __restrict__ scores, int64_t d,
                                                                       int64_t ld_s, int64_t k,
                                                                       int32_t* __restrict__ idx, int64_t ld_idx) {
  __shared__ uint32_t wcnt[2][32][4];
  __shared__ uint32_t warp_cnt[33];
  const float* s = scores + static_cast<int64_t>(blockIdx.x) * ld_s;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.x) * ld_idx;
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  pdl_wait();
  pdl_trigger();

  uint32_t key[KPT];
  uint32_t valid = 0u;
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const int64_t j = tid + static_cast<int64_t>(i) * kTopkThreads;
    key[i] = j < d ? score_key(__ldg(s + j)) : 0u;
    if (j < d) valid |= 1u << i;
  }
  // every probe lies below 2^32 (probes < hi <= 2^32), so 32-bit compares suffice
  auto count_ge = [&](uint64_t t) -> uint32_t {
    const uint32_t t32 = static_cast<uint32_t>(t);
    uint32_t c = 0u;
#pragma unroll
    for (int i = 0; i < KPT; ++i) c += ((valid >> i) & 1u) && key[i] >= t32 ? 1u : 0u;
    return c;
  };

  uint64_t lo = 0ull, hi = 1ull << 32;  // count(>= lo) = d >= k; count(>= 2^32) = 0 < k
  int buf = 0;
  while (hi - lo > 1ull) {
    const uint64_t w = hi - lo;
    const uint64_t t1 = lo + w / 4, t2 = lo + w / 2, t3 = lo + (w * 3) / 4;
    const uint32_t c1 = __reduce_add_sync(0xFFFFFFFFu, count_ge(t1));
    const uint32_t c2 = __reduce_add_sync(0xFFFFFFFFu, count_ge(t2));
    const uint32_t c3 = __reduce_add_sync(0xFFFFFFFFu, count_ge(t3));
    if (lane == 0) {
      wcnt[buf][warp][0] = c1;
      wcnt[buf][warp][1] = c2;
      wcnt[buf][warp][2] = c3;
    }
    __syncthreads();
    // every warp sums the 32 per-warp counts itself (no second barrier)
    const uint32_t n1 = __reduce_add_sync(0xFFFFFFFFu, wcnt[buf][lane][0]);
    const uint32_t n2 = __reduce_add_sync(0xFFFFFFFFu, wcnt[buf][lane][1]);
    const uint32_t n3 = __reduce_add_sync(0xFFFFFFFFu, wcnt[buf][lane][2]);
    const uint64_t kk = static_cast<uint64_t>(k);
    if (n3 >= kk) {
      lo = t3;
    } else if (n2 >= kk) {
      lo = t2;
      hi = t3;
    } else if (n1 >= kk) {
      lo = t1;
      hi = t2;
    } else {
      hi = t1;
    }
    buf ^= 1;
  }
  const uint32_t T = static_cast<uint32_t>(lo);
  // keys strictly above T (all kept), then `need` keys equal to T, lowest index first
  uint32_t gt = 0u;
#pragma unroll
  for (int i = 0; i < KPT; ++i) gt += ((valid >> i) & 1u) && key[i] > T ? 1u : 0u;
  gt = __reduce_add_sync(0xFFFFFFFFu, gt);
  if (lane == 0) wcnt[buf][warp][0] = gt;
  __syncthreads();
  const uint32_t n_gt = __reduce_add_sync(0xFFFFFFFFu, wcnt[buf][lane][0]);
  const uint32_t need = static_cast<uint32_t>(k) - n_gt;

  uint32_t eq_seen = 0u, written = 0u;
#pragma unroll
  for (int i = 0; i < KPT; ++i) {
    const int64_t j = tid + static_cast<int64_t>(i) * kTopkThreads;
    if (static_cast<int64_t>(i) * kTopkThreads >= d) break;  // block-uniform
    const bool in = (valid >> i) & 1u;
    const bool eq = in && key[i] == T;
    uint32_t eq_total;
    const uint32_t eq_rank = eq_seen + block_flag_scan(eq, warp_cnt, &eq_total);
    const bool sel = in && (key[i] > T || (eq && eq_rank < need));
    uint32_t sel_total;
    const uint32_t pos = written + block_flag_scan(sel, warp_cnt, &sel_total);
    if (sel) out[pos] = static_cast<int32_t>(j);
    eq_seen += eq_total;
    written += sel_total;
  }
}

constexpr int64_t kMaxStagedBytes = 200 * 1024;

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k, int32_t* idx,
                        int64_t ld_idx, cudaStream_t stream) {
  const unsigned grid = static_cast<unsigned>(batch);
  if (d <= 1 * kTopkThreads) {
    return launch_pdl(topk_search_kernel<1>, dim3(grid), dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx,
                      ld_idx);
  }
  if (d <= 2 * kTopkThreads) {
    return launch_pdl(topk_search_kernel<2>, dim3(grid), dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx,
                      ld_idx);
  }
  if (d <= 4 * kTopkThreads) {
    return launch_pdl(topk_search_kernel<4>, dim3(grid), dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx,
                      ld_idx);
  }
  if (d <= 8 * kTopkThreads) {
    return launch_pdl(topk_search_kernel<8>, dim3(grid), dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx,
                      ld_idx);
  }
  if (d <= 16 * kTopkThreads) {
    return launch_pdl(topk_search_kernel<16>, dim3(grid), dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx,
                      ld_idx);
  }
  const int64_t bytes = d * 4;
  if (bytes <= kMaxStagedBytes) {
    if (bytes > 48 * 1024) {
      const cudaError_t e = cudaFuncSetAttribute(topk_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                                 static_cast<int>(kMaxStagedBytes));
      if (e != cudaSuccess) return e;
    }
    return launch_pdl(topk_kernel<true>, dim3(grid), dim3(kTopkThreads), static_cast<size_t>(bytes), stream, scores,
                      d, ld_s, k, idx, ld_idx);
  }
  return launch_pdl(topk_kernel<false>, dim3(grid), dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx, ld_idx);
}

}  // namespace rmm
