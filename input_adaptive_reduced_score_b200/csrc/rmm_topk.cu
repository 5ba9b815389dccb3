// rmm_topk.cu — deterministic top-k index selection (Reduced Matrix
// Multiplication technical summary, Metodología › Estrategia de Selección:
// keep the k indices with the highest scores).  The tie rule (lowest index
// first) and the ascending output order are this library's reading.
//
// Scores are mapped to order-preserving uint32 keys and staged in shared
// memory (up to 51200 per CTA), where the histogram search of rmm_select.cuh
// finds the k-th largest key in at most three rounds and writes the selected
// indices in ascending order.  A row takes one CTA of 1024 threads, or a
// cluster of 2, 4 or 8 CTAs of 512 threads that each stage a consecutive
// slice of at least 4096 keys, when the rows are too few to fill the SMs or
// a row is too long for one CTA's shared memory; rows longer than eight
// slices take a 4-pass MSB-first radix select that re-reads the scores from
// global memory.  (Measured on B200, back-to-back calls: one 4096-score row
// takes 7.5 us on one CTA and 9-17 us on clusters, where the cluster
// barriers and remote reads cost about 1-2 thousand cycles per round; 32
// rows of 32768 take 17.2 us on one CTA each and 13.6 us on clusters of 4;
// with 1024-thread cluster CTAs every short phase costs 32 warps of issue.)  Integer work only: the result is the unique
// set defined by the rule.
#include <algorithm>
#include <atomic>

#include "rmm_internal.h"
#include "rmm_launch.cuh"
#include "rmm_select.cuh"

namespace rmm {
namespace {

constexpr int kTopkThreads = 1024;

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

// Rows too long to stage: 4-pass radix select over keys re-read from global
// memory (8-bit digits, shared-memory histograms).
__global__ void __launch_bounds__(kTopkThreads) topk_radix_kernel(const float* __restrict__ scores, int64_t d,
                                                             int64_t ld_s, int64_t k, int32_t* __restrict__ idx,
                                                             int64_t ld_idx) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_cnt[33];
  __shared__ uint32_t sh_prefix, sh_need;
  const float* s = scores + static_cast<int64_t>(blockIdx.x) * ld_s;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.x) * ld_idx;
  const int tid = threadIdx.x, lane = tid & 31;
  pdl_wait();
  pdl_trigger();

  auto key_at = [&](int64_t j) -> uint32_t { return score_key(__ldg(s + j)); };

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

constexpr int64_t kMaxStagedKeys = 51200;  // 200 KB of keys + 8 KB (16 KB in a cluster) of bins per CTA
constexpr int kMaxTopkCluster = 8;          // CTAs per row (the portable cluster size)
constexpr int64_t kMinClusterSlice = 4096;   // keys per CTA below which a row is not split further
constexpr int kClusterThreads = 512;         // threads of a cluster CTA

// The staged search with this file's static bins, writing the k selected
// indices, ascending, to out.
template <int NT>
__device__ __forceinline__ void select_staged(uint32_t* keys, int d, uint32_t k, uint32_t kmin, uint32_t kmax,
                                              int32_t* __restrict__ out) {
  __shared__ __align__(16) uint32_t hist[kSelectBins];
  select_staged_keys<NT>(keys, d, k, kmin, kmax, hist, [&](uint32_t pos, int j) { out[pos] = j; });
}

// One score row per CTA: stage its keys, then select_staged.
template <int NT>
__global__ void __launch_bounds__(NT, 1) topk_hist_kernel(const float* __restrict__ scores, int64_t d64, int64_t ld_s,
                                                           int64_t k64, int32_t* __restrict__ idx, int64_t ld_idx) {
  extern __shared__ __align__(16) uint32_t keys[];
  const int d = static_cast<int>(d64);
  const float* s = scores + static_cast<int64_t>(blockIdx.x) * ld_s;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.x) * ld_idx;
  pdl_wait();
  pdl_trigger();
  uint32_t kmin, kmax;
  stage_score_keys<NT>(s, d, keys, kmin, kmax);
  select_staged<NT>(keys, d, static_cast<uint32_t>(k64), kmin, kmax, out);
}

// One score row per cluster of C CTAs (grid x = the cluster, y = the row):
// CTA r stages scores [r * slice, (r + 1) * slice) and writes its selected
// indices at their places in the row's ascending list.
template <int NT, int C>
__global__ void __launch_bounds__(NT, 1)
    topk_cluster_kernel(const float* __restrict__ scores, int64_t d64, int64_t ld_s, int64_t k64,
                        int32_t* __restrict__ idx, int64_t ld_idx, int slice) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ __align__(16) uint32_t hist[2 * kSelectBins];
  const int d = static_cast<int>(d64);
  const int j0 = static_cast<int>(blockIdx.x) * slice;
  const int dl = max(0, min(slice, d - j0));
  const float* s = scores + static_cast<int64_t>(blockIdx.y) * ld_s + j0;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.y) * ld_idx;
  pdl_wait();
  pdl_trigger();
  uint32_t kmin, kmax;
  stage_score_keys<NT>(s, dl, keys, kmin, kmax);
  const StagedSelection sel = select_staged_compact<NT, C>(keys, dl, static_cast<uint32_t>(k64), kmin, kmax, hist);
  for (int q = threadIdx.x; q < static_cast<int>(sel.count); q += NT)
    out[sel.base + q] = j0 + static_cast<int32_t>(keys[q]);
  cluster_wait();  // no CTA leaves while another may still read its shared memory
}

// A few activation rows (decode): column scores of A [M x d], the top-k
// selection and the compaction A_I = A[:, I] in one CTA of 1024 threads.
// Scores are fp32 sums of the rows' exact squares in row order.  Optional
// ss output.  keys in dynamic shared memory (d words, d <= kMaxStagedKeys).
__global__ void __launch_bounds__(1024, 1)
    select_rows_kernel(const uint16_t* __restrict__ A, int M, int64_t d64, int64_t lda, int64_t k64,
                       int32_t* __restrict__ idx, float* __restrict__ ss, uint16_t* __restrict__ AI, int64_t ld_ai) {
  extern __shared__ __align__(16) uint32_t keys[];
  const int d = static_cast<int>(d64);
  const int tid = threadIdx.x;
  pdl_wait();
  pdl_trigger();
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  const bool vec = (reinterpret_cast<uintptr_t>(A) & 15u) == 0 && (lda & 7) == 0 && (d & 7) == 0;
  if (vec) {
    for (int v = tid; v < d / 8; v += 1024) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int m = 0; m < M; ++m) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(A + static_cast<int64_t>(m) * lda) + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float lo = __uint_as_float(w[t] << 16), hi = __uint_as_float(w[t] & 0xFFFF0000u);
          acc[2 * t] = fmaf(lo, lo, acc[2 * t]);
          acc[2 * t + 1] = fmaf(hi, hi, acc[2 * t + 1]);
        }
      }
#pragma unroll
      for (int e = 0; e < 8; ++e) {
        const uint32_t key = score_key(acc[e]);
        keys[8 * v + e] = key;
        kmin = min(kmin, key);
        kmax = max(kmax, key);
        if (ss) ss[8 * v + e] = acc[e];
      }
    }
  } else {
    for (int j = tid; j < d; j += 1024) {
      float acc = 0.f;
      for (int m = 0; m < M; ++m) {
        const float x = __uint_as_float(static_cast<uint32_t>(A[static_cast<int64_t>(m) * lda + j]) << 16);
        acc = fmaf(x, x, acc);
      }
      const uint32_t key = score_key(acc);
      keys[j] = key;
      kmin = min(kmin, key);
      kmax = max(kmax, key);
      if (ss) ss[j] = acc;
    }
  }
  const uint32_t k = static_cast<uint32_t>(k64);
  select_staged<1024>(keys, d, k, kmin, kmax, idx);
  __syncthreads();  // this block's index writes are visible to all its threads
  // idx was written by this kernel: read it with coherent loads, not through
  // the read-only path
  for (int64_t e = tid; e < static_cast<int64_t>(M) * k; e += 1024) {
    const int m = static_cast<int>(e / k);
    const int64_t r = e % k;
    AI[m * ld_ai + r] = A[static_cast<int64_t>(m) * lda + idx[r]];
  }
}

// Opt a kernel into `bytes` of dynamic shared memory, once per device.
template <auto Kernel>
bool allow_smem_once(size_t bytes) {
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = 1ull << dev;
  if (configured.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(bytes)) !=
      cudaSuccess)
    return false;
  configured.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

template <int NT, int C>
cudaError_t launch_topk_cluster(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k, int32_t* idx,
                                int64_t ld_idx, int slice, cudaStream_t stream) {
  if (!allow_smem_once<topk_cluster_kernel<NT, C>>(kMaxStagedKeys * 4)) return cudaErrorInvalidValue;
  return launch_pdl_cluster(topk_cluster_kernel<NT, C>, dim3(C, static_cast<unsigned>(batch)), dim3(NT),
                            static_cast<size_t>(slice) * 4, C, stream, scores, d, ld_s, k, idx, ld_idx, slice);
}

}  // namespace

int topk_cluster_size(int64_t batch, int64_t d) {
  // a cluster launch puts the rows on grid y (at most 65535 of them)
  if (batch > 65535) return d <= kMaxStagedKeys ? 1 : 0;
  const int64_t sms = std::max(device_sm_count(), 1);
  int c = 1;
  // split while the clusters still fit the SMs and each slice keeps at
  // least kMinClusterSlice keys; a slice must fit the staging limit
  while (c < kMaxTopkCluster && batch * 2 * c <= sms && d / (2 * c) >= kMinClusterSlice) c *= 2;
  while (c < kMaxTopkCluster && (d + c - 1) / c > kMaxStagedKeys) c *= 2;
  return (d + c - 1) / c > kMaxStagedKeys ? 0 : c;
}

int topk_cluster_slice(int64_t d, int c) { return static_cast<int>(((d + c - 1) / c + 3) / 4 * 4); }

bool select_rows_supported(int64_t M, int64_t d) { return M >= 1 && M <= 16 && d >= 1 && d <= kMaxStagedKeys; }

cudaError_t launch_select_rows(const void* A, int64_t M, int64_t d, int64_t lda, int64_t k, int32_t* idx, float* ss,
                               void* A_I, int64_t ld_ai, cudaStream_t stream) {
  const size_t bytes = static_cast<size_t>(d) * 4;
  if (bytes > 48 * 1024 && !allow_smem_once<select_rows_kernel>(kMaxStagedKeys * 4)) return cudaErrorInvalidValue;
  return launch_pdl(select_rows_kernel, dim3(1), dim3(1024), bytes, stream, static_cast<const uint16_t*>(A),
                    static_cast<int>(M), d, lda, k, idx, ss, static_cast<uint16_t*>(A_I), ld_ai);
}

cudaError_t launch_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k, int32_t* idx,
                        int64_t ld_idx, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(batch));
  if (d <= 2048)  // 8 KB of keys: no opt-in needed
    return launch_pdl(topk_hist_kernel<256>, grid, dim3(256), static_cast<size_t>(d) * 4, stream, scores, d, ld_s,
                      k, idx, ld_idx);
  const int c = topk_cluster_size(batch, d);
  const int slice = c > 0 ? topk_cluster_slice(d, c) : 0;
  switch (c) {
    case 1: {
      const size_t bytes = static_cast<size_t>(d) * 4;
      if (bytes > 48 * 1024 && !allow_smem_once<topk_hist_kernel<1024>>(kMaxStagedKeys * 4))
        return cudaErrorInvalidValue;
      return launch_pdl(topk_hist_kernel<1024>, grid, dim3(1024), bytes, stream, scores, d, ld_s, k, idx, ld_idx);
    }
    case 2: return launch_topk_cluster<kClusterThreads, 2>(scores, batch, d, ld_s, k, idx, ld_idx, slice, stream);
    case 4: return launch_topk_cluster<kClusterThreads, 4>(scores, batch, d, ld_s, k, idx, ld_idx, slice, stream);
    case 8: return launch_topk_cluster<kClusterThreads, 8>(scores, batch, d, ld_s, k, idx, ld_idx, slice, stream);
    default: break;
  }
  return launch_pdl(topk_radix_kernel, grid, dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx, ld_idx);
}

}  // namespace rmm
