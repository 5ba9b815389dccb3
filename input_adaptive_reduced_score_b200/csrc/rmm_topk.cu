// rmm_topk.cu — deterministic top-k index selection (Reduced Matrix
// Multiplication technical summary, Metodología › Estrategia de Selección:
// keep the k indices with the highest scores).  The tie rule (lowest index
// first) and the ascending output order are this library's reading.
//
// One CTA per score row; scores are mapped to order-preserving uint32 keys.
// Rows of up to 51200 scores are staged once in shared memory and selected
// by a histogram search: the key range [min, max] is cut into 2048 bins,
// the bin holding the k-th largest key becomes the new range, and the search
// stops when the range is a single key (at most three rounds for 32-bit
// keys) or when the keys at or above the range's start are exactly k.  Each
// round costs three block barriers.  The selected indices are then written in
// ascending order in one sweep: each warp owns a contiguous block of indices,
// one barrier exchanges the warps' counts, and ballots place each index.
// Longer rows use a 4-pass MSB-first radix select that re-reads the scores
// from global memory.  Integer work only: the result is the unique set
// defined by the rule.
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

constexpr int64_t kMaxStagedKeys = 51200;  // 200 KB of keys + 8 KB of bins per CTA

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
  const uint32_t k = static_cast<uint32_t>(k64);
  const float* s = scores + static_cast<int64_t>(blockIdx.x) * ld_s;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.x) * ld_idx;
  const int tid = threadIdx.x;
  const bool vec4 = (reinterpret_cast<uintptr_t>(s) & 15u) == 0 && (d & 3) == 0;
  pdl_wait();
  pdl_trigger();

  // stage the keys, zero the bins, find the key range; the loads of a batch
  // are all issued before the first is used (one memory round trip per batch)
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  if (vec4) {
    const int nv = d >> 2;
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
  } else {
    for (int j0 = tid; j0 < d; j0 += 8 * NT) {
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
  select_staged<NT>(keys, d, k, kmin, kmax, out);
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

bool allow_select_rows() {
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = 1ull << dev;
  if (configured.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(select_rows_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMaxStagedKeys * 4)) != cudaSuccess)
    return false;
  configured.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

// Opt the histogram kernel into kMaxStagedKeys * 4 bytes of dynamic shared
// memory, once per device.
template <int NT>
bool allow_staged_rows() {
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = 1ull << dev;
  if (configured.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(topk_hist_kernel<NT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                           static_cast<int>(kMaxStagedKeys * 4)) != cudaSuccess)
    return false;
  configured.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

}  // namespace

bool select_rows_supported(int64_t M, int64_t d) { return M >= 1 && M <= 16 && d >= 1 && d <= kMaxStagedKeys; }

cudaError_t launch_select_rows(const void* A, int64_t M, int64_t d, int64_t lda, int64_t k, int32_t* idx, float* ss,
                               void* A_I, int64_t ld_ai, cudaStream_t stream) {
  const size_t bytes = static_cast<size_t>(d) * 4;
  if (bytes > 48 * 1024 && !allow_select_rows()) return cudaErrorInvalidValue;
  return launch_pdl(select_rows_kernel, dim3(1), dim3(1024), bytes, stream, static_cast<const uint16_t*>(A),
                    static_cast<int>(M), d, lda, k, idx, ss, static_cast<uint16_t*>(A_I), ld_ai);
}

cudaError_t launch_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k, int32_t* idx,
                        int64_t ld_idx, cudaStream_t stream) {
  const dim3 grid(static_cast<unsigned>(batch));
  if (d <= kMaxStagedKeys) {
    const size_t bytes = static_cast<size_t>(d) * 4;
    if (d <= 2048)  // 8 KB of keys: no opt-in needed
      return launch_pdl(topk_hist_kernel<256>, grid, dim3(256), bytes, stream, scores, d, ld_s, k, idx, ld_idx);
    if (bytes > 48 * 1024 && !allow_staged_rows<1024>()) return cudaErrorInvalidValue;
    return launch_pdl(topk_hist_kernel<1024>, grid, dim3(1024), bytes, stream, scores, d, ld_s, k, idx, ld_idx);
  }
  return launch_pdl(topk_radix_kernel, grid, dim3(kTopkThreads), 0, stream, scores, d, ld_s, k, idx, ld_idx);
}

}  // namespace rmm
