// rmm_topk.cu — deterministic top-k index selection (Reduced Matrix
// Multiplication technical summary, Metodología › Estrategia de Selección:
// keep the k indices with the highest scores).  The tie rule (lowest index
// first) and the ascending output order are this library's reading.
//
// One 1024-thread CTA per score row.  Scores are mapped to order-preserving
// uint32 keys.  A 4-pass MSB-first radix select (8-bit digits, shared-memory
// histograms) finds the exact key T of the k-th largest score and how many
// keys equal to T must be kept.  A final ordered sweep emits, in ascending
// index order, every index with key > T and the first `need` indices with
// key == T, using warp ballots and a block-wide scan for output positions.
// Integer work only: the result is the unique set defined by the rule.
#include "rmm_internal.h"

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

__global__ void __launch_bounds__(kTopkThreads) topk_kernel(const float* __restrict__ scores, int64_t d,
                                                             int64_t ld_s, int64_t k, int32_t* __restrict__ idx,
                                                             int64_t ld_idx) {
  __shared__ uint32_t hist[256];
  __shared__ uint32_t warp_cnt[33];
  __shared__ uint32_t sh_prefix, sh_need;
  const float* s = scores + static_cast<int64_t>(blockIdx.x) * ld_s;
  int32_t* out = idx + static_cast<int64_t>(blockIdx.x) * ld_idx;
  const int tid = threadIdx.x, lane = tid & 31;

  uint32_t prefix = 0u, mask = 0u, need = static_cast<uint32_t>(k);
  for (int pass = 0; pass < 4; ++pass) {
    const int shift = 24 - 8 * pass;
    if (tid < 256) hist[tid] = 0u;
    __syncthreads();
    for (int64_t j = tid; j < d; j += kTopkThreads) {
      const uint32_t key = score_key(__ldg(s + j));
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
    const uint32_t key = j < d ? score_key(__ldg(s + j)) : 0u;
    const bool in = j < d;
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
  (void)lane;
}

}  // namespace

cudaError_t launch_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k, int32_t* idx,
                        int64_t ld_idx, cudaStream_t stream) {
  topk_kernel<<<static_cast<unsigned>(batch), kTopkThreads, 0, stream>>>(scores, d, ld_s, k, idx, ld_idx);
  return cudaGetLastError();
}

}  // namespace rmm
