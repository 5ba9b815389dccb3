// rmm_compact.cu — the reduced operands of A_{:,I} B_{I,:} (Reduced Matrix
// Multiplication technical summary, Metodología › Mecanismo Central):
//   compact_kernel      A_I[:, r] = A[:, I_r]   (column gather of the activation)
//   gather_rows_kernel  B_I[r, :] = B[I_r, :]   (row gather of the weight)
//
// HBM-bound gather.  Each thread produces 8 consecutive output columns (one
// 16-byte store for bf16) of each of 8 rows: it reads its 8 indices once,
// gathers the source elements through the read-only cache (the kept indices
// are increasing, so a warp's 256 gathers cover a short run of the source row
// and reuse its sectors), and writes them with vector stores.
#include <cuda_bf16.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

constexpr int kCompactThreads = 256;
constexpr int kPerThread = 8;
constexpr int kRowsPerCta = 8;
constexpr int64_t kColsPerCta = kCompactThreads * kPerThread;

// A CTA covers 2048 output columns of 8 consecutive rows: each thread reads
// its 8 indices once and gathers them from every row, so several rows'
// gathers are in flight together.
template <typename T>
__device__ __forceinline__ void compact_block(int64_t blk, const T* __restrict__ A, int64_t M, int64_t d, int64_t lda,
                                              const int32_t* __restrict__ idx, int64_t k, T* __restrict__ AI,
                                              int64_t ld_ai, int64_t chunks, bool vec_ok, unsigned* err) {
  const int64_t row0 = (blk / chunks) * kRowsPerCta;
  const int64_t chunk = blk % chunks;
  const int64_t c0 = chunk * kColsPerCta + static_cast<int64_t>(threadIdx.x) * kPerThread;
  if (row0 >= M || c0 >= k) return;
  int32_t j[kPerThread];
  bool bad = false;
#pragma unroll
  for (int e = 0; e < kPerThread; ++e) {
    j[e] = -1;
    if (c0 + e < k) {
      const int32_t v = __ldg(idx + c0 + e);
      if (v >= 0 && v < d) {
        j[e] = v;
      } else {
        bad = true;
      }
    }
  }
  if (bad) record_error(err, kDevErrBadIndex);
  const bool full = vec_ok && c0 + kPerThread <= k;
#pragma unroll 4
  for (int rr = 0; rr < kRowsPerCta; ++rr) {
    const int64_t row = row0 + rr;
    if (row >= M) break;
    const T* a = A + row * lda;
    T* o = AI + row * ld_ai + c0;
    alignas(16) T v[kPerThread];
#pragma unroll
    for (int e = 0; e < kPerThread; ++e) v[e] = j[e] >= 0 ? __ldg(a + j[e]) : T(0.f);
    if (full) {
      if constexpr (sizeof(T) == 2) {
        *reinterpret_cast<uint4*>(o) = *reinterpret_cast<const uint4*>(v);
      } else {
        reinterpret_cast<float4*>(o)[0] = *reinterpret_cast<const float4*>(&v[0]);
        reinterpret_cast<float4*>(o)[1] = *reinterpret_cast<const float4*>(&v[4]);
      }
    } else {
#pragma unroll
      for (int e = 0; e < kPerThread; ++e)
        if (c0 + e < k) o[e] = v[e];
    }
  }
}

template <typename T>
__global__ void __launch_bounds__(kCompactThreads) compact_kernel(const T* __restrict__ A, int64_t M, int64_t d,
                                                                  int64_t lda, const int32_t* __restrict__ idx,
                                                                  int64_t k, T* __restrict__ AI, int64_t ld_ai,
                                                                  int64_t chunks, bool vec_ok, unsigned* err) {
  pdl_wait();
  pdl_trigger();
  compact_block<T>(blockIdx.x, A, M, d, lda, idx, k, AI, ld_ai, chunks, vec_ok, err);
}

// One CTA per kept row: the row I_r of B is copied whole with 16-byte loads and
// stores, four in flight per thread (rows are contiguous, so this is a pure
// streaming copy); a row length that is not a multiple of 16 bytes ends with
// 2-byte copies.  Out-of-range indices produce a zero row and are flagged.
constexpr int kGatherThreads = 256;
static_assert(kGatherThreads == kCompactThreads, "the fused kernel runs compaction blocks at the gather block size");

__device__ __forceinline__ void gather_row_block(int64_t r, const uint4* __restrict__ B, int64_t d, int64_t vecs,
                                                 int64_t tail_halves, int64_t ldb_vec,
                                                 const int32_t* __restrict__ idx, int64_t k,
                                                 uint4* __restrict__ BI, int64_t ldbi_vec, unsigned* err) {
  if (r >= k) return;
  const int32_t j = __ldg(idx + r);
  uint4* dst = BI + r * ldbi_vec;
  if (j < 0 || j >= d) {
    if (threadIdx.x == 0) record_error(err, kDevErrBadIndex);
    for (int64_t v = threadIdx.x; v < vecs; v += kGatherThreads) dst[v] = make_uint4(0, 0, 0, 0);
    if (threadIdx.x < tail_halves) reinterpret_cast<uint16_t*>(dst + vecs)[threadIdx.x] = 0;
    return;
  }
  const uint4* src = B + static_cast<int64_t>(j) * ldb_vec;
  if (threadIdx.x < tail_halves)  // bytes past the last whole 16-byte vector of the row
    reinterpret_cast<uint16_t*>(dst + vecs)[threadIdx.x] = reinterpret_cast<const uint16_t*>(src + vecs)[threadIdx.x];
  int64_t v = threadIdx.x;
  for (; v + 3 * kGatherThreads < vecs; v += 4 * kGatherThreads) {
    const uint4 a0 = __ldcs(src + v);
    const uint4 a1 = __ldcs(src + v + kGatherThreads);
    const uint4 a2 = __ldcs(src + v + 2 * kGatherThreads);
    const uint4 a3 = __ldcs(src + v + 3 * kGatherThreads);
    dst[v] = a0;
    dst[v + kGatherThreads] = a1;
    dst[v + 2 * kGatherThreads] = a2;
    dst[v + 3 * kGatherThreads] = a3;
  }
  for (; v < vecs; v += kGatherThreads) dst[v] = __ldcs(src + v);
}

__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(const uint4* __restrict__ B, int64_t d,
                                                                       int64_t vecs, int64_t tail_halves,
                                                                       int64_t ldb_vec, const int32_t* __restrict__ idx,
                                                                       int64_t k, uint4* __restrict__ BI,
                                                                       int64_t ldbi_vec, unsigned* err) {
  pdl_wait();
  pdl_trigger();
  gather_row_block(blockIdx.x, B, d, vecs, tail_halves, ldb_vec, idx, k, BI, ldbi_vec, err);
}

// Both reduced operands in one grid: blocks [0, k) gather the kept rows of B,
// the remaining blocks compact the kept columns of A (bf16), so the two HBM
// streams overlap.
__global__ void __launch_bounds__(kGatherThreads) compact_gather_kernel(
    const uint4* __restrict__ B, int64_t d, int64_t vecs, int64_t tail_halves, int64_t ldb_vec,
    uint4* __restrict__ BI, int64_t ldbi_vec, const __nv_bfloat16* __restrict__ A, int64_t M, int64_t lda,
    __nv_bfloat16* __restrict__ AI, int64_t ld_ai, int64_t chunks, bool vec_ok, const int32_t* __restrict__ idx,
    int64_t k, unsigned* err) {
  pdl_wait();
  pdl_trigger();
  const int64_t blk = blockIdx.x;
  if (blk < k) {
    gather_row_block(blk, B, d, vecs, tail_halves, ldb_vec, idx, k, BI, ldbi_vec, err);
  } else {
    compact_block<__nv_bfloat16>(blk - k, A, M, d, lda, idx, k, AI, ld_ai, chunks, vec_ok, err);
  }
}

}  // namespace

cudaError_t launch_gather_rows(const void* B, int64_t d, int64_t row_bytes, int64_t ldb_bytes, const int32_t* idx,
                               int64_t k, void* B_I, int64_t ldbi_bytes, unsigned* err, cudaStream_t stream) {
  if (k == 0 || row_bytes == 0) return cudaSuccess;
  if (k > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  return launch_pdl(gather_rows_kernel, dim3(static_cast<unsigned>(k)), dim3(kGatherThreads), 0, stream,
                    static_cast<const uint4*>(B), d, row_bytes / 16, (row_bytes % 16) / 2, ldb_bytes / 16, idx, k,
                    static_cast<uint4*>(B_I), ldbi_bytes / 16, err);
}

cudaError_t launch_compact(const void* A, int dtype, int64_t M, int64_t d, int64_t lda, const int32_t* idx,
                           int64_t k, void* A_I, int64_t ld_ai, unsigned* err, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const int64_t chunks = (k + kColsPerCta - 1) / kColsPerCta;
  const int64_t blocks = ((M + kRowsPerCta - 1) / kRowsPerCta) * chunks;
  const size_t elt = dtype == 1 ? 2 : 4;
  const bool vec_ok = reinterpret_cast<uintptr_t>(A_I) % 16 == 0 && (ld_ai * elt) % 16 == 0;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  if (dtype == 1)
    return launch_pdl(compact_kernel<__nv_bfloat16>, dim3(static_cast<unsigned>(blocks)), dim3(kCompactThreads), 0,
                      stream, static_cast<const __nv_bfloat16*>(A), M, d, lda, idx, k,
                      static_cast<__nv_bfloat16*>(A_I), ld_ai, chunks, vec_ok, err);
  return launch_pdl(compact_kernel<float>, dim3(static_cast<unsigned>(blocks)), dim3(kCompactThreads), 0, stream,
                    static_cast<const float*>(A), M, d, lda, idx, k, static_cast<float*>(A_I), ld_ai, chunks, vec_ok,
                    err);
}

cudaError_t launch_compact_and_gather(const void* A, int64_t M, int64_t d, int64_t lda, const void* B, int64_t N,
                                      int64_t ldb, const int32_t* idx, int64_t k, void* A_I, int64_t ld_ai,
                                      void* B_I, int64_t ld_bi, unsigned* err, cudaStream_t stream) {
  const int64_t chunks = (k + kColsPerCta - 1) / kColsPerCta;
  const int64_t cblocks = M > 0 ? ((M + kRowsPerCta - 1) / kRowsPerCta) * chunks : 0;
  const int64_t blocks = k + cblocks;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const bool vec_ok = reinterpret_cast<uintptr_t>(A_I) % 16 == 0 && (ld_ai * 2) % 16 == 0;
  const int64_t row_bytes = N * 2;
  return launch_pdl(compact_gather_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kGatherThreads), 0, stream,
                    static_cast<const uint4*>(B), d, row_bytes / 16, (row_bytes % 16) / 2, ldb * 2 / 16,
                    static_cast<uint4*>(B_I), ld_bi * 2 / 16, static_cast<const __nv_bfloat16*>(A), M, lda,
                    static_cast<__nv_bfloat16*>(A_I), ld_ai, chunks, vec_ok, idx, k, err);
}

}  // namespace rmm
