// rmm_compact.cu — the reduced operands of A_{:,I} B_{I,:} (Reduced Matrix
// Multiplication technical summary, Metodología › Mecanismo Central):
//   A_I[:, r] = A[:, I_r]   (column gather of the activation)
//   B_I[r, :] = B[I_r, :]   (row gather of the weight)
//
// HBM-bound gathers.
//  - bf16 A with 16-byte aligned rows: a block copies R whole rows of A into
//    shared memory with one bulk copy per row (the copy engine reads them at
//    full width); then the lanes of a warp take 32 consecutive output
//    columns, read their sources from shared memory (increasing and close
//    together, so without bank conflicts) and store 64 contiguous bytes.
//    R is chosen so a block stages about 32 KB.
//  - other layouts: each thread gathers its 8 output columns of 8 rows
//    straight from global memory through the read-only cache.
//  - B rows are whole contiguous rows: one block per kept row streams it with
//    16-byte loads and stores.  An int8 B (weight-only quantisation) is
//    widened to exact bf16 values on the way; its scales are applied by the
//    product.
#include <cuda_bf16.h>

#include <atomic>

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

// Staged compaction of R rows (bf16).  The caller guarantees: A and every row
// start 16-byte aligned (lda a multiple of 8), d a multiple of 8, R * 2d bytes
// of dynamic shared memory.
constexpr int kStageTargetBytes = 32 * 1024;
constexpr int64_t kMaxStagedRowBytes = 200 * 1024;

__device__ __forceinline__ void compact_rows_block(int64_t blk, const uint16_t* __restrict__ A, int64_t M, int64_t d,
                                                   int64_t lda, const int32_t* __restrict__ idx, int64_t k,
                                                   uint16_t* __restrict__ AI, int64_t ld_ai, int R, unsigned* err,
                                                   uint8_t* stage) {
  __shared__ uint64_t bar;
  __shared__ int abort_flag;
  const int64_t row0 = blk * R;
  if (row0 >= M) return;  // block-uniform
  const int rows = static_cast<int>(min(static_cast<int64_t>(R), M - row0));
  const uint32_t row_bytes = static_cast<uint32_t>(2 * d);
  const uint32_t sbase = smem_u32(stage);
  const uint32_t b = smem_u32(&bar);
  if (threadIdx.x == 0) {
    abort_flag = 0;
    mbar_init(b, 1);
    fence_mbar_init();
    mbar_arrive_expect_tx(b, static_cast<uint32_t>(rows) * row_bytes);
    for (int r = 0; r < rows; ++r) bulk_load_1d(sbase + r * row_bytes, A + (row0 + r) * lda, row_bytes, b);
  }
  __syncthreads();
  const uint16_t* srows = reinterpret_cast<const uint16_t*>(stage);
  bool landed = false;
  // Output columns in chunks of 2048: thread t writes columns
  // cbase + i*256 + t (i < 8), so a warp's 32 lanes handle 32 consecutive
  // output columns, whose sources are increasing and close together in the
  // staged row (conflict-free shared-memory reads, 64-byte stores).  The
  // indices of the next chunk are loaded before the current chunk's stores.
  auto load_idx = [&](int64_t cbase, int32_t (&j)[kPerThread]) {
    bool bad = false;
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) {
      const int64_t c = cbase + i * kCompactThreads + threadIdx.x;
      j[i] = -2;  // no such output column
      if (c < k) {
        const int32_t v = __ldg(idx + c);
        if (v >= 0 && v < d) {
          j[i] = v;
        } else {
          j[i] = -1;
          bad = true;
        }
      }
    }
    if (bad) record_error(err, kDevErrBadIndex);
  };
  int32_t jn[kPerThread];
  load_idx(0, jn);
  for (int64_t cbase = 0; cbase < k; cbase += kColsPerCta) {
    int32_t j[kPerThread];
#pragma unroll
    for (int i = 0; i < kPerThread; ++i) j[i] = jn[i];
    if (cbase + kColsPerCta < k) load_idx(cbase + kColsPerCta, jn);
    if (!landed) {
      // bounded wait; on expiry the site is recorded and no row is written
      if (!mbar_wait(b, 0, &abort_flag, err, 61)) break;
      landed = true;
    }
    for (int r = 0; r < rows; ++r) {
      const uint16_t* sr = srows + static_cast<int64_t>(r) * d;
      uint16_t* o = AI + (row0 + r) * ld_ai + cbase + threadIdx.x;
#pragma unroll
      for (int i = 0; i < kPerThread; ++i)
        if (j[i] != -2) o[i * kCompactThreads] = j[i] >= 0 ? sr[j[i]] : static_cast<uint16_t>(0);
    }
  }
  // thread 0 always has an output column, so it has waited for the copies;
  // after an expired wait it waits once more, briefly, before the block retires
  if (!landed && threadIdx.x == 0) wait_drain(b, 0);
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

__global__ void __launch_bounds__(kCompactThreads) compact_staged_kernel(const uint16_t* __restrict__ A, int64_t M,
                                                                         int64_t d, int64_t lda,
                                                                         const int32_t* __restrict__ idx, int64_t k,
                                                                         uint16_t* __restrict__ AI, int64_t ld_ai,
                                                                         int R, unsigned* err) {
  extern __shared__ __align__(128) uint8_t stage[];
  pdl_wait();
  pdl_trigger();
  compact_rows_block(blockIdx.x, A, M, d, lda, idx, k, AI, ld_ai, R, err, stage);
}

// Kept rows of B, several per CTA when the copied slice of a row is short: CTA
// `blk` copies kept rows [blk * rpb, +rpb).  Their source rows are read once
// into shared memory; the (row, 16-byte vector) pairs are numbered row-major
// and thread t copies pairs t, t + 256, ... with four loads in flight, so a
// CTA moves at least ~16 KB however short the slice is (one CTA per row of a
// few KB left the copy bound by block turnover).  A slice length that is not
// a multiple of 16 bytes ends with 2-byte copies.  Out-of-range indices give
// zero rows and are flagged.  kW8: B is int8 (vectors of 16 values, widened
// to exact bf16: two 16-byte stores each; tail_elems trailing bytes); the
// per-column scales are applied later, in the product's epilogue.
constexpr int kGatherThreads = 256;
constexpr int kGatherMaxRows = 32;                // kept rows per CTA at most
constexpr int64_t kGatherTargetVecs = 1024;       // 16-byte source vectors per CTA (16 KB)
static_assert(kGatherThreads == kCompactThreads, "the fused kernel runs compaction blocks at the gather block size");

// Kept rows per gather CTA for rows of `vecs` 16-byte source vectors.
__host__ __device__ inline int gather_rows_per_block(int64_t vecs) {
  if (vecs >= kGatherTargetVecs) return 1;
  const int64_t r = kGatherTargetVecs / (vecs > 0 ? vecs : 1);
  return static_cast<int>(r < kGatherMaxRows ? r : kGatherMaxRows);
}

template <bool kW8>
__device__ __forceinline__ void gather_rows_block(int64_t blk, int rpb, const uint4* __restrict__ B, int64_t d,
                                                  int64_t vecs, int64_t tail_elems, int64_t ldb_vec,
                                                  const int32_t* __restrict__ idx, int64_t k,
                                                  uint4* __restrict__ BI, int64_t ldbi_vec, unsigned* err) {
  __shared__ int32_t src_row[kGatherMaxRows];
  const int64_t r0 = blk * rpb;
  if (r0 >= k) return;  // block-uniform
  const int nr = static_cast<int>(k - r0 < rpb ? k - r0 : rpb);
  if (threadIdx.x < nr) {
    const int32_t j = __ldg(idx + r0 + threadIdx.x);
    const bool ok = j >= 0 && j < d;
    if (!ok) record_error(err, kDevErrBadIndex);
    src_row[threadIdx.x] = ok ? j : -1;
  }
  __syncthreads();
  constexpr int OUT = kW8 ? 2 : 1;  // 16-byte output vectors per source vector
  auto put = [&](int64_t r, int64_t v, const uint4& q) {
    uint4* dst = BI + (r0 + r) * ldbi_vec + OUT * v;
    if constexpr (kW8) {
      const uint32_t w[4] = {q.x, q.y, q.z, q.w};
      uint32_t o[8];
#pragma unroll
      for (int e = 0; e < 4; ++e) {
        float f[4];
        i8x4_to_f32(w[e], f);
        o[2 * e] = pack_bf16x2(f[0], f[1]);
        o[2 * e + 1] = pack_bf16x2(f[2], f[3]);
      }
      dst[0] = make_uint4(o[0], o[1], o[2], o[3]);
      dst[1] = make_uint4(o[4], o[5], o[6], o[7]);
    } else {
      dst[0] = q;
    }
  };
  const int64_t items = static_cast<int64_t>(nr) * vecs;
  for (int64_t it = threadIdx.x; it < items; it += 4 * kGatherThreads) {
    uint4 a[4];
    int64_t rr[4], vv[4];
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int64_t i = it + u * kGatherThreads;
      rr[u] = i / vecs;
      vv[u] = i - rr[u] * vecs;
      const int32_t j = i < items ? src_row[rr[u]] : -1;
      a[u] = j >= 0 ? __ldcs(B + static_cast<int64_t>(j) * ldb_vec + vv[u]) : make_uint4(0, 0, 0, 0);
    }
#pragma unroll
    for (int u = 0; u < 4; ++u)
      if (it + u * kGatherThreads < items) put(rr[u], vv[u], a[u]);
  }
  // elements past the last whole 16-byte vector of each row
  for (int e = threadIdx.x; e < nr * tail_elems; e += kGatherThreads) {
    const int r = static_cast<int>(e / tail_elems), t = static_cast<int>(e % tail_elems);
    const int32_t j = src_row[r];
    if constexpr (kW8) {
      __nv_bfloat16* dst = reinterpret_cast<__nv_bfloat16*>(BI + (r0 + r) * ldbi_vec + 2 * vecs);
      dst[t] = __float2bfloat16_rn(
          j >= 0 ? static_cast<float>(reinterpret_cast<const int8_t*>(B + static_cast<int64_t>(j) * ldb_vec + vecs)[t])
                 : 0.f);
    } else {
      uint16_t* dst = reinterpret_cast<uint16_t*>(BI + (r0 + r) * ldbi_vec + vecs);
      dst[t] = j >= 0 ? reinterpret_cast<const uint16_t*>(B + static_cast<int64_t>(j) * ldb_vec + vecs)[t]
                      : static_cast<uint16_t>(0);
    }
  }
}

__global__ void __launch_bounds__(kGatherThreads) gather_rows_i8_kernel(const uint4* __restrict__ Bq, int64_t d,
                                                                          int64_t vecs, int64_t tail_bytes,
                                                                          int64_t ldb_vec,
                                                                          const int32_t* __restrict__ idx, int64_t k,
                                                                          uint4* __restrict__ BI, int64_t ldbi_vec,
                                                                          int rpb, unsigned* err) {
  pdl_wait();
  pdl_trigger();
  gather_rows_block<true>(blockIdx.x, rpb, Bq, d, vecs, tail_bytes, ldb_vec, idx, k, BI, ldbi_vec, err);
}

__global__ void __launch_bounds__(kGatherThreads) gather_rows_kernel(const uint4* __restrict__ B, int64_t d,
                                                                       int64_t vecs, int64_t tail_halves,
                                                                       int64_t ldb_vec, const int32_t* __restrict__ idx,
                                                                       int64_t k, uint4* __restrict__ BI,
                                                                       int64_t ldbi_vec, int rpb, unsigned* err) {
  pdl_wait();
  pdl_trigger();
  gather_rows_block<false>(blockIdx.x, rpb, B, d, vecs, tail_halves, ldb_vec, idx, k, BI, ldbi_vec, err);
}

// Both reduced operands in one grid: blocks [0, kb) gather the kept rows of B
// (rpb rows each), the remaining blocks compact the kept columns of A (bf16;
// staged R rows per block, or the direct gather of 8 rows x 2048 columns), so
// the two HBM streams overlap.
// kW8: B is int8 (vecs counts 16-value vectors, tail_elems trailing bytes)
// and B_I is written as bf16; otherwise B is bf16 (tail_elems trailing halves).
template <bool kStagedA, bool kW8>
__global__ void __launch_bounds__(kGatherThreads) compact_gather_kernel(
    const uint4* __restrict__ B, int64_t d, int64_t vecs, int64_t tail_elems, int64_t ldb_vec,
    uint4* __restrict__ BI, int64_t ldbi_vec, const uint16_t* __restrict__ A, int64_t M, int64_t lda,
    uint16_t* __restrict__ AI, int64_t ld_ai, int64_t chunks, int R, bool vec_ok, const int32_t* __restrict__ idx,
    int64_t k, int rpb, int64_t kb, unsigned* err, uint32_t* zero, int64_t n_zero) {
  extern __shared__ __align__(128) uint8_t stage[];
  pdl_wait();
  pdl_trigger();
  const int64_t blk = blockIdx.x;
  if (blk == 0)
    for (int64_t i = threadIdx.x; i < n_zero; i += kGatherThreads) zero[i] = 0u;
  if (blk < kb) {
    gather_rows_block<kW8>(blk, rpb, B, d, vecs, tail_elems, ldb_vec, idx, k, BI, ldbi_vec, err);
  } else if constexpr (kStagedA) {
    compact_rows_block(blk - kb, A, M, d, lda, idx, k, AI, ld_ai, R, err, stage);
  } else {
    compact_block<__nv_bfloat16>(blk - kb, reinterpret_cast<const __nv_bfloat16*>(A), M, d, lda, idx, k,
                                 reinterpret_cast<__nv_bfloat16*>(AI), ld_ai, chunks, vec_ok, err);
  }
}

// Rows per block of the staged compaction, or 0 when A's layout does not allow
// whole-row bulk copies (16-byte aligned rows, d a multiple of 8, a row of at
// most kMaxStagedRowBytes).
int staged_rows(const void* A, int64_t d, int64_t lda) {
  if (reinterpret_cast<uintptr_t>(A) % 16 || lda % 8 || d % 8) return 0;
  const int64_t row_bytes = 2 * d;
  // rows wider than the staging target (one row per block, an index round
  // trip exposed per 2048-column chunk) measured slower than the direct
  // gather: 172 vs 133 us for 2048 x 28672 at rho = 0.8; up to 32 KB (one
  // row of 14336 columns) staging was the faster, 50 vs 57 us
  if (row_bytes > kMaxStagedRowBytes || row_bytes > kStageTargetBytes) return 0;
  const int64_t r = kStageTargetBytes / row_bytes;
  return static_cast<int>(r < 1 ? 1 : (r > 8 ? 8 : r));
}

// Opt a kernel into kMaxStagedRowBytes of dynamic shared memory, once per device.
template <auto Kernel>
bool allow_staged_smem() {
  static std::atomic<uint64_t> configured{0};  // bit per device
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  const uint64_t bit = 1ull << dev;
  if (configured.load(std::memory_order_acquire) & bit) return true;
  if (cudaFuncSetAttribute(Kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(kMaxStagedRowBytes)) !=
      cudaSuccess)
    return false;
  configured.fetch_or(bit, std::memory_order_acq_rel);
  return true;
}

}  // namespace

cudaError_t launch_gather_rows(const void* B, int64_t d, int64_t row_bytes, int64_t ldb_bytes, const int32_t* idx,
                               int64_t k, void* B_I, int64_t ldbi_bytes, unsigned* err, cudaStream_t stream) {
  if (k == 0 || row_bytes == 0) return cudaSuccess;
  const int rpb = gather_rows_per_block(row_bytes / 16);
  const int64_t blocks = (k + rpb - 1) / rpb;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  return launch_pdl(gather_rows_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kGatherThreads), 0, stream,
                    static_cast<const uint4*>(B), d, row_bytes / 16, (row_bytes % 16) / 2, ldb_bytes / 16, idx, k,
                    static_cast<uint4*>(B_I), ldbi_bytes / 16, rpb, err);
}

cudaError_t launch_compact(const void* A, int dtype, int64_t M, int64_t d, int64_t lda, const int32_t* idx,
                           int64_t k, void* A_I, int64_t ld_ai, unsigned* err, cudaStream_t stream) {
  if (M == 0) return cudaSuccess;
  const size_t elt = dtype == 1 ? 2 : 4;
  const bool vec_ok = reinterpret_cast<uintptr_t>(A_I) % 16 == 0 && (ld_ai * elt) % 16 == 0;
  const int R = dtype == 1 ? staged_rows(A, d, lda) : 0;
  if (R > 0) {
    const int64_t blocks = (M + R - 1) / R;
    const size_t smem = static_cast<size_t>(R) * 2 * d;
    if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    if (smem > 48 * 1024 && !allow_staged_smem<compact_staged_kernel>()) return cudaErrorInvalidValue;
    return launch_pdl(compact_staged_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kCompactThreads), smem, stream,
                      static_cast<const uint16_t*>(A), M, d, lda, idx, k, static_cast<uint16_t*>(A_I), ld_ai, R, err);
  }
  const int64_t chunks = (k + kColsPerCta - 1) / kColsPerCta;
  const int64_t blocks = ((M + kRowsPerCta - 1) / kRowsPerCta) * chunks;
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
                                      void* B_I, int64_t ld_bi, unsigned* err, cudaStream_t stream, bool b_int8,
                                      uint32_t* zero, int64_t n_zero) {
  if (!zero) n_zero = 0;
  const int R = M > 0 ? staged_rows(A, d, lda) : 0;
  const int64_t chunks = (k + kColsPerCta - 1) / kColsPerCta;
  const int64_t cblocks = M <= 0 ? 0 : (R > 0 ? (M + R - 1) / R : ((M + kRowsPerCta - 1) / kRowsPerCta) * chunks);
  const int64_t belt = b_int8 ? 1 : 2;
  const int64_t row_bytes = N * belt;
  const int64_t vecs = row_bytes / 16, tail = (row_bytes % 16) / belt;
  const int rpb = gather_rows_per_block(vecs);
  const int64_t kb = (k + rpb - 1) / rpb;
  const int64_t blocks = kb + cblocks;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  const bool vec_ok = reinterpret_cast<uintptr_t>(A_I) % 16 == 0 && (ld_ai * 2) % 16 == 0;
  const int64_t ldb_vec = ldb * belt / 16, ldbi_vec = ld_bi * 2 / 16;
  const dim3 grid(static_cast<unsigned>(blocks)), block(kGatherThreads);
  const uint4* b = static_cast<const uint4*>(B);
  uint4* bi = static_cast<uint4*>(B_I);
  const uint16_t* a = static_cast<const uint16_t*>(A);
  uint16_t* ai = static_cast<uint16_t*>(A_I);
  auto go = [&](auto kernel, size_t smem, int r) {
    return launch_pdl(kernel, grid, block, smem, stream, b, d, vecs, tail, ldb_vec, bi, ldbi_vec, a, M, lda, ai, ld_ai,
                      chunks, r, vec_ok, idx, k, rpb, kb, err, zero, n_zero);
  };
  if (R > 0) {
    const size_t smem = static_cast<size_t>(R) * 2 * d;
    if (b_int8) {
      if (smem > 48 * 1024 && !allow_staged_smem<compact_gather_kernel<true, true>>()) return cudaErrorInvalidValue;
      return go(compact_gather_kernel<true, true>, smem, R);
    }
    if (smem > 48 * 1024 && !allow_staged_smem<compact_gather_kernel<true, false>>()) return cudaErrorInvalidValue;
    return go(compact_gather_kernel<true, false>, smem, R);
  }
  if (b_int8) return go(compact_gather_kernel<false, true>, 0, 0);
  return go(compact_gather_kernel<false, false>, 0, 0);
}

cudaError_t launch_gather_rows_i8(const void* Bq, int64_t d, int64_t N, int64_t ldb, const int32_t* idx, int64_t k,
                                  void* B_I, int64_t ld_bi, unsigned* err, cudaStream_t stream) {
  if (k == 0 || N == 0) return cudaSuccess;
  const int rpb = gather_rows_per_block(N / 16);
  const int64_t blocks = (k + rpb - 1) / rpb;
  if (blocks > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
  return launch_pdl(gather_rows_i8_kernel, dim3(static_cast<unsigned>(blocks)), dim3(kGatherThreads), 0, stream,
                    static_cast<const uint4*>(Bq), d, N / 16, N % 16, ldb / 16, idx, k, static_cast<uint4*>(B_I),
                    ld_bi * 2 / 16, rpb, err);
}

}  // namespace rmm
