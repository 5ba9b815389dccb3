// rmm_gemv.cu — reduced product for a few activation rows (decode), Y =
// A_I · B[I, :] with M <= 16 (Reduced Matrix Multiplication technical
// summary, Metodología › Mecanismo Central, at the batch sizes of
// autoregressive generation, Resultados Experimentales).
//
// HBM-bound: only the k kept rows of B are read, each once, in place (no
// gathered copy).  A block owns 256 columns of Y (128 above 8 activation
// rows) and a range of kept rows; its 8 warps take alternate rows of the
// range, every lane loading 8 columns (16 bytes; 4 columns, 8 bytes, above 8
// rows) of a row and accumulating them into fp32 sums.  The block's
// kept-row indices and A_I values are staged in shared memory first (A_I as
// fp32, [row][m], so one vector load serves four activation rows), so each
// batch of row loads goes out without waiting for its indices.  Warps are summed in a fixed order in shared
// memory.  Row ranges (splits) of one column slice run as one thread-block
// cluster (up to 8 blocks): each block adds every split's sums for its share
// of the outputs, in split order, through distributed shared memory; beyond 8
// splits the sums go through global memory and a second kernel adds them in
// split order.  Either way the result depends only on the shape.
//
// An int8 weight (weight-only quantisation with one fp32 scale per output
// column; Resultados Experimentales › Compatibilidad) takes the same path
// with half the bytes per row: each lane loads 8 (or 4) int8 values, widens
// them exactly to fp32, and the column scale multiplies the finished sum.
//
// Up to 8 activation rows the rows are streamed rather than loaded into
// registers (gemv_stream_kernel): each warp keeps six stages of four kept
// rows in flight as 16-byte asynchronous copies into its own ring in shared
// memory, so a block has 192 rows in flight without holding them in
// registers.  The register-loading kernel serves 9 to 16 rows, where the
// FMAs rather than the loads set the time.
#include <cuda_bf16.h>

#include <algorithm>
#include <type_traits>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

constexpr int kGemvThreads = 256;
constexpr int kGemvWarps = kGemvThreads / 32;
constexpr int kGemvMaxRows = 4096;  // kept rows per block (the staging buffer bounds it further)
constexpr int kGemvMaxCluster = 8;  // splits reduced through distributed shared memory (portable cluster size)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// Columns per lane: 8 up to 8 activation rows, else 4, so the accumulators
// stay at MT x CPL <= 64 registers; a lane's load is CPL weights (16 or 8
// bytes of bf16, 8 or 4 bytes of int8).
template <int MT, bool kW8 = false>
struct GemvShape {
  static constexpr int CPL = MT <= 8 ? 8 : 4;
  static constexpr int COLS = 32 * CPL;            // columns of Y per block
  // rows per batch (two batches in flight per warp); int8 rows are half the
  // bytes, so up to 4 activation rows they take twice the batch in the same
  // registers
  static constexpr int U = (MT == 8 ? 4 : 8) * (kW8 && MT <= 4 ? 2 : 1);
  using Vec16 = typename std::conditional<CPL == 8, uint4, uint2>::type;
  using Vec8 = typename std::conditional<CPL == 8, uint2, unsigned int>::type;
  using Vec = typename std::conditional<kW8, Vec8, Vec16>::type;
};

// grid: x = column slice, y = row split.  Dynamic shared memory:
// max(rows x (MT + 1), warps x MT x COLS) words.
// kW8: B is int8 (ldb in bytes) and b_scale[c] multiplies column c.
template <int MT, bool kW8>
__global__ void __launch_bounds__(kGemvThreads, 2)
    gemv_rows_kernel(const uint16_t* __restrict__ AI, int64_t ld_ai, const void* __restrict__ Bv, int64_t ldb,
                     const float* __restrict__ b_scale, const int32_t* __restrict__ idx, int M, int64_t d, int64_t N,
                     int64_t k, int rows_per_split, float* __restrict__ partial, void* __restrict__ Y, int out_f32,
                     int64_t ldy, int clustered, unsigned* err) {
  using Sh = GemvShape<MT, kW8>;
  using Vec = typename Sh::Vec;
  constexpr int CPL = Sh::CPL, COLS = Sh::COLS, U = Sh::U;
  extern __shared__ __align__(16) float sm[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int nrows = static_cast<int>(k - r0 < rows_per_split ? k - r0 : rows_per_split);
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * COLS + lane * CPL;
  pdl_wait();
  pdl_trigger();

  // stage A_I[:, r0 .. r0 + nrows) as fp32 [row][m] (rows of MT, zero past
  // M; read along rows, so coalesced) and the rows' indices after it (-1 for
  // an index outside [0, d))
  int32_t* sidx = reinterpret_cast<int32_t*>(sm + nrows * MT);
  for (int m = 0; m < MT; ++m)
    for (int rr = threadIdx.x; rr < nrows; rr += kGemvThreads)
      sm[rr * MT + m] =
          m < M ? __uint_as_float(static_cast<uint32_t>(AI[static_cast<int64_t>(m) * ld_ai + r0 + rr]) << 16) : 0.f;
  bool bad = false;
  for (int rr = threadIdx.x; rr < nrows; rr += kGemvThreads) {
    const int32_t j = __ldg(idx + r0 + rr);
    const bool ok = j >= 0 && j < d;
    bad |= !ok;
    sidx[rr] = ok ? j : -1;
  }
  if (bad) record_error(err, kDevErrBadIndex);
  __syncthreads();

  float acc[MT][CPL];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[m][c] = 0.f;

  const bool col_ok = c0 < N;
  // batch t holds rows warp + (t*U + u)*8, u < U; the loads of batch t+1 are
  // issued before batch t is consumed (two register buffers)
  auto load = [&](int t, Vec (&w)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rr = warp + (t * U + u) * kGemvWarps;
      w[u] = Vec{};
      if (rr < nrows) {
        const int32_t j = sidx[rr];
        if (j >= 0 && col_ok) {
          if constexpr (kW8)
            w[u] = __ldcs(reinterpret_cast<const Vec*>(static_cast<const int8_t*>(Bv) + static_cast<int64_t>(j) * ldb + c0));
          else
            w[u] = __ldcs(reinterpret_cast<const Vec*>(static_cast<const uint16_t*>(Bv) + static_cast<int64_t>(j) * ldb + c0));
        }
      }
    }
  };
  auto consume = [&](int t, const Vec (&w)[U]) {
#pragma unroll
    for (int u = 0; u < U; ++u) {
      const int rr = warp + (t * U + u) * kGemvWarps;
      if (rr < nrows) {
        float b[CPL];
        const uint32_t* wv = reinterpret_cast<const uint32_t*>(&w[u]);
        if constexpr (kW8) {
#pragma unroll
          for (int q = 0; q < CPL / 4; ++q) {
            float f[4];
            i8x4_to_f32(wv[q], f);
#pragma unroll
            for (int e = 0; e < 4; ++e) b[4 * q + e] = f[e];
          }
        } else {
#pragma unroll
          for (int q = 0; q < CPL / 2; ++q) {
            b[2 * q] = bf16_lo(wv[q]);
            b[2 * q + 1] = bf16_hi(wv[q]);
          }
        }
        const float* a = sm + rr * MT;
#pragma unroll
        for (int m4 = 0; m4 < MT; m4 += 4) {
          float av[4];
          if (MT >= 4) {
            const float4 q = *reinterpret_cast<const float4*>(a + m4);
            av[0] = q.x; av[1] = q.y; av[2] = q.z; av[3] = q.w;
          } else {
#pragma unroll
            for (int q = 0; q < 4; ++q) av[q] = q < MT ? a[q] : 0.f;
          }
#pragma unroll
          for (int q = 0; q < 4 && m4 + q < MT; ++q)
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[m4 + q][c] = fmaf(av[q], b[c], acc[m4 + q][c]);
        }
      }
    }
  };
  const int rows_w = (nrows - warp + kGemvWarps - 1) / kGemvWarps;  // rows of this warp
  const int nbatch = (rows_w + U - 1) / U;
  Vec wa[U], wb[U];
  if (nbatch > 0) load(0, wa);
  for (int t = 0; t < nbatch; t += 2) {
    if (t + 1 < nbatch) load(t + 1, wb);
    consume(t, wa);
    if (t + 1 < nbatch) {
      if (t + 2 < nbatch) load(t + 2, wa);
      consume(t + 1, wb);
    }
  }

  // sum the warps in a fixed order (the staging buffer is reused): red[m][c]
  // (in warp 0's slot) = sum over warps
  __syncthreads();
  float* red = sm;  // [warp][m][COLS]
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < CPL; c += 4)
      *reinterpret_cast<float4*>(red + (warp * MT + m) * COLS + lane * CPL + c) =
          make_float4(acc[m][c], acc[m][c + 1], acc[m][c + 2], acc[m][c + 3]);
  __syncthreads();
  const int nout = MT * COLS;
  for (int e = threadIdx.x; e < nout; e += kGemvThreads) {
    float sum = 0.f;
#pragma unroll
    for (int wq = 0; wq < kGemvWarps; ++wq) sum += red[wq * nout + e];
    red[e] = sum;
  }
  auto store = [&](int e, float v) {
    const int m = e / COLS, cl = e % COLS;
    const int64_t c = static_cast<int64_t>(blockIdx.x) * COLS + cl;
    if (m >= M || c >= N) return;
    if constexpr (kW8) v *= __ldg(b_scale + c);
    if (out_f32) {
      static_cast<float*>(Y)[static_cast<int64_t>(m) * ldy + c] = v;
    } else {
      static_cast<__nv_bfloat16*>(Y)[static_cast<int64_t>(m) * ldy + c] = __float2bfloat16_rn(v);
    }
  };
  if (gridDim.y == 1) {
    __syncthreads();
    for (int e = threadIdx.x; e < nout; e += kGemvThreads) store(e, red[e]);
  } else if (clustered) {
    // the splits of this column slice form the cluster (rank = split)
    cluster_sync();
    const uint32_t nsplit = gridDim.y, rank = cluster_ctarank();
    const uint32_t red_s = smem_u32(red);
    for (int e = static_cast<int>(rank) * kGemvThreads + threadIdx.x; e < nout;
         e += static_cast<int>(nsplit) * kGemvThreads) {
      float v = 0.f;
      for (uint32_t q = 0; q < nsplit; ++q) v += ld_dsmem_f32(mapa_shared(red_s + e * 4, q));
      store(e, v);
    }
    cluster_sync();  // no block leaves while another may still read its shared memory
  } else {
    __syncthreads();
    for (int e = threadIdx.x; e < nout; e += kGemvThreads) {
      const int m = e / COLS, cl = e % COLS;
      const int64_t c = static_cast<int64_t>(blockIdx.x) * COLS + cl;
      if (m < M && c < N) partial[(static_cast<int64_t>(blockIdx.y) * M + m) * N + c] = red[e];
    }
  }
}

// ---------------------------------------------------------------- streamed rows (M <= 8)

constexpr int kStreamWarps = 8;
constexpr int kStreamThreads = 32 * kStreamWarps;
constexpr int kStreamRowsPerStage = 4;              // kept rows per stage of a warp
constexpr int kStreamStages = 6;                    // stages in flight per warp
constexpr int kStreamCols = 256;                    // columns of Y per block
constexpr int kStreamAiBytes = 16 * 1024;           // A_I staging (fp32 [row][m]) per block: two blocks fit an SM

template <bool kW8>
constexpr int stream_row_bytes() { return kStreamCols * (kW8 ? 1 : 2); }

template <bool kW8>
constexpr size_t stream_ring_bytes() {
  return static_cast<size_t>(kStreamWarps) * kStreamStages * kStreamRowsPerStage * stream_row_bytes<kW8>();
}

// Dynamic shared memory: each warp's ring of stages, then A_I as fp32
// [row][MT], then the rows' indices; the warp sums of the epilogue reuse the
// start of it once every copy has landed.
template <int MT, bool kW8>
size_t stream_smem_bytes(int rows_per_split) {
  const size_t stage_ai = static_cast<size_t>(rows_per_split) * (MT + 1) * 4;
  const size_t red = static_cast<size_t>(kStreamWarps) * MT * kStreamCols * 4;
  return std::max(stream_ring_bytes<kW8>() + stage_ai, red);
}

// grid: x = column slice of 256, y = row split.  Warp w takes the split's
// kept rows w, w + 8, w + 16, ..., four per stage, and keeps six stages of
// 16-byte asynchronous copies in flight (no registers held, no copy engine
// requests); a row whose index is out of range is copied as zeros.
template <int MT, bool kW8>
__global__ void __launch_bounds__(kStreamThreads, 2)
    gemv_stream_kernel(const uint16_t* __restrict__ AI, int64_t ld_ai, const void* __restrict__ Bv, int64_t ldb,
                       const float* __restrict__ b_scale, const int32_t* __restrict__ idx, int M, int64_t d,
                       int64_t N, int64_t k, int rows_per_split, float* __restrict__ partial, void* __restrict__ Y,
                       int out_f32, int64_t ldy, int clustered, unsigned* err) {
  constexpr int ELT = kW8 ? 1 : 2;
  constexpr int ROWB = stream_row_bytes<kW8>();
  constexpr int CPL = kStreamCols / 32;  // 8 columns per lane
  constexpr int COLS = kStreamCols;
  constexpr int RPS = kStreamRowsPerStage;
  constexpr int S = kStreamStages;
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int nrows = static_cast<int>(k - r0 < rows_per_split ? k - r0 : rows_per_split);
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * COLS;
  const int ncols = static_cast<int>(N - c0 < COLS ? N - c0 : COLS);
  float* sa = reinterpret_cast<float*>(smem + stream_ring_bytes<kW8>());  // A_I [row][MT]
  int32_t* sidx = reinterpret_cast<int32_t*>(sa + static_cast<size_t>(rows_per_split) * MT);
  pdl_wait();
  pdl_trigger();
  for (int m = 0; m < MT; ++m)
    for (int rr = threadIdx.x; rr < nrows; rr += kStreamThreads)
      sa[rr * MT + m] =
          m < M ? __uint_as_float(static_cast<uint32_t>(AI[static_cast<int64_t>(m) * ld_ai + r0 + rr]) << 16) : 0.f;
  bool bad = false;
  for (int rr = threadIdx.x; rr < nrows; rr += kStreamThreads) {
    const int32_t j = __ldg(idx + r0 + rr);
    const bool ok = j >= 0 && j < d;
    bad |= !ok;
    sidx[rr] = ok ? j : -1;
  }
  if (bad) record_error(err, kDevErrBadIndex);
  __syncthreads();

  // this lane's 16-byte piece of a row slice: bf16, piece = lane (its own 8
  // columns); int8, 16 lanes per row, two rows per instruction
  const char* B8 = static_cast<const char*>(Bv);
  const uint32_t ring = smem_u32(smem) + static_cast<uint32_t>(warp * S * RPS * ROWB);
  const int rows_w = nrows > warp ? (nrows - warp + kStreamWarps - 1) / kStreamWarps : 0;
  const int nst = (rows_w + RPS - 1) / RPS;
  auto issue = [&](int st) {
    if (st < nst) {
      const uint32_t base = ring + static_cast<uint32_t>((st % S) * RPS * ROWB);
      if constexpr (kW8) {
#pragma unroll
        for (int h = 0; h < RPS / 2; ++h) {
          const int u = 2 * h + (lane >> 4), piece = lane & 15;
          const int i = st * RPS + u;
          const int rr = warp + i * kStreamWarps;
          const int32_t j = i < rows_w ? sidx[rr] : -1;
          const int rem = ncols - piece * 16;
          const uint32_t nb = j < 0 || rem <= 0 ? 0u : static_cast<uint32_t>(rem < 16 ? rem : 16);
          const void* src = nb ? static_cast<const void*>(B8 + static_cast<int64_t>(j) * ldb + c0 + piece * 16) : Bv;
          cp_async16(base + u * ROWB + piece * 16, src, nb);
        }
      } else {
#pragma unroll
        for (int u = 0; u < RPS; ++u) {
          const int i = st * RPS + u;
          const int rr = warp + i * kStreamWarps;
          const int32_t j = i < rows_w ? sidx[rr] : -1;
          const int rem = ncols - lane * CPL;
          const uint32_t nb = j < 0 || rem <= 0 ? 0u : static_cast<uint32_t>((rem < CPL ? rem : CPL) * 2);
          const void* src = nb ? static_cast<const void*>(B8 + (static_cast<int64_t>(j) * ldb + c0 + lane * CPL) * 2)
                               : Bv;
          cp_async16(base + u * ROWB + lane * 16, src, nb);
        }
      }
    }
    cp_async_commit();  // one group per stage, empty past the end, so the wait count stays fixed
  };

  float acc[MT][CPL];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[m][c] = 0.f;

#pragma unroll
  for (int st = 0; st < S - 1; ++st) issue(st);
  for (int st = 0; st < nst; ++st) {
    issue(st + S - 1);
    cp_async_wait<S - 1>();  // stage st has landed (this lane's copies)
    __syncwarp();            // ... and every lane's
    const uint8_t* base = smem + warp * S * RPS * ROWB + (st % S) * RPS * ROWB + lane * CPL * ELT;
#pragma unroll
    for (int u = 0; u < RPS; ++u) {
      const int i = st * RPS + u;
      if (i < rows_w) {
        const int rr = warp + i * kStreamWarps;
        float b[CPL];
        if constexpr (kW8) {
          const uint2 w = *reinterpret_cast<const uint2*>(base + u * ROWB);
          float f[4];
          i8x4_to_f32(w.x, f);
#pragma unroll
          for (int e = 0; e < 4; ++e) b[e] = f[e];
          i8x4_to_f32(w.y, f);
#pragma unroll
          for (int e = 0; e < 4; ++e) b[4 + e] = f[e];
        } else {
          const uint4 w = *reinterpret_cast<const uint4*>(base + u * ROWB);
          const uint32_t wv[4] = {w.x, w.y, w.z, w.w};
#pragma unroll
          for (int e = 0; e < 4; ++e) {
            b[2 * e] = bf16_lo(wv[e]);
            b[2 * e + 1] = bf16_hi(wv[e]);
          }
        }
        const float* a = sa + rr * MT;
#pragma unroll
        for (int m4 = 0; m4 < MT; m4 += 4) {
          float av[4];
          if (MT >= 4) {
            const float4 v = *reinterpret_cast<const float4*>(a + m4);
            av[0] = v.x; av[1] = v.y; av[2] = v.z; av[3] = v.w;
          } else {
#pragma unroll
            for (int e = 0; e < 4; ++e) av[e] = e < MT ? a[e] : 0.f;
          }
#pragma unroll
          for (int e = 0; e < 4 && m4 + e < MT; ++e)
#pragma unroll
            for (int c = 0; c < CPL; ++c) acc[m4 + e][c] = fmaf(av[e], b[c], acc[m4 + e][c]);
        }
      }
    }
    __syncwarp();  // every lane has read the stage before a later issue overwrites it
  }
  cp_async_wait<0>();
  __syncthreads();  // the rings and the staging are free

  // warp sums in a fixed order: red[m][c] = sum over warps
  float* red = reinterpret_cast<float*>(smem);
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < CPL; c += 4)
      *reinterpret_cast<float4*>(red + (warp * MT + m) * COLS + lane * CPL + c) =
          make_float4(acc[m][c], acc[m][c + 1], acc[m][c + 2], acc[m][c + 3]);
  __syncthreads();
  const int nout = MT * COLS;
  for (int e = threadIdx.x; e < nout; e += kStreamThreads) {
    float sum = 0.f;
#pragma unroll
    for (int wq = 0; wq < kStreamWarps; ++wq) sum += red[wq * nout + e];
    red[e] = sum;
  }
  auto store = [&](int e, float v) {
    const int m = e / COLS, cl = e % COLS;
    const int64_t c = c0 + cl;
    if (m >= M || c >= N) return;
    if constexpr (kW8) v *= __ldg(b_scale + c);
    if (out_f32) {
      static_cast<float*>(Y)[static_cast<int64_t>(m) * ldy + c] = v;
    } else {
      static_cast<__nv_bfloat16*>(Y)[static_cast<int64_t>(m) * ldy + c] = __float2bfloat16_rn(v);
    }
  };
  if (gridDim.y == 1) {
    __syncthreads();
    for (int e = threadIdx.x; e < nout; e += kStreamThreads) store(e, red[e]);
  } else if (clustered) {
    cluster_sync();
    const uint32_t nsplit = gridDim.y, rank = cluster_ctarank();
    const uint32_t red_s = smem_u32(red);
    for (int e = static_cast<int>(rank) * kStreamThreads + threadIdx.x; e < nout;
         e += static_cast<int>(nsplit) * kStreamThreads) {
      float v = 0.f;
      for (uint32_t q = 0; q < nsplit; ++q) v += ld_dsmem_f32(mapa_shared(red_s + e * 4, q));
      store(e, v);
    }
    cluster_sync();  // no block leaves while another may still read its shared memory
  } else {
    __syncthreads();
    for (int e = threadIdx.x; e < nout; e += kStreamThreads) {
      const int m = e / COLS, cl = e % COLS;
      const int64_t c = c0 + cl;
      if (m < M && c < N) partial[(static_cast<int64_t>(blockIdx.y) * M + m) * N + c] = red[e];
    }
  }
}

// Y[m, c] = sum over splits (in order) of partial[split][m][c], times
// b_scale[c] when given.
__global__ void __launch_bounds__(256) gemv_reduce_kernel(const float* __restrict__ partial, int splits, int M,
                                                          int64_t N, const float* __restrict__ b_scale,
                                                          void* __restrict__ Y, int out_f32, int64_t ldy) {
  pdl_wait();
  pdl_trigger();
  const int64_t e = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (e >= static_cast<int64_t>(M) * N) return;
  const int m = static_cast<int>(e / N);
  const int64_t c = e % N;
  float s = 0.f;
  for (int t = 0; t < splits; ++t) s += __ldg(partial + static_cast<int64_t>(t) * M * N + e);
  if (b_scale) s *= __ldg(b_scale + c);
  if (out_f32) {
    static_cast<float*>(Y)[static_cast<int64_t>(m) * ldy + c] = s;
  } else {
    static_cast<__nv_bfloat16*>(Y)[static_cast<int64_t>(m) * ldy + c] = __float2bfloat16_rn(s);
  }
}

template <int MT>
GemvPlan plan_mt(int64_t M, int64_t N, int64_t k, int sms) {
  GemvPlan p{};
  p.slices = (N + GemvShape<MT>::COLS - 1) / GemvShape<MT>::COLS;
  // one wave of two blocks per SM (a partial second wave would double the
  // time); each split at least 32 rows and at most what the A_I staging holds
  // (~96 KB for the register-loading kernel, 16 KB beside the streaming ring)
  const int64_t stage_bytes = MT <= 8 ? kStreamAiBytes : 96 * 1024;
  const int64_t max_rows = std::min<int64_t>(kGemvMaxRows, stage_bytes / ((MT + 1) * 4) / 8 * 8);
  int64_t splits = std::max<int64_t>(1, 2 * static_cast<int64_t>(std::max(sms, 1)) / p.slices);
  splits = std::min<int64_t>(splits, kGemvMaxCluster);  // splits of a slice form one cluster
  splits = std::min<int64_t>(splits, std::max<int64_t>(1, k / 32));
  splits = std::max<int64_t>(splits, (k + max_rows - 1) / max_rows);
  p.rows_per_split = static_cast<int>((k + splits - 1) / splits);
  p.splits = static_cast<int>((k + p.rows_per_split - 1) / p.rows_per_split);
  p.clustered = p.splits > 1 && p.splits <= kGemvMaxCluster;
  p.partial_bytes = p.splits > 1 && !p.clustered ? static_cast<size_t>(p.splits) * M * N * 4 : 0;
  return p;
}

template <int MT, bool kW8>
cudaError_t launch_gemv_mt(const uint16_t* AI, int64_t ld_ai, const void* B, int64_t ldb, const float* b_scale,
                           const int32_t* idx, int M, int64_t d, int64_t N, int64_t k, const GemvPlan& pl,
                           float* partial, void* Y, int out_f32, int64_t ldy, unsigned* err, cudaStream_t stream) {
  constexpr bool kStream = MT <= 8;
  static_assert(!kStream || GemvShape<MT, kW8>::COLS == kStreamCols, "one column slicing for both kernels");
  auto kernel = [] {
    if constexpr (kStream)
      return gemv_stream_kernel<MT, kW8>;
    else
      return gemv_rows_kernel<MT, kW8>;
  }();
  const int threads = kStream ? kStreamThreads : kGemvThreads;
  const size_t smem =
      kStream ? stream_smem_bytes<MT, kW8>(pl.rows_per_split)
              : static_cast<size_t>(std::max(pl.rows_per_split * (MT + 1), kGemvWarps * MT * GemvShape<MT>::COLS)) * 4;
  if (smem > 48 * 1024) {
    const cudaError_t e =
        cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, static_cast<int>(smem));
    if (e != cudaSuccess) return e;
  }
  const dim3 grid(static_cast<unsigned>(pl.slices), static_cast<unsigned>(pl.splits));
  cudaError_t e;
  if (pl.clustered) {
    cudaLaunchConfig_t cfg{};
    cfg.gridDim = grid;
    cfg.blockDim = dim3(threads);
    cfg.dynamicSmemBytes = smem;
    cfg.stream = stream;
    cudaLaunchAttribute attr[2];
    attr[0].id = cudaLaunchAttributeClusterDimension;
    attr[0].val.clusterDim.x = 1;
    attr[0].val.clusterDim.y = static_cast<unsigned>(pl.splits);
    attr[0].val.clusterDim.z = 1;
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.attrs = attr;
    cfg.numAttrs = 2;
    e = cudaLaunchKernelEx(&cfg, kernel, AI, ld_ai, B, ldb, b_scale, idx, M, d, N, k, pl.rows_per_split, partial, Y,
                           out_f32, ldy, 1, err);
    return e;
  }
  e = launch_pdl(kernel, grid, dim3(threads), smem, stream, AI, ld_ai, B, ldb, b_scale, idx, M, d, N, k,
                 pl.rows_per_split, partial, Y, out_f32, ldy, 0, err);
  if (e != cudaSuccess || pl.splits == 1) return e;
  const int64_t outs = static_cast<int64_t>(M) * N;
  return launch_pdl(gemv_reduce_kernel, dim3(static_cast<unsigned>((outs + 255) / 256)), dim3(256), 0, stream,
                    static_cast<const float*>(partial), pl.splits, M, N, kW8 ? b_scale : nullptr, Y, out_f32, ldy);
}

}  // namespace

GemvPlan gemv_plan(int64_t M, int64_t N, int64_t k, int sms) {
  if (M <= 1) return plan_mt<1>(M, N, k, sms);
  if (M <= 2) return plan_mt<2>(M, N, k, sms);
  if (M <= 4) return plan_mt<4>(M, N, k, sms);
  if (M <= 8) return plan_mt<8>(M, N, k, sms);
  return plan_mt<16>(M, N, k, sms);
}

cudaError_t launch_gemv(const void* A_I, int64_t ld_ai, const void* B, int64_t ldb, const int32_t* idx, int64_t M,
                        int64_t d, int64_t N, int64_t k, const GemvPlan& pl, float* partial, void* Y, int out_dtype,
                        int64_t ldy, unsigned* err, cudaStream_t stream, const float* b_scale) {
  if (M == 0 || N == 0) return cudaSuccess;
  const uint16_t* ai = static_cast<const uint16_t*>(A_I);
  const int out_f32 = out_dtype == 0 ? 1 : 0;
  const int m = static_cast<int>(M);
  auto go = [&](auto mt) {
    constexpr int MT = decltype(mt)::value;
    if (b_scale)
      return launch_gemv_mt<MT, true>(ai, ld_ai, B, ldb, b_scale, idx, m, d, N, k, pl, partial, Y, out_f32, ldy, err,
                                      stream);
    return launch_gemv_mt<MT, false>(ai, ld_ai, B, ldb, nullptr, idx, m, d, N, k, pl, partial, Y, out_f32, ldy, err,
                                     stream);
  };
  if (M <= 1) return go(std::integral_constant<int, 1>{});
  if (M <= 2) return go(std::integral_constant<int, 2>{});
  if (M <= 4) return go(std::integral_constant<int, 4>{});
  if (M <= 8) return go(std::integral_constant<int, 8>{});
  return go(std::integral_constant<int, 16>{});
}

}  // namespace rmm
