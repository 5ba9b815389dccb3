// rmm_gemv.cu — reduced product for a few activation rows (decode), Y =
// A_I · B[I, :] with M <= 16 (Reduced Matrix Multiplication technical
// summary, Metodología › Mecanismo Central, at the batch sizes of
// autoregressive generation, Resultados Experimentales).
//
// HBM-bound: only the k kept rows of B are read, each once, in place (no
// gathered copy).  A block owns 256 columns of Y and a range of kept rows;
// the block's kept-row indices and A_I values are staged in shared memory
// first.  Two kernels:
//  - up to 4 activation rows, gemv_stream_kernel: each warp keeps six stages
//    of four kept rows in flight as 16-byte asynchronous copies into its own
//    ring in shared memory (192 rows in flight per block without holding
//    them in registers); every lane then reads its 8 columns and accumulates
//    fp32 FMAs; warps are summed in a fixed order.
//  - 5 to 16 rows, gemv_mma_kernel: the FMAs (8 per row and column) would
//    set the time, so the block runs mma.sync m16n8k16 (16 activation rows
//    are one tile's M): stages of 32 kept rows x 256 columns arrive by
//    cp.async, A_I comes from shared memory with ldmatrix and each stage's
//    row-major weight tile with ldmatrix.trans; each warp owns 32 columns.
// Row ranges (splits) of one column slice run as one thread-block cluster
// (up to 8 blocks): each block adds every split's sums for its share of the
// outputs, in split order, through distributed shared memory; beyond 8
// splits the sums go through global memory and a second kernel adds them in
// split order.  Either way the result depends only on the shape.
//
// An int8 weight (weight-only quantisation with one fp32 scale per output
// column; Resultados Experimentales › Compatibilidad) takes the same paths
// with half the bytes per row: the stream kernel widens 8 int8 values per
// lane exactly to fp32, the tensor-core kernel widens each stage to bf16
// (exact) in shared memory; the column scale multiplies the finished sum.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>
#include <type_traits>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"
#include "rmm_select.cuh"

namespace rmm {
namespace {

constexpr int kGemvMaxRows = 4096;  // kept rows per block (the staging buffer bounds it further)
constexpr int kGemvMaxSmem = 200 * 1024;  // dynamic shared memory the decode kernels are opted into
constexpr int kGemvMaxCluster = 8;  // splits reduced through distributed shared memory (portable cluster size)

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

// ---------------------------------------------------------------- streamed rows (M <= 4)

constexpr int kStreamWarps = 8;
constexpr int kStreamThreads = 32 * kStreamWarps;
constexpr int kStreamRowsPerStage = 4;              // kept rows per stage of a warp
// stages in flight per warp (twelve for int8 rows, filling the same ring,
// measured no faster: the one-row product is bound by fixed latency)
template <bool kW8>
constexpr int stream_stages() { return 6; }
constexpr int kStreamCols = 256;                    // columns of Y per block
constexpr int kStreamAiBytes = 16 * 1024;           // A_I staging (fp32 [row][m]) per block: two blocks fit an SM

template <bool kW8>
constexpr int stream_row_bytes() { return kStreamCols * (kW8 ? 1 : 2); }

template <bool kW8>
constexpr size_t stream_ring_bytes() {
  return static_cast<size_t>(kStreamWarps) * stream_stages<kW8>() * kStreamRowsPerStage * stream_row_bytes<kW8>();
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

// The selection done inside the product (kSel): the activation rows X
// [M x d] bf16 (base and rows 16-byte aligned, d a multiple of 8), and the
// outputs CTA (0, 0) writes for the caller.
struct GemvSelect {
  const uint16_t* X;
  int64_t ldx;
  int32_t* idx_out;  // the k kept indices, ascending
  float* ss_out;     // the d column scores (may be null)
};

// Largest d the fused selection stages: its keys and bins use the ring.
template <bool kW8>
constexpr int64_t stream_select_max_d() {
  return static_cast<int64_t>(stream_ring_bytes<kW8>()) / 4 - kSelectBins;
}

// grid: x = column slice of 256, y = row split.  Warp w takes the split's
// kept rows w, w + 8, w + 16, ..., four per stage, and keeps six stages of
// 16-byte asynchronous copies in flight (no registers held, no copy engine
// requests); a row whose index is out of range is copied as zeros.
//
// kSel: no selection launch before this one.  Every CTA computes the column
// scores of X (fp32 sums of the rows' exact squares, in row order: the same
// arithmetic as the selection kernel) into keys staged where its ring will
// be, runs the exact top-k search on them, and keeps the kept indices of its
// own rank range [r0, r0 + rows) straight in shared memory; CTA (0, 0) also
// writes the whole ascending index list and the scores.  A_I is read from X.
// The redundant selections run concurrently on every SM, so the product
// streams after a few microseconds instead of after a separate launch.
template <int MT, bool kW8, bool kSel>
__global__ void __launch_bounds__(kStreamThreads, 2)
    gemv_stream_kernel(const uint16_t* __restrict__ AI, int64_t ld_ai, const void* __restrict__ Bv, int64_t ldb,
                       const float* __restrict__ b_scale, const int32_t* __restrict__ idx, int M, int64_t d,
                       int64_t N, int64_t k, int rows_per_split, float* __restrict__ partial, void* __restrict__ Y,
                       int out_f32, int64_t ldy, int clustered, unsigned* err, GemvSelect sel) {
  constexpr int ELT = kW8 ? 1 : 2;
  constexpr int ROWB = stream_row_bytes<kW8>();
  constexpr int CPL = kStreamCols / 32;  // 8 columns per lane
  constexpr int COLS = kStreamCols;
  constexpr int RPS = kStreamRowsPerStage;
  constexpr int S = stream_stages<kW8>();
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int nrows = static_cast<int>(k - r0 < rows_per_split ? k - r0 : rows_per_split);
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * COLS;
  const int ncols = static_cast<int>(N - c0 < COLS ? N - c0 : COLS);
  float* sa = reinterpret_cast<float*>(smem + stream_ring_bytes<kW8>());  // A_I [row][MT]
  int32_t* sidx = reinterpret_cast<int32_t*>(sa + static_cast<size_t>(rows_per_split) * MT);
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

  pdl_wait();
  pdl_trigger();
  if constexpr (kSel) {
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);                       // d words, in the ring
    uint32_t* hist = keys + (static_cast<int>(d) + 3) / 4 * 4;                 // kSelectBins words
    const bool first = blockIdx.x == 0 && blockIdx.y == 0;
    const int dv = static_cast<int>(d / 8);
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int v = threadIdx.x; v < dv; v += kStreamThreads) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int m = 0; m < M; ++m) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(sel.X + static_cast<int64_t>(m) * sel.ldx) + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float lo = bf16_lo(w[t]), hi = bf16_hi(w[t]);
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
        if (first && sel.ss_out) sel.ss_out[8 * v + e] = acc[e];
      }
    }
    const uint32_t lo_rank = static_cast<uint32_t>(r0), hi_rank = static_cast<uint32_t>(r0 + nrows);
    select_staged_keys<kStreamThreads>(keys, static_cast<int>(d), static_cast<uint32_t>(k), kmin, kmax, hist,
                                       [&](uint32_t pos, int j) {
                                         if (pos >= lo_rank && pos < hi_rank) sidx[pos - lo_rank] = j;
                                         if (first) sel.idx_out[pos] = j;
                                       });
    __syncthreads();  // sidx is complete and the ring's keys and bins are no longer read
    // the first stages' copies go out before A_I is gathered from X, so the
    // two latencies overlap
#pragma unroll
    for (int st = 0; st < S - 1; ++st) issue(st);
    for (int m = 0; m < MT; ++m)
      for (int rr = threadIdx.x; rr < nrows; rr += kStreamThreads)
        sa[rr * MT + m] =
            m < M ? __uint_as_float(static_cast<uint32_t>(sel.X[static_cast<int64_t>(m) * sel.ldx + sidx[rr]]) << 16)
                  : 0.f;
    __syncthreads();
  } else {
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
  }

  float acc[MT][CPL];
#pragma unroll
  for (int m = 0; m < MT; ++m)
#pragma unroll
    for (int c = 0; c < CPL; ++c) acc[m][c] = 0.f;

  if constexpr (!kSel) {
#pragma unroll
    for (int st = 0; st < S - 1; ++st) issue(st);
  }
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

// ---------------------------------------------------------------- 9 to 16 rows on the tensor cores

constexpr int kMmaThreads = 256;
constexpr int kMmaCols = 256;          // columns of Y per block, 32 per warp
constexpr int kMmaRowsPerStage = 32;   // kept rows per stage: two k16 steps
template <bool kW8>
constexpr int mma_stages() { return kW8 ? 8 : 5; }  // two blocks fit an SM
constexpr int kMmaAiBytes = 32 * 1024; // A_I staging (bf16 [16][rows]) per block

template <bool kW8>
constexpr int mma_stage_pitch() { return kMmaCols * (kW8 ? 1 : 2) + 16; }  // bytes per staged row
constexpr int kMmaWidePitch = kMmaCols * 2 + 16;                           // widened int8 row

template <bool kW8>
size_t mma_smem_bytes(int rows_per_split) {
  const size_t ring = static_cast<size_t>(mma_stages<kW8>()) * kMmaRowsPerStage * mma_stage_pitch<kW8>();
  const size_t wide = kW8 ? static_cast<size_t>(kMmaRowsPerStage) * kMmaWidePitch : 0;
  const size_t ai = static_cast<size_t>(16) * ((rows_per_split + 31) / 32 * 32 * 2 + 16);
  const size_t idx = static_cast<size_t>(rows_per_split + 32) * 4;
  const size_t red = static_cast<size_t>(16) * kMmaCols * 4;
  return std::max(ring + wide + ai + idx, red + ai + idx);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_trans(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

// Largest d the fused selection of the tensor-core kernel stages (its ring).
template <bool kW8>
constexpr int64_t mma_select_max_d() {
  return static_cast<int64_t>(mma_stages<kW8>()) * kMmaRowsPerStage * mma_stage_pitch<kW8>() / 4 - kSelectBins;
}

// grid: x = column slice of 256, y = row split; M <= 16 (rows past M are zero).
// kSel: the selection inside the product, as in the streaming kernel.
template <bool kW8, bool kSel>
__global__ void __launch_bounds__(kMmaThreads, 2)
    gemv_mma_kernel(const uint16_t* __restrict__ AI, int64_t ld_ai, const void* __restrict__ Bv, int64_t ldb,
                    const float* __restrict__ b_scale, const int32_t* __restrict__ idx, int M, int64_t d, int64_t N,
                    int64_t k, int rows_per_split, float* __restrict__ partial, void* __restrict__ Y, int out_f32,
                    int64_t ldy, int clustered, unsigned* err, GemvSelect sel) {
  constexpr int ELT = kW8 ? 1 : 2;
  constexpr int PITCH = mma_stage_pitch<kW8>();
  constexpr int RPS = kMmaRowsPerStage;
  constexpr int S = mma_stages<kW8>();
  constexpr int COLS = kMmaCols;
  constexpr int CHUNKS = RPS * COLS * ELT / 16;  // 16-byte copies per stage
  extern __shared__ __align__(128) uint8_t smem[];
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int nrows = static_cast<int>(k - r0 < rows_per_split ? k - r0 : rows_per_split);
  const int64_t c0 = static_cast<int64_t>(blockIdx.x) * COLS;
  const int ncols = static_cast<int>(N - c0 < COLS ? N - c0 : COLS);
  const int rows16 = (rows_per_split + RPS - 1) / RPS * RPS;  // staged rows, whole stages
  const int ai_pitch = rows16 * 2 + 16;  // bytes per A_I row (bf16), padded
  const size_t ring_bytes = static_cast<size_t>(S) * RPS * PITCH;
  const size_t wide_bytes = kW8 ? static_cast<size_t>(RPS) * kMmaWidePitch : 0;
  uint8_t* wide = smem + ring_bytes;
  uint8_t* sai = smem + std::max(ring_bytes + wide_bytes, static_cast<size_t>(16) * COLS * 4);
  int32_t* sidx = reinterpret_cast<int32_t*>(sai + static_cast<size_t>(16) * ai_pitch);
  const char* B8 = static_cast<const char*>(Bv);
  const int nst = (nrows + RPS - 1) / RPS;
  const uint32_t ring = smem_u32(smem);
  auto issue = [&](int st) {
    if (st < nst) {
      const uint32_t base = ring + static_cast<uint32_t>((st % S) * RPS * PITCH);
      for (int e = threadIdx.x; e < CHUNKS; e += kMmaThreads) {
        const int r = e / (COLS * ELT / 16), piece = e % (COLS * ELT / 16);
        const int32_t j = sidx[st * RPS + r];
        const int rem = (ncols - piece * (16 / ELT)) * ELT;  // bytes of this piece inside the matrix
        const uint32_t nb = j < 0 || rem <= 0 ? 0u : static_cast<uint32_t>(rem < 16 ? rem : 16);
        const void* src = nb ? static_cast<const void*>(B8 + (static_cast<int64_t>(j) * ldb + c0) * ELT + piece * 16)
                             : Bv;
        cp_async16(base + r * PITCH + piece * 16, src, nb);
      }
    }
    cp_async_commit();
  };

  pdl_wait();
  pdl_trigger();

  if constexpr (kSel) {
    // scores of X, the exact top-k, and this split's kept indices (ranks
    // [r0, r0 + nrows)), with keys and bins where the ring will be
    uint32_t* keys = reinterpret_cast<uint32_t*>(smem);
    uint32_t* hist = keys + (static_cast<int>(d) + 3) / 4 * 4;
    const bool first = blockIdx.x == 0 && blockIdx.y == 0;
    for (int r = nrows + threadIdx.x; r < rows16; r += kMmaThreads) sidx[r] = -1;
    const int dv = static_cast<int>(d / 8);
    uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
    for (int v = threadIdx.x; v < dv; v += kMmaThreads) {
      float acc[8] = {0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f, 0.f};
      for (int m = 0; m < M; ++m) {
        const uint4 q = __ldg(reinterpret_cast<const uint4*>(sel.X + static_cast<int64_t>(m) * sel.ldx) + v);
        const uint32_t w[4] = {q.x, q.y, q.z, q.w};
#pragma unroll
        for (int t = 0; t < 4; ++t) {
          const float lo = bf16_lo(w[t]), hi = bf16_hi(w[t]);
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
        if (first && sel.ss_out) sel.ss_out[8 * v + e] = acc[e];
      }
    }
    const uint32_t lo_rank = static_cast<uint32_t>(r0), hi_rank = static_cast<uint32_t>(r0 + nrows);
    select_staged_keys<kMmaThreads>(keys, static_cast<int>(d), static_cast<uint32_t>(k), kmin, kmax, hist,
                                    [&](uint32_t pos, int j) {
                                      if (pos >= lo_rank && pos < hi_rank) sidx[pos - lo_rank] = j;
                                      if (first) sel.idx_out[pos] = j;
                                    });
    __syncthreads();  // sidx complete; keys and bins no longer read
    // the first stages' copies go out before A_I is gathered from X
#pragma unroll
    for (int st = 0; st < S - 1; ++st) issue(st);
    for (int e = threadIdx.x; e < 16 * rows16; e += kMmaThreads) {
      const int m = e / rows16, r = e % rows16;
      const uint16_t v = (m < M && r < nrows) ? sel.X[static_cast<int64_t>(m) * sel.ldx + sidx[r]] : uint16_t{0};
      *reinterpret_cast<uint16_t*>(sai + m * ai_pitch + r * 2) = v;
    }
  } else {
    // A_I rows (zero past M and past the split's rows) and the kept indices
    // (-1 for an index outside [0, d) and past the split's rows)
    for (int e = threadIdx.x; e < 16 * rows16; e += kMmaThreads) {
      const int m = e / rows16, r = e % rows16;
      const uint16_t v = (m < M && r < nrows) ? AI[static_cast<int64_t>(m) * ld_ai + r0 + r] : uint16_t{0};
      *reinterpret_cast<uint16_t*>(sai + m * ai_pitch + r * 2) = v;
    }
    bool bad = false;
    for (int r = threadIdx.x; r < rows16; r += kMmaThreads) {
      int32_t j = -1;
      if (r < nrows) {
        j = __ldg(idx + r0 + r);
        if (j < 0 || j >= d) {
          bad = true;
          j = -1;
        }
      }
      sidx[r] = j;
    }
    if (bad) record_error(err, kDevErrBadIndex);
  }
  __syncthreads();

  float acc[4][4];
#pragma unroll
  for (int t = 0; t < 4; ++t)
#pragma unroll
    for (int e = 0; e < 4; ++e) acc[t][e] = 0.f;
  const uint32_t ai_base = smem_u32(sai);
  const uint32_t wide_base = smem_u32(wide);
  if constexpr (!kSel) {
#pragma unroll
    for (int st = 0; st < S - 1; ++st) issue(st);
  }
  for (int st = 0; st < nst; ++st) {
    issue(st + S - 1);
    cp_async_wait<S - 1>();
    __syncthreads();  // every thread's copies of stage st have landed
    uint32_t tile = ring + static_cast<uint32_t>((st % S) * RPS * PITCH);
    uint32_t tpitch = PITCH;
    if constexpr (kW8) {
      // widen the int8 stage to bf16 (exact) in a separate buffer
      const uint8_t* src = smem + (st % S) * RPS * PITCH;
      for (int e = threadIdx.x; e < RPS * COLS / 4; e += kMmaThreads) {
        const int r = e / (COLS / 4), c4 = e % (COLS / 4);
        float f[4];
        i8x4_to_f32(*reinterpret_cast<const uint32_t*>(src + r * PITCH + c4 * 4), f);
        *reinterpret_cast<uint2*>(wide + r * kMmaWidePitch + c4 * 8) =
            make_uint2(pack_bf16x2(f[0], f[1]), pack_bf16x2(f[2], f[3]));
      }
      __syncthreads();
      tile = wide_base;
      tpitch = kMmaWidePitch;
    }
#pragma unroll
    for (int ks = 0; ks < RPS / 16; ++ks) {
      uint32_t a[4];
      ldsm_x4(ai_base + ((lane & 7) + ((lane >> 3) & 1) * 8) * ai_pitch + (st * RPS + ks * 16 + (lane >> 4) * 8) * 2,
              a);
#pragma unroll
      for (int t2 = 0; t2 < 2; ++t2) {
        // two 8-column tiles: lanes 0-15 address rows k 0-15 of the first,
        // lanes 16-31 the same rows of the second
        uint32_t b[4];
        const int n0 = warp * 32 + t2 * 16 + (lane >> 4) * 8;
        ldsm_x4_trans(tile + (ks * 16 + (lane & 15)) * tpitch + n0 * 2, b);
        mma_16816(acc[2 * t2], a, b[0], b[1]);
        mma_16816(acc[2 * t2 + 1], a, b[2], b[3]);
      }
    }
    __syncthreads();  // the stage (and the widened copy) may be refilled now
  }
  cp_async_wait<0>();
  __syncthreads();

  // this block's [16 x 256] sums: warp w owns columns 32 w .. 32 w + 31
  float* red = reinterpret_cast<float*>(smem);
  {
    const int g = lane >> 2, c2 = (lane & 3) * 2;
#pragma unroll
    for (int t = 0; t < 4; ++t) {
      const int col = warp * 32 + t * 8 + c2;
      red[g * COLS + col] = acc[t][0];
      red[g * COLS + col + 1] = acc[t][1];
      red[(g + 8) * COLS + col] = acc[t][2];
      red[(g + 8) * COLS + col + 1] = acc[t][3];
    }
  }
  const int nout = 16 * COLS;
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
    for (int e = threadIdx.x; e < nout; e += kMmaThreads) store(e, red[e]);
  } else if (clustered) {
    cluster_sync();
    const uint32_t nsplit = gridDim.y, rank = cluster_ctarank();
    const uint32_t red_s = smem_u32(red);
    for (int e = static_cast<int>(rank) * kMmaThreads + threadIdx.x; e < nout;
         e += static_cast<int>(nsplit) * kMmaThreads) {
      float v = 0.f;
      for (uint32_t q = 0; q < nsplit; ++q) v += ld_dsmem_f32(mapa_shared(red_s + e * 4, q));
      store(e, v);
    }
    cluster_sync();  // no block leaves while another may still read its shared memory
  } else {
    __syncthreads();
    for (int e = threadIdx.x; e < nout; e += kMmaThreads) {
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
  constexpr int64_t cols = MT <= 4 ? kStreamCols : kMmaCols;
  p.slices = (N + cols - 1) / cols;
  // one wave of two blocks per SM (a partial second wave would double the
  // time); each split at least 32 rows and at most what the A_I staging holds
  // (~96 KB for the register-loading kernel, 16 KB beside the streaming ring)
  const int64_t max_rows = MT <= 4 ? std::min<int64_t>(kGemvMaxRows, kStreamAiBytes / ((MT + 1) * 4) / 8 * 8)
                                    : kMmaAiBytes / (16 * 2) / 32 * 32;
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

template <int MT, bool kW8, bool kSel = false>
cudaError_t launch_gemv_mt(const uint16_t* AI, int64_t ld_ai, const void* B, int64_t ldb, const float* b_scale,
                           const int32_t* idx, int M, int64_t d, int64_t N, int64_t k, const GemvPlan& pl,
                           float* partial, void* Y, int out_f32, int64_t ldy, unsigned* err, cudaStream_t stream,
                           GemvSelect sel = GemvSelect{}) {
  constexpr bool kStream = MT <= 4;
  auto kernel = [] {
    if constexpr (kStream)
      return gemv_stream_kernel<MT, kW8, kSel>;
    else
      return gemv_mma_kernel<kW8, kSel>;
  }();
  const int threads = kStream ? kStreamThreads : kMmaThreads;
  const size_t smem = kStream ? stream_smem_bytes<MT, kW8>(pl.rows_per_split) : mma_smem_bytes<kW8>(pl.rows_per_split);
  {
    // opt in once per device, to the most any plan of this kernel asks for
    static std::atomic<uint64_t> configured{0};
    int dev = 0;
    if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return cudaErrorInvalidDevice;
    const uint64_t bit = 1ull << dev;
    if (!(configured.load(std::memory_order_acquire) & bit)) {
      const cudaError_t e =
          cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, kGemvMaxSmem);
      if (e != cudaSuccess) return e;
      configured.fetch_or(bit, std::memory_order_acq_rel);
    }
    if (smem > static_cast<size_t>(kGemvMaxSmem)) return cudaErrorInvalidConfiguration;
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
                           out_f32, ldy, 1, err, sel);
    return e;
  }
  e = launch_pdl(kernel, grid, dim3(threads), smem, stream, AI, ld_ai, B, ldb, b_scale, idx, M, d, N, k,
                 pl.rows_per_split, partial, Y, out_f32, ldy, 0, err, sel);
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

bool gemv_select_supported(const void* X, int64_t M, int64_t d, int64_t ldx, bool b_int8) {
  const int64_t max_d = M <= 4 ? (b_int8 ? stream_select_max_d<true>() : stream_select_max_d<false>())
                               : (b_int8 ? mma_select_max_d<true>() : mma_select_max_d<false>());
  return M >= 1 && M <= 16 && d >= 8 && d % 8 == 0 && d <= max_d && ldx % 8 == 0 &&
         reinterpret_cast<uintptr_t>(X) % 16 == 0;
}

cudaError_t launch_gemv_select(const void* X, int64_t ldx, int64_t M, int64_t d, const void* B, int64_t ldb,
                               const float* b_scale, int64_t N, int64_t k, const GemvPlan& pl, float* partial,
                               void* Y, int out_dtype, int64_t ldy, int32_t* idx_out, float* ss_out, unsigned* err,
                               cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  const GemvSelect sel{static_cast<const uint16_t*>(X), ldx, idx_out, ss_out};
  const int out_f32 = out_dtype == 0 ? 1 : 0;
  const int m = static_cast<int>(M);
  auto go = [&](auto mt) {
    constexpr int MT = decltype(mt)::value;
    if (b_scale)
      return launch_gemv_mt<MT, true, true>(nullptr, 0, B, ldb, b_scale, nullptr, m, d, N, k, pl, partial, Y, out_f32,
                                            ldy, err, stream, sel);
    return launch_gemv_mt<MT, false, true>(nullptr, 0, B, ldb, nullptr, nullptr, m, d, N, k, pl, partial, Y, out_f32,
                                           ldy, err, stream, sel);
  };
  if (M <= 1) return go(std::integral_constant<int, 1>{});
  if (M <= 2) return go(std::integral_constant<int, 2>{});
  if (M <= 4) return go(std::integral_constant<int, 4>{});
  if (M <= 8) return go(std::integral_constant<int, 8>{});
  return go(std::integral_constant<int, 16>{});
}

}  // namespace rmm
