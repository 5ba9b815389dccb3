// rmm_score.cu — column scores ss_j = sum_i A[i,j]^2 (Reduced Matrix
// Multiplication technical summary, Metodología › Estrategia de Selección:
// s_j = ||A[:,j]||_2; the square keeps the ranking).
//
// HBM-bound design: each thread owns one 16-byte column vector (8 bf16 or 4
// fp32 columns) and loads 16 rows of it at once, so a warp reads 512
// contiguous bytes of a row per load.  A 256-thread CTA is col_threads wide and
// row_groups tall; CTAs tile (column strip, row split, batch).  Squares of bf16
// values are exact in fp32 and accumulate with one rounding per row (fma).
// Row groups combine by a fixed pairwise tree in shared memory; row splits are
// combined by a second kernel in a fixed order.  No atomics, so the
// result depends only on the shape.
//
// For bf16 with 16-byte aligned rows, score_cluster_kernel does it in one
// launch: at most 8 row splits of a column strip run as one thread-block
// cluster and are added in split order through distributed shared memory.
// The grid is sized to one wave of resident CTAs (two per SM), and every
// thread keeps 8-16 loads in flight as a ring that is refilled as it drains,
// so each SM streams from its first cycle to its last.  (The two-kernel form
// spent a third of its partial pass ramping and draining one wave, and its
// finalize pass was a launch of pure latency; a grid of 1.5-1.7 waves of
// one-shot CTAs left SMs idle behind the partial second wave.)
//
// silu_mul_score_kernel fuses the score of the MLP down projection into the
// producer of its activation: H = SiLU(G) * U (G, U the gate and up outputs,
// bf16), rounded to bf16 and stored, and ss_j = sum_i H[i,j]^2 of the stored
// values, on the same plan, so H is read back by nobody before the top-k.
#include <cuda_bf16.h>

#include <algorithm>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

constexpr int kScoreThreads = 256;
// Every thread sums exactly kRowsPerThread rows of its column vector, with all
// of those 16-byte loads issued before the first is consumed: one round of
// memory latency per CTA.  A CTA therefore covers kRowsPerThread * row_groups
// rows; the row splits this produces are summed by the finalize kernel.  The
// plan depends only on the shape, so the summation order does too.
constexpr int kRowsPerThread = 16;
static_assert(kRowsPerThread % 8 == 0, "loads are issued eight at a time");

template <typename T>
struct Lanes;
template <>
struct Lanes<__nv_bfloat16> {
  static constexpr int kVec = 8;
  __device__ static void unpack(const uint4 v, float (&x)[8]) {
    const uint32_t w[4] = {v.x, v.y, v.z, v.w};
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      x[2 * i] = __uint_as_float(w[i] << 16);
      x[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
    }
  }
  __device__ static float scalar(const __nv_bfloat16* p) { return __bfloat162float(p[0]); }
};
template <>
struct Lanes<float> {
  static constexpr int kVec = 4;
  __device__ static void unpack(const uint4 v, float (&x)[4]) {
    x[0] = __uint_as_float(v.x);
    x[1] = __uint_as_float(v.y);
    x[2] = __uint_as_float(v.z);
    x[3] = __uint_as_float(v.w);
  }
  __device__ static float scalar(const float* p) { return __ldg(p); }
};

// Grid: x = column strip, y = row split, z = batch.
template <typename T>
__global__ void __launch_bounds__(kScoreThreads) score_partial_kernel(
    const T* __restrict__ A, int64_t M, int64_t d, int64_t lda, int64_t batch_stride, int col_threads,
    int64_t rows_per_split, bool vec_ok, float* __restrict__ out, int64_t out_batch_stride,
    int64_t out_split_stride, int sqrt_out) {
  constexpr int V = Lanes<T>::kVec;
  __shared__ float red[kScoreThreads * V];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x % col_threads;
  const int ty = threadIdx.x / col_threads;
  const int row_groups = kScoreThreads / col_threads;
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * col_threads + tx) * V;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(M, r0 + rows_per_split);
  const T* Ab = A + static_cast<int64_t>(blockIdx.z) * batch_stride;

  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;

  if (col0 < d) {
    if (vec_ok && col0 + V <= d) {
      // two rounds of eight independent 16-byte loads (more in flight costs
      // registers, hence occupancy, for no gain)
#pragma unroll
      for (int u0 = 0; u0 < kRowsPerThread; u0 += 8) {
        uint4 raw[8];
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          const int64_t r = r0 + ty + static_cast<int64_t>(u0 + u) * row_groups;
          raw[u] = r < r1 ? __ldg(reinterpret_cast<const uint4*>(Ab + r * lda + col0)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 8; ++u) {
          float x[V];
          Lanes<T>::unpack(raw[u], x);
#pragma unroll
          for (int e = 0; e < V; ++e) acc[e] = fmaf(x[e], x[e], acc[e]);
        }
      }
    } else {
      for (int64_t r = r0 + ty; r < r1; r += row_groups) {
#pragma unroll
        for (int e = 0; e < V; ++e) {
          if (col0 + e < d) {
            const float x = Lanes<T>::scalar(Ab + r * lda + col0 + e);
            acc[e] = fmaf(x, x, acc[e]);
          }
        }
      }
    }
  }

  // pairwise tree over the row groups (fixed order)
#pragma unroll
  for (int e = 0; e < V; ++e) red[(ty * col_threads + tx) * V + e] = acc[e];
  __syncthreads();
  for (int s = row_groups / 2; s >= 1; s >>= 1) {
    if (ty < s) {
#pragma unroll
      for (int e = 0; e < V; ++e) red[(ty * col_threads + tx) * V + e] += red[((ty + s) * col_threads + tx) * V + e];
    }
    __syncthreads();
  }
  if (ty == 0) {
    float* o = out + static_cast<int64_t>(blockIdx.z) * out_batch_stride +
               static_cast<int64_t>(blockIdx.y) * out_split_stride;
#pragma unroll
    for (int e = 0; e < V; ++e) {
      if (col0 + e < d) {
        const float v = red[tx * V + e];
        o[col0 + e] = sqrt_out ? sqrtf(v) : v;
      }
    }
  }
}

// Grid: x = column strip, y = row split (the cluster), z = batch.  Two CTAs
// per SM are resident (the ring below takes about 110 registers per thread),
// and the host sizes the grid to one resident wave.
__global__ void __launch_bounds__(kScoreThreads, 2) score_cluster_kernel(
    const __nv_bfloat16* __restrict__ A, int64_t M, int64_t d, int64_t lda, int64_t batch_stride, int col_threads,
    int64_t rows_per_split, float* __restrict__ ss, int64_t ld_ss, int sqrt_out) {
  constexpr int V = 8;
  // ring slots per thread: the compiler issues a round's refills ahead of its
  // consumption, so 8 slots keep 8-16 loads in flight (111 registers, two CTAs
  // per SM: 64-128 KB in flight per SM); 16 slots would spill
  constexpr int U = 8;
  __shared__ float red[kScoreThreads * V];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x % col_threads;
  const int ty = threadIdx.x / col_threads;
  const int row_groups = kScoreThreads / col_threads;
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * col_threads + tx) * V;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(M, r0 + rows_per_split);
  const __nv_bfloat16* Ab = A + static_cast<int64_t>(blockIdx.z) * batch_stride;
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  auto add = [&](const uint4 raw) {
    float x[V];
    Lanes<__nv_bfloat16>::unpack(raw, x);
#pragma unroll
    for (int e = 0; e < V; ++e) acc[e] = fmaf(x[e], x[e], acc[e]);
  };
  if (col0 < d) {
    if (col0 + V <= d) {
      // this thread's rows r0 + ty + i * row_groups, i < n, summed in order;
      // slot u of the ring holds row i + u while rows i.. are consumed, and is
      // refilled with row i + u + U as soon as it has been read
      const int64_t first = r0 + ty;
      const int64_t n = first < r1 ? (r1 - first + row_groups - 1) / row_groups : 0;
      const uint4* p = reinterpret_cast<const uint4*>(Ab + first * lda + col0);  // next row to load
      const int64_t step = static_cast<int64_t>(row_groups) * lda / V;          // uint4 per row step
      uint4 ring[U];
#pragma unroll
      for (int u = 0; u < U; ++u) {
        ring[u] = u < n ? __ldg(p) : make_uint4(0, 0, 0, 0);
        p += step;
      }
      int64_t i = 0;
#pragma unroll 1
      for (; i + 2 * U <= n; i += U) {  // every refill is a row of this thread
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint4 x = ring[u];
          ring[u] = __ldg(p);
          p += step;
          add(x);
        }
      }
      if (i + U < n) {  // the last, partial refill
#pragma unroll
        for (int u = 0; u < U; ++u) {
          const uint4 x = ring[u];
          ring[u] = i + U + u < n ? __ldg(p) : make_uint4(0, 0, 0, 0);
          p += step;
          add(x);
        }
        i += U;
      }
#pragma unroll
      for (int u = 0; u < U; ++u)
        if (i + u < n) add(ring[u]);
    } else {
      for (int64_t r = r0 + ty; r < r1; r += row_groups) {
#pragma unroll
        for (int e = 0; e < V; ++e) {
          if (col0 + e < d) {
            const float x = __bfloat162float(Ab[r * lda + col0 + e]);
            acc[e] = fmaf(x, x, acc[e]);
          }
        }
      }
    }
  }
  // pairwise tree over the row groups (fixed order): the CTA's sums end in
  // red[0 .. col_threads * V)
#pragma unroll
  for (int e = 0; e < V; ++e) red[(ty * col_threads + tx) * V + e] = acc[e];
  __syncthreads();
  for (int st = row_groups / 2; st >= 1; st >>= 1) {
    if (ty < st) {
#pragma unroll
      for (int e = 0; e < V; ++e) red[(ty * col_threads + tx) * V + e] += red[((ty + st) * col_threads + tx) * V + e];
    }
    __syncthreads();
  }
  const int ncols = col_threads * V;
  const int64_t cbase = static_cast<int64_t>(blockIdx.x) * ncols;
  float* out = ss + static_cast<int64_t>(blockIdx.z) * ld_ss;
  if (gridDim.y == 1) {
    for (int e = threadIdx.x; e < ncols; e += kScoreThreads)
      if (cbase + e < d) out[cbase + e] = sqrt_out ? sqrtf(red[e]) : red[e];
    return;
  }
  // the splits of this strip are the cluster (rank = split): each CTA adds
  // every split's sums for its share of the columns, in split order
  cluster_sync();
  const uint32_t nsplit = gridDim.y, rank = cluster_ctarank();
  const uint32_t red_s = smem_u32(red);
  for (int e = static_cast<int>(rank) * kScoreThreads + threadIdx.x; e < ncols;
       e += static_cast<int>(nsplit) * kScoreThreads) {
    float v = 0.f;
    for (uint32_t q = 0; q < nsplit; ++q) v += ld_dsmem_f32(mapa_shared(red_s + e * 4, q));
    if (cbase + e < d) out[cbase + e] = sqrt_out ? sqrtf(v) : v;
  }
  cluster_sync();  // no CTA leaves while another may still read its shared memory
}

// H = bf16(SiLU(G) * U) with SiLU(g) = g / (1 + e^-g) in fp32, and the
// column sums of the stored H's squares, on the bf16 score plan (16-byte
// vectors; G, U, H 16-byte aligned with row pitches multiples of 8).
// Grid: x = column strip, y = row split.
__global__ void __launch_bounds__(kScoreThreads) silu_mul_score_kernel(
    const __nv_bfloat16* __restrict__ G, int64_t ldg, const __nv_bfloat16* __restrict__ U, int64_t ldu,
    __nv_bfloat16* __restrict__ H, int64_t ldh, int64_t M, int64_t d, int col_threads, int64_t rows_per_split,
    float* __restrict__ out, int64_t out_split_stride) {
  constexpr int V = 8;
  __shared__ float red[kScoreThreads * V];
  pdl_wait();
  pdl_trigger();
  const int tx = threadIdx.x % col_threads;
  const int ty = threadIdx.x / col_threads;
  const int row_groups = kScoreThreads / col_threads;
  const int64_t col0 = (static_cast<int64_t>(blockIdx.x) * col_threads + tx) * V;
  const int64_t r0 = static_cast<int64_t>(blockIdx.y) * rows_per_split;
  const int64_t r1 = min(M, r0 + rows_per_split);
  float acc[V];
#pragma unroll
  for (int e = 0; e < V; ++e) acc[e] = 0.f;
  auto produce = [&](float gv, float uv) {
    const float h = gv / (1.f + expf(-gv)) * uv;
    return __float2bfloat16_rn(h);
  };
  if (col0 < d) {
    if (col0 + V <= d) {
#pragma unroll
      for (int u0 = 0; u0 < kRowsPerThread; u0 += 4) {
        uint4 rg[4], ru[4];
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t r = r0 + ty + static_cast<int64_t>(u0 + u) * row_groups;
          rg[u] = r < r1 ? __ldg(reinterpret_cast<const uint4*>(G + r * ldg + col0)) : make_uint4(0, 0, 0, 0);
          ru[u] = r < r1 ? __ldg(reinterpret_cast<const uint4*>(U + r * ldu + col0)) : make_uint4(0, 0, 0, 0);
        }
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int64_t r = r0 + ty + static_cast<int64_t>(u0 + u) * row_groups;
          float gx[V], ux[V];
          Lanes<__nv_bfloat16>::unpack(rg[u], gx);
          Lanes<__nv_bfloat16>::unpack(ru[u], ux);
          uint32_t packed[4];
#pragma unroll
          for (int e = 0; e < V; e += 2) {
            const __nv_bfloat16 h0 = produce(gx[e], ux[e]), h1 = produce(gx[e + 1], ux[e + 1]);
            const float f0 = __bfloat162float(h0), f1 = __bfloat162float(h1);
            acc[e] = fmaf(f0, f0, acc[e]);
            acc[e + 1] = fmaf(f1, f1, acc[e + 1]);
            packed[e / 2] = static_cast<uint32_t>(__bfloat16_as_ushort(h0)) |
                            (static_cast<uint32_t>(__bfloat16_as_ushort(h1)) << 16);
          }
          if (r < r1)
            *reinterpret_cast<uint4*>(H + r * ldh + col0) = make_uint4(packed[0], packed[1], packed[2], packed[3]);
        }
      }
    } else {
      for (int64_t r = r0 + ty; r < r1; r += row_groups) {
        for (int e = 0; e < V && col0 + e < d; ++e) {
          const __nv_bfloat16 h = produce(__bfloat162float(G[r * ldg + col0 + e]), __bfloat162float(U[r * ldu + col0 + e]));
          H[r * ldh + col0 + e] = h;
          const float f = __bfloat162float(h);
          acc[e] = fmaf(f, f, acc[e]);
        }
      }
    }
  }
#pragma unroll
  for (int e = 0; e < V; ++e) red[(ty * col_threads + tx) * V + e] = acc[e];
  __syncthreads();
  for (int s = row_groups / 2; s >= 1; s >>= 1) {
    if (ty < s) {
#pragma unroll
      for (int e = 0; e < V; ++e) red[(ty * col_threads + tx) * V + e] += red[((ty + s) * col_threads + tx) * V + e];
    }
    __syncthreads();
  }
  if (ty == 0) {
    float* o = out + static_cast<int64_t>(blockIdx.y) * out_split_stride;
#pragma unroll
    for (int e = 0; e < V; ++e)
      if (col0 + e < d) o[col0 + e] = red[tx * V + e];
  }
}

// Sum the row-split partials: a 256-thread CTA covers 32 columns; thread
// (c, g) adds splits g, g+8, g+16, ... of column c in increasing order, then
// the 8 group sums combine by a fixed pairwise tree.  Grid: x = column
// blocks of 32, y = batch.
__global__ void __launch_bounds__(256) score_finalize_kernel(const float* __restrict__ partial, int64_t d,
                                                             int64_t splits, float* __restrict__ ss, int64_t ld_ss,
                                                             int sqrt_out) {
  __shared__ float part[8][33];
  pdl_wait();
  pdl_trigger();
  const int c = threadIdx.x & 31, g = threadIdx.x >> 5;
  const int64_t j = static_cast<int64_t>(blockIdx.x) * 32 + c;
  const float* p = partial + static_cast<int64_t>(blockIdx.y) * splits * d + j;
  float acc = 0.f;
  if (j < d) {
    int64_t s = g;
    for (; s + 24 < splits; s += 32) {  // four independent loads in flight, added in split order
      const float a0 = __ldg(p + s * d), a1 = __ldg(p + (s + 8) * d);
      const float a2 = __ldg(p + (s + 16) * d), a3 = __ldg(p + (s + 24) * d);
      acc += a0;
      acc += a1;
      acc += a2;
      acc += a3;
    }
    for (; s < splits; s += 8) acc += __ldg(p + s * d);
  }
  part[g][c] = acc;
  __syncthreads();
  if (g == 0 && j < d) {
    const float t = ((part[0][c] + part[1][c]) + (part[2][c] + part[3][c])) +
                    ((part[4][c] + part[5][c]) + (part[6][c] + part[7][c]));
    ss[static_cast<int64_t>(blockIdx.y) * ld_ss + j] = sqrt_out ? sqrtf(t) : t;
  }
}

}  // namespace

ScorePlan score_plan(int dtype, int64_t batch, int64_t M, int64_t d) {
  ScorePlan p{};
  p.vec = dtype == 1 ? 8 : 4;
  const int64_t vecs = (d + p.vec - 1) / p.vec;
  int ct = 1;
  while (ct < 64 && ct < vecs) ct <<= 1;
  p.col_threads = ct;
  p.row_groups = kScoreThreads / ct;
  p.strips = (vecs + ct - 1) / ct;
  const int64_t rps = static_cast<int64_t>(kRowsPerThread) * p.row_groups;
  p.rows_per_split = rps;
  p.splits = M > 0 ? (M + rps - 1) / rps : 1;
  return p;
}

size_t score_workspace_bytes(int dtype, int64_t batch, int64_t M, int64_t d) {
  const ScorePlan p = score_plan(dtype, batch, M, d);
  if (p.splits <= 1) return 0;
  return align_up(static_cast<size_t>(batch) * p.splits * d * sizeof(float), kWsAlign);
}

namespace {

// One-launch plan for bf16.  The grid is one wave of resident CTAs (two per
// SM): each (column strip, row split, batch) CTA streams its rows through the
// ring above from start to end, so no SM idles behind a partial second wave.
// Among column-strip widths (col_threads 64 down to 4 vectors) the plan takes
// the one whose strips x splits x batch fills the most of that wave, the
// widest on ties (longer contiguous row segments); splits are at most 8 (one
// cluster) and at least 16 rows per thread.  Shapes with more strips than the
// wave holds take several waves of single-split CTAs.
struct ClusterScorePlan {
  int col_threads;
  int64_t strips, splits, rows_per_split;
};

ClusterScorePlan cluster_score_plan(int64_t batch, int64_t M, int64_t d) {
  const int64_t slots = 2 * static_cast<int64_t>(std::max(device_sm_count(), 1));
  const int64_t vecs = (d + 7) / 8;
  int ct0 = 4;
  while (ct0 < 64 && ct0 < vecs) ct0 <<= 1;  // no wider than the row
  ClusterScorePlan best{};
  int64_t best_fill = -1;
  for (int ct = ct0; ct >= 4; ct >>= 1) {
    const int rg = kScoreThreads / ct;
    const int64_t strips = (vecs + ct - 1) / ct;
    const int64_t max_splits = std::min<int64_t>(std::max<int64_t>((M + 16 * rg - 1) / (16 * rg), 1), 8);
    const int64_t per_split = strips * batch;
    const int64_t splits = std::max<int64_t>(std::min<int64_t>(max_splits, slots / std::max<int64_t>(per_split, 1)), 1);
    const int64_t ctas = per_split * splits;
    const int64_t fill = std::min(ctas, slots);
    if (fill > best_fill) {
      best_fill = fill;
      best = {ct, strips, splits, (M + splits - 1) / splits};
    }
  }
  return best;
}

}  // namespace

namespace {

// 16-byte vector loads are possible: aligned base, row pitch and batch stride.
bool score_vec_ok(const void* A, int dtype, int64_t batch, int64_t lda, int64_t batch_stride) {
  const size_t elt = dtype == 1 ? 2 : 4;
  return (reinterpret_cast<uintptr_t>(A) % 16 == 0) && ((lda * elt) % 16 == 0) &&
         (batch == 1 || (batch_stride * elt) % 16 == 0);
}

// The one-launch cluster kernel serves this call (it writes no partial sums).
bool score_cluster_path(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                        int64_t batch_stride) {
  return dtype == 1 && score_vec_ok(A, dtype, batch, lda, batch_stride) && M > 0 && batch <= 65535 &&
         cluster_score_plan(batch, M, d).strips <= 0x7FFFFFFFLL;
}

}  // namespace

size_t score_workspace_used(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                            int64_t batch_stride) {
  if (M == 0 || score_cluster_path(A, dtype, batch, M, d, lda, batch_stride)) return 0;
  return score_workspace_bytes(dtype, batch, M, d);
}

cudaError_t launch_score(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                         int64_t batch_stride, float* ss, int64_t ld_ss, int sqrt_out, void* ws,
                         cudaStream_t stream) {
  const ScorePlan p = score_plan(dtype, batch, M, d);
  const bool vec_ok = score_vec_ok(A, dtype, batch, lda, batch_stride);
  if (score_cluster_path(A, dtype, batch, M, d, lda, batch_stride)) {
    const ClusterScorePlan c = cluster_score_plan(batch, M, d);
    {
      cudaLaunchConfig_t cfg{};
      cfg.gridDim = dim3(static_cast<unsigned>(c.strips), static_cast<unsigned>(c.splits),
                         static_cast<unsigned>(batch));
      cfg.blockDim = dim3(kScoreThreads);
      cfg.dynamicSmemBytes = 0;
      cfg.stream = stream;
      cudaLaunchAttribute attr[2];
      attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
      attr[0].val.programmaticStreamSerializationAllowed = 1;
      attr[1].id = cudaLaunchAttributeClusterDimension;
      attr[1].val.clusterDim.x = 1;
      attr[1].val.clusterDim.y = static_cast<unsigned>(c.splits);
      attr[1].val.clusterDim.z = 1;
      cfg.attrs = attr;
      cfg.numAttrs = 2;
      return cudaLaunchKernelEx(&cfg, score_cluster_kernel, static_cast<const __nv_bfloat16*>(A), M, d, lda,
                                batch_stride, c.col_threads, c.rows_per_split, ss, ld_ss, sqrt_out);
    }
  }
  const dim3 grid(static_cast<unsigned>(p.strips), static_cast<unsigned>(p.splits), static_cast<unsigned>(batch));
  const bool direct = p.splits <= 1;
  float* out = direct ? ss : static_cast<float*>(ws);
  const int64_t out_bs = direct ? ld_ss : p.splits * d;
  const int64_t out_ss = direct ? 0 : d;
  const int sq = direct ? sqrt_out : 0;
  cudaError_t e;
  if (dtype == 1) {
    e = launch_pdl(score_partial_kernel<__nv_bfloat16>, grid, dim3(kScoreThreads), 0, stream,
                   static_cast<const __nv_bfloat16*>(A), M, d, lda, batch_stride, p.col_threads, p.rows_per_split,
                   vec_ok, out, out_bs, out_ss, sq);
  } else {
    e = launch_pdl(score_partial_kernel<float>, grid, dim3(kScoreThreads), 0, stream, static_cast<const float*>(A),
                   M, d, lda, batch_stride, p.col_threads, p.rows_per_split, vec_ok, out, out_bs, out_ss, sq);
  }
  if (e != cudaSuccess || direct) return e;
  const dim3 g2(static_cast<unsigned>((d + 31) / 32), static_cast<unsigned>(batch));
  return launch_pdl(score_finalize_kernel, g2, dim3(256), 0, stream, static_cast<const float*>(ws), d, p.splits, ss,
                    ld_ss, sqrt_out);
}

cudaError_t launch_silu_mul_score(const void* G, int64_t ldg, const void* U, int64_t ldu, void* H, int64_t ldh,
                                  int64_t M, int64_t d, float* ss, void* ws, cudaStream_t stream) {
  const ScorePlan p = score_plan(1, 1, M, d);
  const dim3 grid(static_cast<unsigned>(p.strips), static_cast<unsigned>(p.splits));
  const bool direct = p.splits <= 1;
  float* out = direct ? ss : static_cast<float*>(ws);
  cudaError_t e = launch_pdl(silu_mul_score_kernel, grid, dim3(kScoreThreads), 0, stream,
                             static_cast<const __nv_bfloat16*>(G), ldg, static_cast<const __nv_bfloat16*>(U), ldu,
                             static_cast<__nv_bfloat16*>(H), ldh, M, d, p.col_threads, p.rows_per_split, out,
                             direct ? int64_t{0} : d);
  if (e != cudaSuccess || direct) return e;
  const dim3 g2(static_cast<unsigned>((d + 31) / 32), 1u);
  return launch_pdl(score_finalize_kernel, g2, dim3(256), 0, stream, static_cast<const float*>(ws), d, p.splits, ss,
                    d, 0);
}

}  // namespace rmm
