// rmm_decode_attention.cu — reduced attention for one new query token per
// sequence over a KV cache (Reduced Matrix Multiplication technical summary:
// Metodología › Alcance de Aplicación reduces the feature dimension of QK^T
// and the token dimension of PV; Resultados Experimentales runs the method
// in autoregressive generation, one token per step).
//
// Per (sequence b, q-head h), with kv-head g = h * Hkv / Hq:
//   I_d = top ceil(rho_d D) of q_c^2 (lowest index first among equals);
//   s_j = scale * sum_{c in I_d} q_c K[g, j, c] for the L cached tokens;
//   lse = logsumexp_j s_j;  P_j = exp(s_j - lse);
//   I_t = top ceil(rho_t L) of t_j = P_j^2;  O = sum_{j in I_t} P_j V[g, j, :].
//
// Six launches on one stream (programmatic dependent launch between them):
//  1. dec_select_kernel, one warp per (b, h): the head_dim set from the query
//     row; the query is kept as fp32 with the dropped entries zeroed.
//  2. dec_logits_kernel, grid (token chunks of 128, B * Hkv): the chunk's key
//     rows are copied into shared memory with coalesced 16-byte asynchronous
//     copies (rows padded by 16 bytes, so 8x8 matrix loads hit no bank
//     twice); then each warp forms the logits of 32 tokens for every q-head
//     of the group as a tensor-core product (mma m16n8k16, bf16 operands,
//     fp32 accumulation): keys [tokens x head_dim] times the masked queries
//     [head_dim x heads].  The dropped entries add exact zeros, so each sum
//     is the reduced dot product.  Logits go to a [B*Hq, L] buffer; each CTA
//     also leaves its chunk's maximum and sum of exponentials per head.  A
//     plain FMA form of this contraction was bound by shared-memory traffic
//     and issue (about 800 instructions per key row) at half the HBM rate.
//  3. the histogram top-k over each head's L logits.  t_j = exp(2(s_j - lse))
//     is increasing in s_j, so ranking the logits ranks the token scores
//     (without the rounding of the exponential merging close values).
//  4. dec_prefix_kernel: for each head, where each 512-token chunk starts in
//     its ascending kept list.
//  5. dec_out_kernel, grid (token chunks of 512, B * Hkv): the weights
//     P_j = exp(s_j - lse) of every q-head of the group are scattered into a
//     table over the chunk's positions; the value rows kept by any of the
//     group's heads are read once each (16-byte asynchronous copies, six
//     stages of four rows per warp) and added into every head that keeps
//     them; per-chunk sums go to global memory.
//  6. dec_reduce_kernel: O = the chunk sums added in chunk order.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

constexpr int kDecThreads = 256;                // output and prefix kernels
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kLogitThreads = 128;              // logits kernel
constexpr int kDecChunk = kLogitThreads;        // tokens per logits CTA, one per thread
constexpr int kDecOutChunk = 512;               // token positions per output CTA
constexpr int kDecStages = 6;
constexpr int kDecRowsPerStage = 4;

struct DecParams {
  int B, Hq, Hkv, G, L, Lmax, kd, kt, chunks, out_chunks;
  float scale;
};

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
constexpr int key_pitch() { return D * 2 + 16; }  // bytes per staged key row

template <int D>
constexpr size_t dec_logits_smem() { return static_cast<size_t>(kDecChunk) * key_pitch<D>(); }

// The head_dim set of one (b, h), one warp: rank of q_c^2 (exact in fp32 for
// bf16 q) counting larger values and equal ones at lower indices.  Writes
// the query as fp32 with the dropped entries zeroed, and the ascending set.
template <int D>
__global__ void __launch_bounds__(32) dec_select_kernel(const uint16_t* __restrict__ q, DecParams p,
                                                        float* __restrict__ qm, int32_t* __restrict__ idx_d) {
  constexpr int PER = D / 32;
  __shared__ float sq[D];
  const int lane = threadIdx.x;
  const int64_t bh = blockIdx.x;
  pdl_wait();
  pdl_trigger();
  float v[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    v[e] = __uint_as_float(static_cast<uint32_t>(q[bh * D + lane * PER + e]) << 16);
    sq[lane * PER + e] = v[e] * v[e];
  }
  __syncwarp();
  int rank[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) rank[e] = 0;
#pragma unroll 16
  for (int c = 0; c < D; ++c) {
    const float sx = sq[c];
#pragma unroll
    for (int e = 0; e < PER; ++e) {
      const float se = sq[lane * PER + e];
      rank[e] += (sx > se || (sx == se && c < lane * PER + e)) ? 1 : 0;
    }
  }
  int nkept = 0;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const bool kept = rank[e] < p.kd;
    qm[bh * D + lane * PER + e] = kept ? v[e] : 0.f;
    nkept += kept ? 1 : 0;
  }
  if (idx_d) {
    // ascending position of each kept entry: kept entries at lower lanes, then lower e
    int before = nkept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, before, o);
      if (lane >= o) before += t;
    }
    before -= nkept;
#pragma unroll
    for (int e = 0; e < PER; ++e)
      if (rank[e] < p.kd) idx_d[bh * p.kd + before++] = lane * PER + e;
  }
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t (&r)[4]) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r[0]), "=r"(r[1]), "=r"(r[2]), "=r"(r[3])
               : "r"(addr));
}

// c += a b for one 16 x 8 x 16 tile (bf16 operands, fp32 accumulators).
__device__ __forceinline__ void mma_16816(float (&c)[4], const uint32_t (&a)[4], uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(c[0]), "+f"(c[1]), "+f"(c[2]), "+f"(c[3])
      : "r"(a[0]), "r"(a[1]), "r"(a[2]), "r"(a[3]), "r"(b0), "r"(b1));
}

template <int D, int G>
__global__ void __launch_bounds__(kLogitThreads)
    dec_logits_kernel(const float* __restrict__ qmask, const uint16_t* __restrict__ K, DecParams p,
                      float* __restrict__ logits, float2* __restrict__ part) {
  extern __shared__ __align__(128) uint8_t kt_smem[];  // [kDecChunk][key_pitch]
  constexpr int NW = kLogitThreads / 32;
  constexpr int NT = (G + 7) / 8;   // 8-head column tiles
  constexpr int KS = D / 16;        // 16-deep head_dim steps
  __shared__ float wred[NW][NT * 8];
  __shared__ float hmax[NT * 8];
  constexpr int PITCH = key_pitch<D>();
  constexpr int PIECES = D * 2 / 16;  // 16-byte pieces per key row
  const int chunk = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int gq = lane >> 2, cq = lane & 3;  // fragment row group and column pair of this lane
  const int j0 = chunk * kDecChunk;
  pdl_wait();
  pdl_trigger();

  // the chunk's key rows, coalesced: consecutive threads copy consecutive
  // pieces of a row; rows past L are zero-filled without a read
  {
    const char* Kg = reinterpret_cast<const char*>(K + (static_cast<int64_t>(b) * p.Hkv + g) * p.Lmax * D);
    const uint32_t base = smem_u32(kt_smem);
#pragma unroll 4
    for (int e = threadIdx.x; e < kDecChunk * PIECES; e += kLogitThreads) {
      const int r = e / PIECES, piece = e % PIECES;
      const bool ok = j0 + r < p.L;
      const void* src = ok ? static_cast<const void*>(Kg + static_cast<int64_t>(j0 + r) * D * 2 + piece * 16)
                           : static_cast<const void*>(Kg);
      cp_async16(base + r * PITCH + piece * 16, src, ok ? 16u : 0u);
    }
    cp_async_commit();
  }
  // B fragments: masked query of head (8 t + gq), head_dim 16 s + 2 cq (+1)
  // and 16 s + 2 cq + 8 (+1), as bf16 pairs (exact: the values are bf16)
  uint32_t bq[NT][KS][2];
  const float* qg = qmask + (static_cast<int64_t>(b) * p.Hq + g * G) * D;
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int hh = t * 8 + gq;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      if (hh < G) {
        const float2 lo = __ldg(reinterpret_cast<const float2*>(qg + hh * D + 16 * s + 2 * cq));
        const float2 hi = __ldg(reinterpret_cast<const float2*>(qg + hh * D + 16 * s + 2 * cq + 8));
        bq[t][s][0] = pack_bf16x2(lo.x, lo.y);
        bq[t][s][1] = pack_bf16x2(hi.x, hi.y);
      } else {
        bq[t][s][0] = 0u;
        bq[t][s][1] = 0u;
      }
    }
  }
  cp_async_wait<0>();
  __syncthreads();

  // warp w: tokens 32 w .. 32 w + 31 as two 16-row tiles
  float acc[2][NT][4];
#pragma unroll
  for (int mt = 0; mt < 2; ++mt)
#pragma unroll
    for (int t = 0; t < NT; ++t)
#pragma unroll
      for (int e = 0; e < 4; ++e) acc[mt][t][e] = 0.f;
  const uint32_t kbase = smem_u32(kt_smem);
#pragma unroll
  for (int mt = 0; mt < 2; ++mt) {
    const int row = warp * 32 + mt * 16 + (lane & 7) + ((lane >> 3) & 1) * 8;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      uint32_t a[4];
      ldsm_x4(kbase + row * PITCH + (16 * s + (lane >> 4) * 8) * 2, a);
#pragma unroll
      for (int t = 0; t < NT; ++t) mma_16816(acc[mt][t], a, bq[t][s][0], bq[t][s][1]);
    }
  }

  // accumulator (mt, t, e): token 32 w + 16 mt + gq + 8 (e >> 1), head 8 t + 2 cq + (e & 1)
  float mloc[NT][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int hh = t * 8 + 2 * cq + e2;
      float m = -INFINITY;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int j = j0 + warp * 32 + mt * 16 + gq + 8 * r;
          float& v = acc[mt][t][2 * r + e2];
          v *= p.scale;
          if (j < p.L) {
            if (hh < G) logits[(static_cast<int64_t>(b) * p.Hq + g * G + hh) * p.L + j] = v;
            m = fmaxf(m, v);
          }
        }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
      mloc[t][e2] = m;
    }
  }
  if (gq == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      wred[warp][t * 8 + 2 * cq] = mloc[t][0];
      wred[warp][t * 8 + 2 * cq + 1] = mloc[t][1];
    }
  }
  __syncthreads();
  if (threadIdx.x < NT * 8) {
    float m = -INFINITY;
    for (int w = 0; w < NW; ++w) m = fmaxf(m, wred[w][threadIdx.x]);
    hmax[threadIdx.x] = m;
  }
  __syncthreads();
#pragma unroll
  for (int t = 0; t < NT; ++t) {
#pragma unroll
    for (int e2 = 0; e2 < 2; ++e2) {
      const int hh = t * 8 + 2 * cq + e2;
      float z = 0.f;
#pragma unroll
      for (int mt = 0; mt < 2; ++mt)
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int j = j0 + warp * 32 + mt * 16 + gq + 8 * r;
          if (j < p.L) z += __expf(acc[mt][t][2 * r + e2] - hmax[hh]);
        }
#pragma unroll
      for (int o = 4; o < 32; o <<= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
      mloc[t][e2] = z;
    }
  }
  __syncthreads();  // every lane has read hmax before wred is reused
  if (gq == 0) {
#pragma unroll
    for (int t = 0; t < NT; ++t) {
      wred[warp][t * 8 + 2 * cq] = mloc[t][0];
      wred[warp][t * 8 + 2 * cq + 1] = mloc[t][1];
    }
  }
  __syncthreads();
  if (threadIdx.x < G) {
    float z = 0.f;
    for (int w = 0; w < NW; ++w) z += wred[w][threadIdx.x];
    part[(static_cast<int64_t>(b) * p.Hq + g * G + threadIdx.x) * p.chunks + chunk] = make_float2(hmax[threadIdx.x], z);
  }
}

// start[bh][c] = index in head bh's ascending kept list of its first token at
// or past position c * kDecOutChunk (c = 0 .. out_chunks; the last is k_t).
// One thread per list index r in [0, k_t]: it writes the chunks its step
// from entry r-1 to entry r crosses.
__global__ void __launch_bounds__(kDecThreads) dec_prefix_kernel(const int32_t* __restrict__ idx_t, DecParams p,
                                                                 int32_t* __restrict__ start) {
  pdl_wait();
  pdl_trigger();
  const int64_t bh = blockIdx.y;
  const int r = blockIdx.x * kDecThreads + threadIdx.x;
  if (r > p.kt) return;
  const int32_t* it = idx_t + bh * p.kt;
  int32_t* st = start + bh * (p.out_chunks + 1);
  auto chunk_of = [&](int i) {
    const int32_t j = __ldg(it + i);
    const int c = j < 0 ? 0 : j / kDecOutChunk;
    return c < p.out_chunks ? c : p.out_chunks - 1;
  };
  const int prev = r == 0 ? -1 : chunk_of(r - 1);
  const int cur = r == p.kt ? p.out_chunks : chunk_of(r);
  for (int c = prev + 1; c <= cur; ++c) st[c] = r;
}

template <int D, int G>
constexpr size_t dec_out_smem() {
  return static_cast<size_t>(kDecWarps) * kDecStages * kDecRowsPerStage * D * 2 +  // value rings
         static_cast<size_t>(G) * kDecOutChunk * 4 * 2 +                            // weights by position, by union row
         static_cast<size_t>(kDecOutChunk) * 4 * 2;                                 // kept flags, union list
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, 2)
    dec_out_kernel(const uint16_t* __restrict__ V, DecParams p, const float* __restrict__ logits,
                   const float2* __restrict__ part, const int32_t* __restrict__ idx_t,
                   const int32_t* __restrict__ start, float* __restrict__ opart, float* __restrict__ lse_out,
                   unsigned* err) {
  constexpr int ROWB = D * 2;                 // bytes of a value row
  constexpr int PIECES = ROWB / 16;           // 16-byte pieces per row
  constexpr int ROWS_PER_COPY = 32 / PIECES;  // rows one warp-wide copy instruction covers
  constexpr int DPL = D / 32;                 // dims per lane
  constexpr int RPS = kDecRowsPerStage;
  constexpr int S = kDecStages;
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ float red[kDecWarps][D];
  __shared__ float s_lse[G];
  __shared__ int s_cnt[kDecWarps];
  __shared__ int s_a[G], s_n[G];
  float* wtab = reinterpret_cast<float*>(smem + static_cast<size_t>(kDecWarps) * S * RPS * ROWB);  // [G][chunk]
  float* wrow = wtab + G * kDecOutChunk;  // [G][chunk]: the weights in union-row order, zero past the union
  int32_t* flag = reinterpret_cast<int32_t*>(wrow + G * kDecOutChunk);
  int32_t* list = flag + kDecOutChunk;
  const int chunk = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int p0 = chunk * kDecOutChunk;
  const int64_t bh0 = static_cast<int64_t>(b) * p.Hq + g * G;  // first q-head of the group
  for (int e = threadIdx.x; e < 2 * G * kDecOutChunk; e += kDecThreads) wtab[e] = 0.f;
  for (int e = threadIdx.x; e < kDecOutChunk; e += kDecThreads) flag[e] = 0;
  pdl_wait();
  pdl_trigger();

  // lse of each q-head of the group from the logits kernel's chunk partials
  for (int hh = warp; hh < G; hh += kDecWarps) {
    const float2* pp = part + (bh0 + hh) * p.chunks;
    float m = -INFINITY;
    for (int c = lane; c < p.chunks; c += 32) m = fmaxf(m, pp[c].x);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) m = fmaxf(m, __shfl_xor_sync(0xFFFFFFFFu, m, o));
    float z = 0.f;
    for (int c = lane; c < p.chunks; c += 32) z += pp[c].y * __expf(pp[c].x - m);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) z += __shfl_xor_sync(0xFFFFFFFFu, z, o);
    if (lane == 0) {
      s_lse[hh] = m + __logf(z);
      if (lse_out && chunk == 0) lse_out[bh0 + hh] = s_lse[hh];
    }
  }
  __syncthreads();

  // weights of the kept tokens in this chunk, every q-head at once: thread t
  // takes entries t, t + 256, ... of the heads' ranges laid end to end
  if (threadIdx.x < G) {
    const int32_t* st = start + (bh0 + threadIdx.x) * (p.out_chunks + 1);
    const int a = min(max(__ldg(st + chunk), 0), p.kt), e = min(max(__ldg(st + chunk + 1), a), p.kt);
    s_a[threadIdx.x] = a;
    s_n[threadIdx.x] = e - a;
  }
  __syncthreads();
  int total = 0;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) total += s_n[hh];
  bool bad = false;
  for (int f = threadIdx.x; f < total; f += kDecThreads) {
    int hh = 0, r = f;
    while (hh < G - 1 && r >= s_n[hh]) r -= s_n[hh++];
    const int32_t j = __ldg(idx_t + (bh0 + hh) * p.kt + s_a[hh] + r);
    if (j < p0 || j >= p0 + kDecOutChunk || j >= p.L) {
      bad = true;
      continue;
    }
    wtab[hh * kDecOutChunk + (j - p0)] = __expf(__ldg(logits + (bh0 + hh) * p.L + j) - s_lse[hh]);
    flag[j - p0] = 1;
  }
  if (bad) record_error(err, kDevErrBadIndex);
  __syncthreads();

  // the union of the group's kept rows, in position order
  constexpr int PT = kDecOutChunk / kDecThreads;  // positions per thread
  int mine = 0;
#pragma unroll
  for (int e = 0; e < PT; ++e) mine += flag[threadIdx.x * PT + e];
  int incl = mine;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const int t = __shfl_up_sync(0xFFFFFFFFu, incl, o);
    if (lane >= o) incl += t;
  }
  if (lane == 31) s_cnt[warp] = incl;
  __syncthreads();
  int before = incl - mine, n = 0;
  for (int w = 0; w < kDecWarps; ++w) {
    if (w < warp) before += s_cnt[w];
    n += s_cnt[w];
  }
#pragma unroll
  for (int e = 0; e < PT; ++e) {
    const int pos = threadIdx.x * PT + e;
    if (flag[pos]) {
#pragma unroll
      for (int hh = 0; hh < G; ++hh) wrow[hh * kDecOutChunk + before] = wtab[hh * kDecOutChunk + pos];
      list[before++] = pos;
    }
  }
  __syncthreads();

  // stream the union rows: warp w takes a contiguous run of them, four per
  // stage; a stage's four weights of a head are one 16-byte load, rows past
  // the run are copied as zeros with zero weight, so no row needs a test
  const char* Vg = reinterpret_cast<const char*>(V + (static_cast<int64_t>(b) * p.Hkv + g) * p.Lmax * D);
  const uint32_t ring = smem_u32(smem) + static_cast<uint32_t>(warp * S * RPS * ROWB);
  const int per = ((n + kDecWarps - 1) / kDecWarps + RPS - 1) / RPS * RPS;
  const int r0w = warp * per;
  const int rend = min(n, r0w + per);
  const int nst = rend > r0w ? (rend - r0w + RPS - 1) / RPS : 0;
  constexpr int NP = DPL / 2;  // dim pairs per lane
  uint64_t acc[G][NP];
#pragma unroll
  for (int hh = 0; hh < G; ++hh)
#pragma unroll
    for (int e = 0; e < NP; ++e) acc[hh][e] = 0ull;
  auto issue = [&](int stg) {
    if (stg < nst) {
      const uint32_t base = ring + static_cast<uint32_t>((stg % S) * RPS * ROWB);
#pragma unroll
      for (int h2 = 0; h2 < RPS / ROWS_PER_COPY; ++h2) {
        const int u = h2 * ROWS_PER_COPY + lane / PIECES, piece = lane % PIECES;
        const int row = r0w + stg * RPS + u;
        const bool ok = row < rend;
        const int j = ok ? p0 + list[row] : 0;
        cp_async16(base + u * ROWB + piece * 16, Vg + static_cast<int64_t>(j) * ROWB + piece * 16, ok ? 16u : 0u);
      }
    }
    cp_async_commit();
  };
#pragma unroll
  for (int stg = 0; stg < S - 1; ++stg) issue(stg);
  for (int stg = 0; stg < nst; ++stg) {
    issue(stg + S - 1);
    cp_async_wait<S - 1>();
    __syncwarp();
    const uint8_t* base = smem + (warp * S + stg % S) * RPS * ROWB + lane * DPL * 2;
    float4 w4[G];
#pragma unroll
    for (int hh = 0; hh < G; ++hh)
      w4[hh] = *reinterpret_cast<const float4*>(wrow + hh * kDecOutChunk + r0w + stg * RPS);
#pragma unroll
    for (int u = 0; u < RPS; ++u) {
      uint64_t v[NP];
      if constexpr (NP == 2) {
        const uint2 w = *reinterpret_cast<const uint2*>(base + u * ROWB);
        v[0] = f2_pack(bf16_lo(w.x), bf16_hi(w.x));
        v[1] = f2_pack(bf16_lo(w.y), bf16_hi(w.y));
      } else {
        const uint32_t w = *reinterpret_cast<const uint32_t*>(base + u * ROWB);
        v[0] = f2_pack(bf16_lo(w), bf16_hi(w));
      }
#pragma unroll
      for (int hh = 0; hh < G; ++hh) {
        const float wu = u == 0 ? w4[hh].x : u == 1 ? w4[hh].y : u == 2 ? w4[hh].z : w4[hh].w;
        const uint64_t ww = f2_pack(wu, wu);
#pragma unroll
        for (int e = 0; e < NP; ++e) acc[hh][e] = f2_fma(ww, v[e], acc[hh][e]);
      }
    }
    __syncwarp();
  }
  cp_async_wait<0>();

  // warps summed in a fixed order, one q-head at a time
  for (int hh = 0; hh < G; ++hh) {
#pragma unroll
    for (int e = 0; e < NP; ++e) f2_unpack(acc[hh][e], red[warp][lane * DPL + 2 * e], red[warp][lane * DPL + 2 * e + 1]);
    __syncthreads();
    if (threadIdx.x < D) {
      float v = 0.f;
#pragma unroll
      for (int w = 0; w < kDecWarps; ++w) v += red[w][threadIdx.x];
      opart[((bh0 + hh) * p.out_chunks + chunk) * D + threadIdx.x] = v;
    }
    __syncthreads();
  }
}

// O[bh, :] = sum over token chunks, in chunk order, of the chunk sums.
template <int D>
__global__ void __launch_bounds__(D) dec_reduce_kernel(const float* __restrict__ opart, DecParams p,
                                                       void* __restrict__ O, int out_f32) {
  pdl_wait();
  pdl_trigger();
  const int64_t bh = blockIdx.x;
  float v = 0.f;
  for (int c = 0; c < p.out_chunks; ++c) v += __ldg(opart + (bh * p.out_chunks + c) * D + threadIdx.x);
  if (out_f32)
    static_cast<float*>(O)[bh * D + threadIdx.x] = v;
  else
    static_cast<__nv_bfloat16*>(O)[bh * D + threadIdx.x] = __float2bfloat16_rn(v);
}

// Opt a kernel into `bytes` of dynamic shared memory, once per device (also
// below 48 KB: with its static arrays a kernel can pass the default limit).
template <auto Kernel>
bool allow_smem(size_t bytes) {
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

struct DecLayout {
  int chunks, out_chunks;
  size_t qm, logits, part, idx_t, start, opart, total;
};

DecLayout dec_layout(int64_t B, int64_t Hq, int64_t L, int64_t D, int64_t kt, bool own_logits, bool own_idx) {
  DecLayout w{};
  size_t off = 0;
  w.qm = off;
  off += align_up(static_cast<size_t>(B * Hq * D) * 4, kWsAlign);
  w.chunks = static_cast<int>((L + kDecChunk - 1) / kDecChunk);
  w.out_chunks = static_cast<int>((L + kDecOutChunk - 1) / kDecOutChunk);
  const size_t heads = static_cast<size_t>(B * Hq);
  w.logits = off;
  if (own_logits) off += align_up(heads * L * 4, kWsAlign);
  w.part = off;
  off += align_up(heads * w.chunks * 8, kWsAlign);
  w.idx_t = off;
  if (own_idx) off += align_up(heads * kt * 4, kWsAlign);
  w.start = off;
  off += align_up(heads * (w.out_chunks + 1) * 4, kWsAlign);
  w.opart = off;
  off += align_up(heads * w.out_chunks * D * 4, kWsAlign);
  w.total = off;
  return w;
}

template <int D, int G>
cudaError_t launch_dec(const void* q, const void* K, const void* V, const DecParams& p, float* qm, float* logits,
                       float2* part, int32_t* idx_d, int32_t* idx_t, int32_t* start, float* opart, void* O,
                       int out_f32, float* lse, unsigned* err, cudaStream_t stream) {
  cudaError_t e = launch_pdl(dec_select_kernel<D>, dim3(p.B * p.Hq), dim3(32), 0, stream,
                             static_cast<const uint16_t*>(q), p, qm, idx_d);
  if (e != cudaSuccess) return e;
  constexpr size_t lsm = dec_logits_smem<D>();
  if (!allow_smem<dec_logits_kernel<D, G>>(lsm)) return cudaErrorInvalidValue;
  e = launch_pdl(dec_logits_kernel<D, G>, dim3(p.chunks, p.B * p.Hkv), dim3(kLogitThreads), lsm, stream,
                 static_cast<const float*>(qm), static_cast<const uint16_t*>(K), p, logits, part);
  if (e != cudaSuccess) return e;
  e = launch_topk(logits, static_cast<int64_t>(p.B) * p.Hq, p.L, p.L, p.kt, idx_t, p.kt, stream);
  if (e != cudaSuccess) return e;
  e = launch_pdl(dec_prefix_kernel, dim3((p.kt + kDecThreads) / kDecThreads, p.B * p.Hq), dim3(kDecThreads), 0,
                 stream, static_cast<const int32_t*>(idx_t), p, start);
  if (e != cudaSuccess) return e;
  constexpr size_t osm = dec_out_smem<D, G>();
  if (!allow_smem<dec_out_kernel<D, G>>(osm)) return cudaErrorInvalidValue;
  e = launch_pdl(dec_out_kernel<D, G>, dim3(p.out_chunks, p.B * p.Hkv), dim3(kDecThreads), osm, stream,
                 static_cast<const uint16_t*>(V), p, static_cast<const float*>(logits),
                 static_cast<const float2*>(part), static_cast<const int32_t*>(idx_t),
                 static_cast<const int32_t*>(start), opart, lse, err);
  if (e != cudaSuccess) return e;
  return launch_pdl(dec_reduce_kernel<D>, dim3(p.B * p.Hq), dim3(D), 0, stream, static_cast<const float*>(opart), p,
                    O, out_f32);
}

template <int D>
cudaError_t launch_dec_g(const void* q, const void* K, const void* V, const DecParams& p, float* qm, float* logits,
                         float2* part,
                         int32_t* idx_d, int32_t* idx_t, int32_t* start, float* opart, void* O, int out_f32,
                         float* lse, unsigned* err, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_dec<D, 1>(q, K, V, p, qm, logits, part, idx_d, idx_t, start, opart, O, out_f32, lse, err, stream);
    case 2: return launch_dec<D, 2>(q, K, V, p, qm, logits, part, idx_d, idx_t, start, opart, O, out_f32, lse, err, stream);
    case 4: return launch_dec<D, 4>(q, K, V, p, qm, logits, part, idx_d, idx_t, start, opart, O, out_f32, lse, err, stream);
    case 8: return launch_dec<D, 8>(q, K, V, p, qm, logits, part, idx_d, idx_t, start, opart, O, out_f32, lse, err, stream);
    case 16:
      return launch_dec<D, 16>(q, K, V, p, qm, logits, part, idx_d, idx_t, start, opart, O, out_f32, lse, err, stream);
    default: return cudaErrorInvalidValue;
  }
}

}  // namespace

bool decode_attention_group_supported(int64_t G) { return G == 1 || G == 2 || G == 4 || G == 8 || G == 16; }

size_t decode_attention_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int64_t D, int64_t kt, bool own_logits,
                                        bool own_idx) {
  return dec_layout(B, Hq, L, D, kt, own_logits, own_idx).total;
}

cudaError_t launch_decode_attention(const void* q, const void* K, const void* V, int64_t B, int64_t Hq, int64_t Hkv,
                                    int64_t L, int64_t Lmax, int64_t D, int64_t kd, int64_t kt, float scale, void* O,
                                    int out_dtype, int32_t* idx_d, int32_t* idx_t, float* lse, float* logits,
                                    void* ws, unsigned* err, cudaStream_t stream) {
  const DecLayout w = dec_layout(B, Hq, L, D, kt, logits == nullptr, idx_t == nullptr);
  char* base = static_cast<char*>(ws);
  float* lg = logits ? logits : reinterpret_cast<float*>(base + w.logits);
  float2* part = reinterpret_cast<float2*>(base + w.part);
  int32_t* it = idx_t ? idx_t : reinterpret_cast<int32_t*>(base + w.idx_t);
  int32_t* start = reinterpret_cast<int32_t*>(base + w.start);
  float* opart = reinterpret_cast<float*>(base + w.opart);
  float* qm = reinterpret_cast<float*>(base + w.qm);
  DecParams p{};
  p.B = static_cast<int>(B);
  p.Hq = static_cast<int>(Hq);
  p.Hkv = static_cast<int>(Hkv);
  p.G = static_cast<int>(Hq / Hkv);
  p.L = static_cast<int>(L);
  p.Lmax = static_cast<int>(Lmax);
  p.kd = static_cast<int>(kd);
  p.kt = static_cast<int>(kt);
  p.chunks = w.chunks;
  p.out_chunks = w.out_chunks;
  p.scale = scale;
  const int out_f32 = out_dtype == 0 ? 1 : 0;
  if (D == 128)
    return launch_dec_g<128>(q, K, V, p, qm, lg, part, idx_d, it, start, opart, O, out_f32, lse, err, stream);
  return launch_dec_g<64>(q, K, V, p, qm, lg, part, idx_d, it, start, opart, O, out_f32, lse, err, stream);
}

}  // namespace rmm
