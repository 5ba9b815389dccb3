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
// Three launches on one stream (programmatic dependent launch between them):
//  1. dec_logits_kernel, grid (token chunks of 128, B * Hkv): the chunk's key
//     rows are copied into shared memory with coalesced 16-byte asynchronous
//     copies (rows padded by 16 bytes, so 8x8 matrix loads hit no bank
//     twice); while they arrive, each warp finds the head_dim set of a q-head
//     of the group (a bitwise search for the k_d-th largest |q_c| with warp
//     ballots) and leaves the masked query in shared memory.  Then each warp
//     forms the logits of 32 tokens for every q-head of the group as a
//     tensor-core product (mma m16n8k16, bf16 operands, fp32 accumulation):
//     keys [tokens x head_dim] times the masked queries [head_dim x heads].
//     The dropped entries add exact zeros, so each sum is the reduced dot
//     product.  Logits go to a [B*Hq, L] buffer; each CTA also leaves its
//     chunk's maximum and sum of exponentials per head.  (A plain FMA form of
//     this contraction was bound by shared-memory traffic and issue, about
//     800 instructions per key row, at half the HBM rate.)
//  2. dec_topk_kernel, the histogram top-k of rmm_select.cuh over each head's
//     L logits, on one CTA or a thread-block cluster of 2, 4 or 8 CTAs per
//     head (so that a few sequences still fill the SMs).  t_j = exp(2(s_j -
//     lse)) is increasing in s_j, so ranking the logits ranks the token
//     scores (without the rounding of the exponential merging close values).
//     It writes each head's kept tokens as a bitmap (and as the ascending
//     list idx_t when that is asked for or copies of the k_t-th largest
//     logit are split), the heads' lse, and clears the output kernel's
//     arrival counters.  (Rows too long for eight CTAs take the radix pass
//     of rmm_topk.cu, then dec_mark_kernel builds the bitmap.)
//  3. dec_out_kernel, grid (token chunks of 512, B * Hkv), four CTAs per SM
//     up to four q-heads per kv-head (two above): each warp takes 64 positions, i.e. two bitmap words per q-head of the
//     group; the union of the group's kept rows and each head's weights
//     P_j = exp(s_j - lse) (zero where the head drops j) come from one round
//     of independent loads, with no block barrier.  The union rows are read
//     once each (16-byte asynchronous copies, five stages of four rows per
//     warp) and added into every head that keeps them; the warps' sums are
//     added in a fixed order, per-chunk sums go to global memory, and the
//     group's last CTA to finish adds them in chunk order into O.
#include <cuda_bf16.h>

#include <algorithm>
#include <atomic>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"
#include "rmm_select.cuh"

namespace rmm {
namespace {

constexpr int kDecThreads = 256;                // output and bitmap kernels
constexpr int kDecWarps = kDecThreads / 32;
constexpr int kLogitThreads = 128;              // logits kernel
constexpr int kDecChunk = kLogitThreads;        // tokens per logits CTA, one per thread
constexpr int kDecOutChunk = 512;               // token positions per output CTA
constexpr int kDecStages = 5;
constexpr int kDecRowsPerStage = 4;
constexpr int kDecMaxSliceKeys = 51200;         // logits one top-k CTA stages (200 KB)
constexpr int kDecWarpTokens = kDecOutChunk / kDecWarps;  // token positions per output warp (64)
static_assert(kDecWarpTokens == 64, "an output warp covers two bitmap words");

struct DecParams {
  int B, Hq, Hkv, G, L, Lmax, kd, kt, chunks, out_chunks, nwords;
  float scale;
};

__device__ __forceinline__ float warp_max(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v = fmaxf(v, __shfl_xor_sync(0xFFFFFFFFu, v, o));
  return v;
}

__device__ __forceinline__ float warp_sum(float v) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xFFFFFFFFu, v, o);
  return v;
}

__device__ __forceinline__ float bf16_lo(uint32_t w) { return __uint_as_float(w << 16); }
__device__ __forceinline__ float bf16_hi(uint32_t w) { return __uint_as_float(w & 0xFFFF0000u); }

template <int D>
constexpr int key_pitch() { return D * 2 + 16; }  // bytes per staged key row

template <int D>
constexpr size_t dec_logits_smem() { return static_cast<size_t>(kDecChunk) * key_pitch<D>(); }

// The head_dim set of query row qh (D bf16 values), one warp: the kd entries
// of largest q_c^2, lowest index first among equals.  q_c^2 is ordered as
// |q_c|, whose bf16 bits without the sign are an order-preserving 15-bit
// key; the kd-th largest key T is found bit by bit (the largest t with at
// least kd keys >= t), then the keys above T and the first equal ones are
// kept.  Lane l holds entries l*PER .. l*PER + PER - 1.  Writes the masked
// row (dropped entries +0) as bf16 pairs to sqm, and, if idx_d is given, the
// ascending set.
template <int D>
__device__ __forceinline__ void head_dim_select(const uint16_t* __restrict__ qh, int kd, uint32_t* sqm,
                                                int32_t* __restrict__ idx_d) {
  constexpr int PER = D / 32;
  const int lane = threadIdx.x & 31;
  uint32_t bits[PER], key[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    bits[e] = __ldg(qh + lane * PER + e);
    key[e] = bits[e] & 0x7FFFu;
  }
  uint32_t T = 0u;
#pragma unroll 1
  for (int bit = 14; bit >= 0; --bit) {
    const uint32_t cand = T | (1u << bit);
    int n = 0;
#pragma unroll
    for (int e = 0; e < PER; ++e) n += __popc(__ballot_sync(0xFFFFFFFFu, key[e] >= cand));
    if (n >= kd) T = cand;
  }
  int gt = 0, eq_before = 0;
  const uint32_t below = (1u << lane) - 1u;
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    gt += __popc(__ballot_sync(0xFFFFFFFFu, key[e] > T));
    eq_before += __popc(__ballot_sync(0xFFFFFFFFu, key[e] == T) & below);
  }
  const int need = kd - gt;  // equal keys kept, lowest index first
  int nkept = 0;
  bool kept[PER];
#pragma unroll
  for (int e = 0; e < PER; ++e) {
    const bool eq = key[e] == T;
    kept[e] = key[e] > T || (eq && eq_before < need);
    eq_before += eq ? 1 : 0;
    nkept += kept[e] ? 1 : 0;
  }
#pragma unroll
  for (int i = 0; i < PER / 2; ++i)
    sqm[lane * (PER / 2) + i] = (kept[2 * i] ? bits[2 * i] : 0u) | ((kept[2 * i + 1] ? bits[2 * i + 1] : 0u) << 16);
  if (idx_d) {
    int before = nkept;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const int t = __shfl_up_sync(0xFFFFFFFFu, before, o);
      if (lane >= o) before += t;
    }
    before -= nkept;
#pragma unroll
    for (int e = 0; e < PER; ++e)
      if (kept[e]) idx_d[before++] = lane * PER + e;
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
    dec_logits_kernel(const uint16_t* __restrict__ q, const uint16_t* __restrict__ K, DecParams p,
                      float* __restrict__ logits, float2* __restrict__ part, int32_t* __restrict__ idx_d) {
  extern __shared__ __align__(128) uint8_t kt_smem[];  // [kDecChunk][key_pitch]
  constexpr int NW = kLogitThreads / 32;
  constexpr int NT = (G + 7) / 8;   // 8-head column tiles
  constexpr int KS = D / 16;        // 16-deep head_dim steps
  constexpr int QP = D / 2 + 4;     // words per masked query row (padded: the 8 heads of a fragment hit 8 banks)
  __shared__ float wred[NW][NT * 8];
  __shared__ float hmax[NT * 8];
  __shared__ uint32_t sqm[G][QP];   // the group's masked queries, bf16 pairs
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
  // while the keys arrive: the head_dim set of each q-head of the group,
  // warp w taking heads w, w + NW, ...; the first chunk's CTA writes idx_d
  for (int hh = warp; hh < G; hh += NW) {
    const int64_t bh = static_cast<int64_t>(b) * p.Hq + g * G + hh;
    head_dim_select<D>(q + bh * D, p.kd, sqm[hh], (idx_d && chunk == 0) ? idx_d + bh * p.kd : nullptr);
  }
  __syncthreads();
  // B fragments: masked query of head (8 t + gq), head_dim 16 s + 2 cq (+1)
  // and 16 s + 2 cq + 8 (+1), as bf16 pairs
  uint32_t bq[NT][KS][2];
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int hh = t * 8 + gq;
#pragma unroll
    for (int s = 0; s < KS; ++s) {
      bq[t][s][0] = hh < G ? sqm[hh][8 * s + cq] : 0u;
      bq[t][s][1] = hh < G ? sqm[hh][8 * s + cq + 4] : 0u;
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

// lse of head bh from the logits kernel's chunk partials (max, sum of
// exponentials), one warp; also zeroes the output kernel's arrival counter
// of the head's kv-group (from its first q-head).
__device__ __forceinline__ void head_lse(const float2* __restrict__ part, const DecParams& p, int64_t bh,
                                         float* __restrict__ lse_ws, float* __restrict__ lse_out,
                                         unsigned* __restrict__ arrivals) {
  const int lane = threadIdx.x & 31;
  const float2* pp = part + bh * p.chunks;
  float m = -INFINITY;
  for (int c = lane; c < p.chunks; c += 32) m = fmaxf(m, pp[c].x);
  m = warp_max(m);
  float z = 0.f;
  for (int c = lane; c < p.chunks; c += 32) z += pp[c].y * __expf(pp[c].x - m);
  z = warp_sum(z);
  if (lane == 0) {
    const float l = m + __logf(z);
    lse_ws[bh] = l;
    if (lse_out) lse_out[bh] = l;
    if (bh % p.G == 0) arrivals[bh / p.G] = 0u;
  }
}

// The token top-k of each head (grid x = the C CTAs of a cluster, y = head):
// CTA r stages the logits of tokens [r * slice, (r + 1) * slice) (slice a
// multiple of 32), takes its part of the exact selection (rmm_select.cuh;
// ranking the logits ranks t_j = exp(2 (s_j - lse))), and writes its kept
// tokens as bits of the head's kept-token bitmap (bit t % 32 of word t / 32)
// and, when the list is wanted or copies of the k_t-th largest logit are
// split, as the ascending list idx_t.  Rank 0 also forms the head's lse.
template <int NT, int C>
__global__ void __launch_bounds__(NT, 1)
    dec_topk_kernel(const float* __restrict__ logits, const float2* __restrict__ part, DecParams p, int slice,
                    int32_t* __restrict__ idx_t, int write_list, uint32_t* __restrict__ kept,
                    float* __restrict__ lse_ws, float* __restrict__ lse_out, unsigned* __restrict__ arrivals) {
  extern __shared__ __align__(16) uint32_t keys[];
  __shared__ __align__(16) uint32_t hist[(C > 1 ? 2 : 1) * kSelectBins];
  const int rank = C > 1 ? static_cast<int>(blockIdx.x) : 0;
  const int64_t bh = blockIdx.y;
  const int j0 = rank * slice;
  const int dl = max(0, min(slice, p.L - j0));
  pdl_wait();
  pdl_trigger();
  if (rank == 0 && threadIdx.x < 32) head_lse(part, p, bh, lse_ws, lse_out, arrivals);
  uint32_t kmin, kmax;
  stage_score_keys<NT>(logits + bh * p.L + j0, dl, keys, kmin, kmax);
  const SelectThreshold thr = select_threshold<NT, C>(keys, dl, static_cast<uint32_t>(p.kt), kmin, kmax, hist);
  const int nw = (dl + 31) / 32;
  uint32_t* kw = kept + bh * p.nwords + j0 / 32;
  if (!thr.split && !write_list) {
    // every key >= lo is kept: the bitmap straight from the staged keys, a
    // word per warp step (lane l tests key 32 w + l)
    if constexpr (C > 1) cluster_arrive();  // released only after every CTA's last read of the bins
    const uint32_t lo32 = static_cast<uint32_t>(thr.lo);
    const int lane = threadIdx.x & 31;
    for (int w = threadIdx.x >> 5; w < nw; w += NT / 32) {
      const int j = 32 * w + lane;
      const uint32_t bits = __ballot_sync(0xFFFFFFFFu, j < dl && keys[j] >= lo32);
      if (lane == 0) kw[w] = bits;
    }
    if constexpr (C > 1) cluster_wait();  // no CTA leaves while another may still read its shared memory
    return;
  }
  const StagedSelection sel = select_compact<NT, C>(keys, dl, thr);
  int32_t* out = idx_t + bh * p.kt;
  for (int q = threadIdx.x; q < static_cast<int>(sel.count); q += NT) out[sel.base + q] = j0 + static_cast<int32_t>(keys[q]);
  // the bitmap of the slice's words, built in the bins (no CTA reads them
  // any more: the search's last remote reads came before the compaction's
  // count exchange)
  for (int w = threadIdx.x; w < nw; w += NT) hist[w] = 0u;
  __syncthreads();
  for (int q = threadIdx.x; q < static_cast<int>(sel.count); q += NT) atomicOr(&hist[keys[q] >> 5], 1u << (keys[q] & 31u));
  __syncthreads();
  for (int w = threadIdx.x; w < nw; w += NT) kw[w] = hist[w];
  if constexpr (C > 1) cluster_wait();  // no CTA leaves while another may still read its shared memory
}

// Rows too long for a cluster to stage (their top-k is the radix pass of
// rmm_topk.cu): the kept-token bitmap from the finished ascending list, one
// thread per word (the word's first entry found by bisection), and the lse.
__global__ void __launch_bounds__(kDecThreads) dec_mark_kernel(const int32_t* __restrict__ idx_t,
                                                               const float2* __restrict__ part, DecParams p,
                                                               uint32_t* __restrict__ kept,
                                                               float* __restrict__ lse_ws,
                                                               float* __restrict__ lse_out,
                                                               unsigned* __restrict__ arrivals) {
  pdl_wait();
  pdl_trigger();
  const int64_t bh = blockIdx.y;
  if (blockIdx.x == 0 && threadIdx.x < 32) head_lse(part, p, bh, lse_ws, lse_out, arrivals);
  const int w = blockIdx.x * kDecThreads + threadIdx.x;
  if (w >= p.nwords) return;
  const int32_t* it = idx_t + bh * p.kt;
  int lo = 0, hi = p.kt;  // first entry >= 32 w
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (it[mid] < 32 * w) lo = mid + 1;
    else hi = mid;
  }
  uint32_t bits = 0u;
  for (int i = lo; i < p.kt && it[i] < 32 * w + 32; ++i) bits |= 1u << (it[i] - 32 * w);
  kept[bh * p.nwords + w] = bits;
}

template <int D, int G>
constexpr size_t dec_out_smem() {
  return static_cast<size_t>(kDecWarps) * kDecStages * kDecRowsPerStage * D * 2 +  // value rings
         static_cast<size_t>(kDecWarps) * kDecWarpTokens * 4 * (G + 1);             // weights, union list
}

template <int D, int G>
__global__ void __launch_bounds__(kDecThreads, G <= 4 ? 4 : 2)
    dec_out_kernel(const uint16_t* __restrict__ V, DecParams p, const float* __restrict__ logits,
                   const float* __restrict__ lse_ws, const uint32_t* __restrict__ kept, float* __restrict__ opart,
                   void* __restrict__ O, int out_f32, unsigned* __restrict__ arrivals) {
  constexpr int ROWB = D * 2;                 // bytes of a value row
  constexpr int PIECES = ROWB / 16;           // 16-byte pieces per row
  constexpr int ROWS_PER_COPY = 32 / PIECES;  // rows one warp-wide copy instruction covers
  constexpr int DPL = D / 32;                 // dims per lane
  constexpr int RPS = kDecRowsPerStage;
  constexpr int S = kDecStages;
  constexpr int WT = kDecWarpTokens;          // token positions per warp (two bitmap words)
  extern __shared__ __align__(128) uint8_t smem[];
  __shared__ unsigned s_last;
  const int chunk = blockIdx.x;
  const int b = blockIdx.y / p.Hkv, g = blockIdx.y % p.Hkv;
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t bh0 = static_cast<int64_t>(b) * p.Hq + g * G;  // first q-head of the group
  const int pw = chunk * kDecOutChunk + warp * WT;              // this warp's first token position
  int32_t* list = reinterpret_cast<int32_t*>(smem + static_cast<size_t>(kDecWarps) * S * RPS * ROWB) + warp * WT;
  float* wl = reinterpret_cast<float*>(smem + static_cast<size_t>(kDecWarps) * S * RPS * ROWB +
                                       static_cast<size_t>(kDecWarps) * WT * 4) + warp * G * WT;
  pdl_wait();
  pdl_trigger();

  // every head's kept bits, lse and logits over the warp's positions: one
  // round of independent loads
  const int w0 = pw >> 5;
  uint32_t m0[G], m1[G];
  float lg0[G], lg1[G], ls[G];
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    const uint32_t* kb = kept + (bh0 + hh) * p.nwords;
    const float* lr = logits + (bh0 + hh) * p.L;
    m0[hh] = w0 < p.nwords ? kb[w0] : 0u;
    m1[hh] = w0 + 1 < p.nwords ? kb[w0 + 1] : 0u;
    ls[hh] = lse_ws[bh0 + hh];
    lg0[hh] = pw + lane < p.L ? lr[pw + lane] : 0.f;
    lg1[hh] = pw + 32 + lane < p.L ? lr[pw + 32 + lane] : 0.f;
  }
  // the union of the group's kept rows in position order, with each head's
  // weight P_j = exp(s_j - lse) (zero where the head does not keep j)
  uint32_t u0 = 0u, u1 = 0u;
#pragma unroll
  for (int hh = 0; hh < G; ++hh) {
    u0 |= m0[hh];
    u1 |= m1[hh];
  }
  const int n0 = __popc(u0), n = n0 + __popc(u1);
  const uint32_t below = (1u << lane) - 1u;
  if ((u0 >> lane) & 1u) {
    const int r = __popc(u0 & below);
    list[r] = lane;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) wl[hh * WT + r] = ((m0[hh] >> lane) & 1u) ? __expf(lg0[hh] - ls[hh]) : 0.f;
  }
  if ((u1 >> lane) & 1u) {
    const int r = n0 + __popc(u1 & below);
    list[r] = 32 + lane;
#pragma unroll
    for (int hh = 0; hh < G; ++hh) wl[hh * WT + r] = ((m1[hh] >> lane) & 1u) ? __expf(lg1[hh] - ls[hh]) : 0.f;
  }
  // rows past the union in its last stage are copied as zeros with zero weight
  const int npad = (n + RPS - 1) / RPS * RPS;
  if (n + lane < npad) {
#pragma unroll
    for (int hh = 0; hh < G; ++hh) wl[hh * WT + n + lane] = 0.f;
  }
  __syncwarp();

  // stream the union rows, four per stage; a stage's four weights of a head
  // are one 16-byte load
  const char* Vg = reinterpret_cast<const char*>(V + (static_cast<int64_t>(b) * p.Hkv + g) * p.Lmax * D);
  const uint32_t ring = smem_u32(smem) + static_cast<uint32_t>(warp * S * RPS * ROWB);
  const int nst = npad / RPS;
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
        const int row = stg * RPS + u;
        const bool ok = row < n;
        const int j = ok ? pw + list[row] : 0;
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
    for (int hh = 0; hh < G; ++hh) w4[hh] = *reinterpret_cast<const float4*>(wl + hh * WT + stg * RPS);
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

  // warps summed in a fixed order, HP q-heads per pass, in the value rings'
  // space (every warp has finished with its ring at the barrier)
  constexpr int HP = (S * RPS * ROWB / (D * 4)) < G ? (S * RPS * ROWB / (D * 4)) : G;
  float* scr = reinterpret_cast<float*>(smem);  // [kDecWarps][HP][D]
  __syncthreads();
#pragma unroll
  for (int h0 = 0; h0 < G; h0 += HP) {
#pragma unroll
    for (int hq = 0; hq < HP; ++hq) {
      if (h0 + hq < G) {
        float* dst = scr + (warp * HP + hq) * D + lane * DPL;
#pragma unroll
        for (int e = 0; e < NP; ++e) f2_unpack(acc[h0 + hq][e], dst[2 * e], dst[2 * e + 1]);
      }
    }
    __syncthreads();
    for (int o = threadIdx.x; o < HP * D; o += kDecThreads) {
      const int hq = o / D, dd = o % D;
      if (h0 + hq < G) {
        float v = 0.f;
#pragma unroll
        for (int w = 0; w < kDecWarps; ++w) v += scr[(w * HP + hq) * D + dd];
        opart[((bh0 + h0 + hq) * p.out_chunks + chunk) * D + dd] = v;
      }
    }
    __syncthreads();
  }

  // the group's last CTA to finish adds the chunk sums, in chunk order:
  // O[bh, :] = sum_c opart[bh, c, :]
  if (threadIdx.x == 0) {
    __threadfence();  // this CTA's chunk sums are visible before its arrival
    s_last = atomicAdd(arrivals + blockIdx.y, 1u) == static_cast<unsigned>(p.out_chunks) - 1u ? 1u : 0u;
  }
  __syncthreads();
  if (!s_last) return;
  __threadfence();
  // two outputs per thread at a time, their loads interleaved (64 in flight)
  auto put = [&](int e, float v) {
    if (out_f32)
      static_cast<float*>(O)[bh0 * D + e] = v;
    else
      static_cast<__nv_bfloat16*>(O)[bh0 * D + e] = __float2bfloat16_rn(v);
  };
  for (int e = threadIdx.x; e < G * D; e += 2 * kDecThreads) {
    const int e1 = e + kDecThreads < G * D ? e + kDecThreads : e;
    const float* s0 = opart + (bh0 + e / D) * p.out_chunks * D + e % D;
    const float* s1 = opart + (bh0 + e1 / D) * p.out_chunks * D + e1 % D;
    float v0 = 0.f, v1 = 0.f;
#pragma unroll 32
    for (int c = 0; c < p.out_chunks; ++c) {
      v0 += __ldcg(s0 + static_cast<int64_t>(c) * D);
      v1 += __ldcg(s1 + static_cast<int64_t>(c) * D);
    }
    put(e, v0);
    if (e1 != e) put(e1, v1);
  }
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
  size_t logits, part, idx_t, kept, opart, lse, arrivals, total;
};

DecLayout dec_layout(int64_t B, int64_t Hq, int64_t L, int64_t D, int64_t kt, bool own_logits, bool own_idx) {
  DecLayout w{};
  size_t off = 0;
  w.chunks = static_cast<int>((L + kDecChunk - 1) / kDecChunk);
  w.out_chunks = static_cast<int>((L + kDecOutChunk - 1) / kDecOutChunk);
  const size_t heads = static_cast<size_t>(B * Hq);
  w.logits = off;
  if (own_logits) off += align_up(heads * L * 4, kWsAlign);
  w.part = off;
  off += align_up(heads * w.chunks * 8, kWsAlign);
  w.idx_t = off;
  if (own_idx) off += align_up(heads * kt * 4, kWsAlign);
  w.kept = off;
  off += align_up(heads * ((L + 31) / 32) * 4, kWsAlign);
  w.opart = off;
  off += align_up(heads * w.out_chunks * D * 4, kWsAlign);
  w.lse = off;
  off += align_up(heads * 4, kWsAlign);
  w.arrivals = off;
  off += align_up(heads * 4, kWsAlign);  // one per kv-group (at most one per head)
  w.total = off;
  return w;
}

struct DecBuffers {
  float* logits;
  float2* part;
  int32_t *idx_d, *idx_t;
  int write_list;  // the caller asked for idx_t
  uint32_t* kept;
  float *opart, *lse_ws, *lse_out;
  unsigned* arrivals;
};

// Token top-k with the kept-token bitmaps: a cluster of C CTAs per head, or
// (rows longer than eight slices) the radix pass followed by dec_mark_kernel.
template <int C>
cudaError_t launch_dec_topk(const DecParams& p, const DecBuffers& b, cudaStream_t stream) {
  constexpr int NT = C > 1 ? 512 : 1024;  // the thread counts of rmm_topk.cu's plan
  const int slice = C > 1 ? (p.L + C - 1) / C : p.L;
  const int slice_c = C > 1 ? (slice + 31) / 32 * 32 : slice;
  if (!allow_smem<dec_topk_kernel<NT, C>>(static_cast<size_t>(kDecMaxSliceKeys) * 4)) return cudaErrorInvalidValue;
  const size_t bytes = static_cast<size_t>(slice_c) * 4;
  const dim3 grid(C, static_cast<unsigned>(p.B * p.Hq));
  if (C > 1)
    return launch_pdl_cluster(dec_topk_kernel<NT, C>, grid, dim3(NT), bytes, C, stream,
                              static_cast<const float*>(b.logits), static_cast<const float2*>(b.part), p, slice_c,
                              b.idx_t, b.write_list, b.kept, b.lse_ws, b.lse_out, b.arrivals);
  return launch_pdl(dec_topk_kernel<NT, C>, grid, dim3(NT), bytes, stream, static_cast<const float*>(b.logits),
                    static_cast<const float2*>(b.part), p, slice_c, b.idx_t, b.write_list, b.kept, b.lse_ws,
                    b.lse_out, b.arrivals);
}

// CTAs per head of the token top-k (0: the radix pass).  A cluster's slices
// are whole bitmap words, so a slice may hold up to 31 more keys than an
// even split.
int dec_topk_cluster(int64_t rows, int64_t L) {
  const int c = topk_cluster_size(rows, L);
  if (c <= 0) return 0;
  const int64_t slice = (L + c - 1) / c;
  const int64_t slice_c = c > 1 ? (slice + 31) / 32 * 32 : slice;
  return slice_c <= kDecMaxSliceKeys ? c : 0;
}

template <int D, int G>
cudaError_t launch_dec(const void* q, const void* K, const void* V, const DecParams& p, const DecBuffers& b, void* O,
                       int out_f32, cudaStream_t stream) {
  constexpr size_t lsm = dec_logits_smem<D>();
  if (!allow_smem<dec_logits_kernel<D, G>>(lsm)) return cudaErrorInvalidValue;
  cudaError_t e = launch_pdl(dec_logits_kernel<D, G>, dim3(p.chunks, p.B * p.Hkv), dim3(kLogitThreads), lsm, stream,
                             static_cast<const uint16_t*>(q), static_cast<const uint16_t*>(K), p, b.logits, b.part,
                             b.idx_d);
  if (e != cudaSuccess) return e;
  switch (dec_topk_cluster(static_cast<int64_t>(p.B) * p.Hq, p.L)) {
    case 1: e = launch_dec_topk<1>(p, b, stream); break;
    case 2: e = launch_dec_topk<2>(p, b, stream); break;
    case 4: e = launch_dec_topk<4>(p, b, stream); break;
    case 8: e = launch_dec_topk<8>(p, b, stream); break;
    default:
      e = launch_topk(b.logits, static_cast<int64_t>(p.B) * p.Hq, p.L, p.L, p.kt, b.idx_t, p.kt, stream);
      if (e == cudaSuccess)
        e = launch_pdl(dec_mark_kernel, dim3((p.nwords + kDecThreads - 1) / kDecThreads, p.B * p.Hq),
                       dim3(kDecThreads), 0, stream, static_cast<const int32_t*>(b.idx_t),
                       static_cast<const float2*>(b.part), p, b.kept, b.lse_ws, b.lse_out, b.arrivals);
  }
  if (e != cudaSuccess) return e;
  constexpr size_t osm = dec_out_smem<D, G>();
  if (!allow_smem<dec_out_kernel<D, G>>(osm)) return cudaErrorInvalidValue;
  return launch_pdl(dec_out_kernel<D, G>, dim3(p.out_chunks, p.B * p.Hkv), dim3(kDecThreads), osm, stream,
                    static_cast<const uint16_t*>(V), p, static_cast<const float*>(b.logits),
                    static_cast<const float*>(b.lse_ws), static_cast<const uint32_t*>(b.kept), b.opart, O, out_f32,
                    b.arrivals);
}

template <int D>
cudaError_t launch_dec_g(const void* q, const void* K, const void* V, const DecParams& p, const DecBuffers& b, void* O,
                         int out_f32, cudaStream_t stream) {
  switch (p.G) {
    case 1: return launch_dec<D, 1>(q, K, V, p, b, O, out_f32, stream);
    case 2: return launch_dec<D, 2>(q, K, V, p, b, O, out_f32, stream);
    case 4: return launch_dec<D, 4>(q, K, V, p, b, O, out_f32, stream);
    case 8: return launch_dec<D, 8>(q, K, V, p, b, O, out_f32, stream);
    case 16: return launch_dec<D, 16>(q, K, V, p, b, O, out_f32, stream);
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
                                    void* ws, cudaStream_t stream) {
  const DecLayout w = dec_layout(B, Hq, L, D, kt, logits == nullptr, idx_t == nullptr);
  char* base = static_cast<char*>(ws);
  DecBuffers b{};
  b.logits = logits ? logits : reinterpret_cast<float*>(base + w.logits);
  b.part = reinterpret_cast<float2*>(base + w.part);
  b.idx_d = idx_d;
  b.idx_t = idx_t ? idx_t : reinterpret_cast<int32_t*>(base + w.idx_t);
  b.write_list = idx_t ? 1 : 0;
  b.kept = reinterpret_cast<uint32_t*>(base + w.kept);
  b.opart = reinterpret_cast<float*>(base + w.opart);
  b.lse_ws = reinterpret_cast<float*>(base + w.lse);
  b.lse_out = lse;
  b.arrivals = reinterpret_cast<unsigned*>(base + w.arrivals);
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
  p.nwords = static_cast<int>((L + 31) / 32);
  p.scale = scale;
  const int out_f32 = out_dtype == 0 ? 1 : 0;
  if (D == 128) return launch_dec_g<128>(q, K, V, p, b, O, out_f32, stream);
  return launch_dec_g<64>(q, K, V, p, b, O, out_f32, stream);
}

}  // namespace rmm
