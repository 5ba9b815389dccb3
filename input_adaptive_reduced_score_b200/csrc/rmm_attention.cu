// rmm_attention.cu — reduced causal attention (Reduced Matrix Multiplication
// technical summary, Metodología › Alcance de Aplicación: reduce the feature
// dimension of QK^T and, optionally, the token dimension of PV; each
// reduction is the method's A_{:,I} B_{I,:} with A the activation-side
// operand).  Readings of what the page leaves open: head_dim indices are
// scored on Q over all S tokens, one set per (batch, q-head), shared by K; the
// logit scale stays 1/sqrt(D); P is the causal softmax of the reduced logits;
// tokens are scored by the squared column norms of P, one set per
// (batch, q-head); P is not renormalised over the kept tokens; q-head h reads
// kv-head h*Hkv/Hq.
//
// Steps (all on one stream, no host synchronisation):
//   1. column scores of Q per (b, h) and head_dim top-k    (rmm_score / rmm_topk kernels)
//   2. Q_I = Q[:, I_d], K_I = K_g[:, I_d] per q-head       (compact_heads_kernel)
//   3. pass A: lse_i = logsumexp_{j<=i} S_ij                (attn_qk_kernel<kLse>)
//   4. pass B: t_j = sum_{i>=j} exp(2 (S_ij - lse_i))       (attn_qk_kernel<kColScore>)
//   5. token top-k of t, causal prefix counts              (rmm_topk kernels, attn_prefix_kernel)
//   6. K_T = K_I[I_t], V_T = V_g[I_t] row gathers           (gather_heads_kernel)
//   7. pass C: O_i = sum_{r: pos_r <= i} exp(S_ir - lse_i) V_T[r]  (attn_out_kernel)
// with S_ij = scale * Q_I[i] . K_I[j].  Passes A-C are tcgen05 kernels: one
// TMA lane, one MMA lane, four softmax/epilogue warps; the 128 x 128 logit
// tile lives in tensor memory (double-buffered); pass C writes P as bf16 in
// the 128-byte-swizzled K-major layout into shared memory and accumulates
// O += P V_T in tensor memory.  Exponentials use the hardware ex2.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <chrono>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <mutex>
#include <thread>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int TILE = 128;                 // rows of every tile (queries or keys)
constexpr int CHUNK_BYTES = TILE * 128;   // one [128 x 64] bf16 tile, 128-byte rows: 16 KB
constexpr int ATT_THREADS = 192;          // warp 0 TMA, warp 1 MMA, warps 2-5 softmax
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;

struct AttnParams {
  int S;            // tokens
  int kc;           // 64-column chunks of Q_I / K_I rows (ceil(k_d / 64))
  int D;            // head dim of V and O (64 or 128)
  int kt;           // kept tokens
  int nqb;          // query (= key) blocks of 128
  int out_f32;      // O written as fp32 (else bf16)
  int c_stages;     // pass C key/value ring depth (1 or 2, as shared memory allows)
  float scale_log2; // logit scale times log2(e)
};

// ------------------------------------------------------------------ prep kernels

// dst[bh][s][c] = src[b][g][s][idx[bh][c]] for c < kd (g = h * Hsrc / Hq);
// 8 columns per thread.  Grid: x = item blocks, y = bh.
__global__ void __launch_bounds__(256) compact_heads_kernel(const __nv_bfloat16* __restrict__ src, int Hq, int Hsrc,
                                                            int S, int Dsrc, const int32_t* __restrict__ idx, int kd,
                                                            __nv_bfloat16* __restrict__ dst, int ldk) {
  const int bh = blockIdx.y, b = bh / Hq, h = bh % Hq, g = (h * Hsrc) / Hq;
  const int groups = (kd + 7) / 8;
  const int64_t item = static_cast<int64_t>(blockIdx.x) * 256 + threadIdx.x;
  if (item >= static_cast<int64_t>(S) * groups) return;
  const int s = static_cast<int>(item / groups), c0 = static_cast<int>(item % groups) * 8;
  const __nv_bfloat16* row = src + ((static_cast<int64_t>(b) * Hsrc + g) * S + s) * Dsrc;
  const int32_t* id = idx + static_cast<int64_t>(bh) * kd;
  alignas(16) __nv_bfloat16 v[8];
#pragma unroll
  for (int e = 0; e < 8; ++e) {
    const int c = c0 + e;
    v[e] = c < kd ? row[__ldg(id + c)] : __float2bfloat16_rn(0.f);
  }
  *reinterpret_cast<uint4*>(dst + (static_cast<int64_t>(bh) * S + s) * ldk + c0) = *reinterpret_cast<const uint4*>(v);
}

// dst[bh][r][:] = src[b][g][idx[bh][r]][:] (row_vecs 16-byte pieces per row);
// one warp per output row.  Grid: x = ceil(kt / 8), y = bh.
__global__ void __launch_bounds__(256) gather_heads_kernel(const uint4* __restrict__ src, int Hq, int Hsrc, int S,
                                                           int src_ld_vec, const int32_t* __restrict__ idx, int kt,
                                                           int row_vecs, uint4* __restrict__ dst, int dst_ld_vec) {
  const int bh = blockIdx.y, b = bh / Hq, h = bh % Hq, g = (h * Hsrc) / Hq;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= kt) return;
  const int j = __ldg(idx + static_cast<int64_t>(bh) * kt + r);
  const uint4* s = src + ((static_cast<int64_t>(b) * Hsrc + g) * S + j) * src_ld_vec;
  uint4* d = dst + (static_cast<int64_t>(bh) * kt + r) * dst_ld_vec;
  for (int v = lane; v < row_vecs; v += 32) d[v] = __ldg(s + v);
}

// nvalid[bh][qb] = number of kept positions <= the block's last query
// (the kept positions are ascending).  One thread per (bh, qb).
__global__ void attn_prefix_kernel(const int32_t* __restrict__ pos, int BH, int kt, int S, int nqb,
                                   int* __restrict__ nvalid) {
  const int t = blockIdx.x * blockDim.x + threadIdx.x;
  if (t >= BH * nqb) return;
  const int bh = t / nqb, qb = t % nqb;
  const int imax = min(S - 1, qb * TILE + TILE - 1);
  const int32_t* p = pos + static_cast<int64_t>(bh) * kt;
  int lo = 0, hi = kt;  // first index with p > imax
  while (lo < hi) {
    const int mid = (lo + hi) >> 1;
    if (__ldg(p + mid) <= imax) {
      lo = mid + 1;
    } else {
      hi = mid;
    }
  }
  nvalid[t] = lo;
}

// ------------------------------------------------------------------ passes A and B

enum { kLse = 0, kColScore = 1 };
constexpr int QK_STAGES = 3;

struct QkBars {
  uint64_t full[QK_STAGES], empty[QK_STAGES];
  uint64_t fixed_full;
  uint64_t sfull[2], sempty[2];
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
  float lsh[4][TILE];  // per softmax warp: log2-domain lse of the current query block
};

// Pass A (kLse): CTA = one query block; the Q tile is loaded once and key
//   blocks 0..qb stream through the ring; thread r of the softmax warps owns
//   query row r and keeps a running max / sum in the log2 domain.
// Pass B (kColScore): CTA = one key block; the K tile is loaded once and query
//   blocks kb..nqb-1 stream through; the tile in tensor memory is S^T (lane =
//   key), so thread r owns key r and sums exp(2 (S_ij - lse_i)) over its
//   queries with no cross-thread reduction: a 128-term block sum added into a
//   running total, queries in ascending order.
template <int MODE>
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_qk_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_k,
                   float* __restrict__ lse, float* __restrict__ tsc, AttnParams p, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t base = smem_u32(smem);
  const int tile_bytes = p.kc * CHUNK_BYTES;
  QkBars* bars = reinterpret_cast<QkBars*>(smem + (1 + QK_STAGES) * tile_bytes);
  volatile int* abort_flag = &bars->abort_flag;
  const uint32_t fixed_tile = base;
  auto ring = [&](uint32_t s) { return base + (1 + s) * tile_bytes; };
  auto full = [&](uint32_t s) { return smem_u32(&bars->full[s]); };
  auto empty = [&](uint32_t s) { return smem_u32(&bars->empty[s]); };
  auto sfull = [&](uint32_t b) { return smem_u32(&bars->sfull[b]); };
  auto sempty = [&](uint32_t b) { return smem_u32(&bars->sempty[b]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  // pass A: heaviest query blocks first; pass B: key block kb (kb = 0 is the heaviest)
  const int fixed_blk = MODE == kLse ? p.nqb - 1 - static_cast<int>(blockIdx.x) : static_cast<int>(blockIdx.x);
  const int n_stream = MODE == kLse ? fixed_blk + 1 : p.nqb - fixed_blk;
  const int first_stream = MODE == kLse ? 0 : fixed_blk;

  if (threadIdx.x == 0) {
    for (int s = 0; s < QK_STAGES; ++s) {
      mbar_init(full(s), 1);
      mbar_init(empty(s), 1);
    }
    mbar_init(smem_u32(&bars->fixed_full), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull(b), 1);
      mbar_init(sempty(b), 4);
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_slot), 256);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_slot;
  const void* tm_fixed = MODE == kLse ? static_cast<const void*>(&tm_q) : static_cast<const void*>(&tm_k);
  const void* tm_stream = MODE == kLse ? static_cast<const void*>(&tm_k) : static_cast<const void*>(&tm_q);

  if (warp == 0) {
    if (lane == 0) {
      mbar_arrive_expect_tx(smem_u32(&bars->fixed_full), tile_bytes);
      for (int c = 0; c < p.kc; ++c)
        tma_load_3d(fixed_tile + c * CHUNK_BYTES, tm_fixed, smem_u32(&bars->fixed_full), c * 64, fixed_blk * TILE, bh);
      uint32_t stage = 0, phase = 0, issued = 0;
      for (int it = 0; it < n_stream; ++it) {
        if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, err, 11)) break;
        mbar_arrive_expect_tx(full(stage), tile_bytes);
        for (int c = 0; c < p.kc; ++c)
          tma_load_3d(ring(stage) + c * CHUNK_BYTES, tm_stream, full(stage), c * 64, (first_stream + it) * TILE, bh);
        ++issued;
        if (++stage == QK_STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      wait_drain(smem_u32(&bars->fixed_full), 0);
      uint32_t st = stage, ph = phase;
      for (uint32_t j = 0; j < (issued < QK_STAGES ? issued : QK_STAGES); ++j) {
        if (st == 0) {
          st = QK_STAGES - 1;
          ph ^= 1u;
        } else {
          --st;
        }
        wait_drain(full(st), ph);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    constexpr uint32_t idesc = idesc_bf16_f32(TILE, TILE, false, false);
    bool ok = mbar_wait_warp(smem_u32(&bars->fixed_full), 0, abort_flag, err, 12);
    uint32_t stage = 0, phase = 0;
    for (int it = 0; ok && it < n_stream; ++it) {
      const uint32_t b = it & 1, sph = (it >> 1) & 1;
      if (!mbar_wait_warp(sempty(b), sph ^ 1u, abort_flag, err, 13)) break;
      if (!mbar_wait_warp(full(stage), phase, abort_flag, err, 14)) break;
      tc_fence_after();
      if (lane == 0) {
        for (int c = 0; c < p.kc; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(fixed_tile + c * CHUNK_BYTES + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(ring(stage) + c * CHUNK_BYTES + kk * 32, 16, 1024);
            mma_f16_ss(tmem_base + b * TILE, ad, bd, idesc, (c | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(empty(stage));
        mma_commit(sfull(b));
      }
      __syncwarp();
      if (++stage == QK_STAGES) {
        stage = 0;
        phase ^= 1u;
      }
    }
    if (lane == 0) {
      mma_commit(smem_u32(&bars->drain));
      wait_drain(smem_u32(&bars->drain), 0);
    }
    __syncwarp();
  } else {
    const int qtr = warp & 3;
    const int r = qtr * 32 + lane;                  // TMEM lane = tile row
    const int own = fixed_blk * TILE + r;           // this thread's query (A) or key (B)
    const uint32_t lane_off = static_cast<uint32_t>(qtr * 32) << 16;
    float m = -INFINITY, l = 0.f;                   // pass A state (log2 domain)
    float total = 0.f;                              // pass B state
    for (int it = 0; it < n_stream; ++it) {
      const uint32_t b = it & 1, sph = (it >> 1) & 1;
      const int sblk = first_stream + it;
      float* lsh = bars->lsh[qtr];
      if (MODE == kColScore) {
        // each warp keeps its own copy of the block's 128 lse values, so only
        // warp-level synchronisation is needed
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = sblk * TILE + u * 32 + lane;
          lsh[u * 32 + lane] = q < p.S ? lse[static_cast<int64_t>(bh) * p.S + q] * kLog2e : 0.f;
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(sfull(b), sph, abort_flag, err, 15)) break;
      tc_fence_after();
      float blk = 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem_base + b * TILE + cc * 32 + lane_off, v);
        tmem_wait_ld();
        if (MODE == kLse) {
          float x[32];
          float mx = -INFINITY;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = sblk * TILE + cc * 32 + e;
            x[e] = (j <= own && j < p.S) ? __uint_as_float(v[e]) * p.scale_log2 : -INFINITY;
            mx = fmaxf(mx, x[e]);
          }
          if (mx > -INFINITY) {
            const float mn = fmaxf(m, mx);
            float add = 0.f;
#pragma unroll
            for (int e = 0; e < 32; ++e) add += fast_exp2(x[e] - mn);
            l = l * fast_exp2(m - mn) + add;
            m = mn;
          }
        } else {
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int i = sblk * TILE + cc * 32 + e;
            const float pe = fast_exp2(2.f * (__uint_as_float(v[e]) * p.scale_log2 - lsh[cc * 32 + e]));
            blk += (i >= own && i < p.S) ? pe : 0.f;
          }
        }
      }
      total += blk;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty(b));
    }
    if (own < p.S) {
      if (MODE == kLse) {
        lse[static_cast<int64_t>(bh) * p.S + own] = (m + log2f(l)) * kLn2;
      } else {
        tsc[static_cast<int64_t>(bh) * p.S + own] = total;
      }
    }
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 256);
  }
}

// ------------------------------------------------------------------ pass C

constexpr int C_STAGES = 2;  // maximum key/value ring depth of pass C

struct OutBars {
  uint64_t kvfull[C_STAGES], kvempty[C_STAGES];
  uint64_t qfull;
  uint64_t sfull[2], sempty[2];
  uint64_t pfull[2], pempty[2];
  uint64_t ofull;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
  int pos[4][TILE];  // per softmax warp: token positions of the current kept block
};

// CTA = one query block.  Kept tokens are processed 128 at a time (only the
// blocks that hold a kept position <= the block's last query): S = Q_I K_T^T
// into tensor memory; the softmax warps turn row i into P_ir = exp(S_ir -
// lse_i) for kept positions <= i (else 0), store it as bf16 in the
// K-major 128-byte-swizzled layout, and the MMA lane accumulates O += P V_T
// (V_T read MN-major).  S and P are double-buffered so the softmax of block r
// overlaps the PV product of block r-1.
__global__ void __launch_bounds__(ATT_THREADS, 1)
    attn_out_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kt,
                    const __grid_constant__ CUtensorMap tm_vt, const float* __restrict__ lse,
                    const int32_t* __restrict__ pos, const int* __restrict__ nvalid, void* __restrict__ O,
                    AttnParams p, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t base = smem_u32(smem);
  const int dc = p.D / 64;
  const int q_bytes = p.kc * CHUNK_BYTES;
  const int kv_bytes = (p.kc + dc) * CHUNK_BYTES;
  const uint32_t q_tile = base;
  auto kv = [&](uint32_t s) { return base + q_bytes + s * kv_bytes; };
  const int nst = p.c_stages;
  const uint32_t p_base = base + q_bytes + nst * kv_bytes;  // two P buffers of 2 chunks
  auto pbuf = [&](uint32_t b) { return p_base + b * 2 * CHUNK_BYTES; };
  OutBars* bars = reinterpret_cast<OutBars*>(smem + q_bytes + nst * kv_bytes + 4 * CHUNK_BYTES);
  volatile int* abort_flag = &bars->abort_flag;
  auto kvfull = [&](uint32_t s) { return smem_u32(&bars->kvfull[s]); };
  auto kvempty = [&](uint32_t s) { return smem_u32(&bars->kvempty[s]); };
  auto sfull = [&](uint32_t b) { return smem_u32(&bars->sfull[b]); };
  auto sempty = [&](uint32_t b) { return smem_u32(&bars->sempty[b]); };
  auto pfull = [&](uint32_t b) { return smem_u32(&bars->pfull[b]); };
  auto pempty = [&](uint32_t b) { return smem_u32(&bars->pempty[b]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.y;
  const int qb = p.nqb - 1 - static_cast<int>(blockIdx.x);  // heaviest blocks first
  const int nv = __ldg(nvalid + static_cast<int64_t>(bh) * p.nqb + qb);
  const int nrb = (nv + TILE - 1) / TILE;

  if (threadIdx.x == 0) {
    for (int s = 0; s < nst; ++s) {
      mbar_init(kvfull(s), 1);
      mbar_init(kvempty(s), 1);
    }
    mbar_init(smem_u32(&bars->qfull), 1);
    for (int b = 0; b < 2; ++b) {
      mbar_init(sfull(b), 1);
      mbar_init(sempty(b), 4);
      mbar_init(pfull(b), 4);
      mbar_init(pempty(b), 1);
    }
    mbar_init(smem_u32(&bars->ofull), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc(smem_u32(&bars->tmem_slot), 512);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_slot;
  const uint32_t o_tmem = tmem_base + 2 * TILE;

  if (warp == 0) {
    if (lane == 0 && nrb > 0) {
      mbar_arrive_expect_tx(smem_u32(&bars->qfull), q_bytes);
      for (int c = 0; c < p.kc; ++c)
        tma_load_3d(q_tile + c * CHUNK_BYTES, &tm_q, smem_u32(&bars->qfull), c * 64, qb * TILE, bh);
      uint32_t stage = 0, phase = 0, issued = 0;
      for (int rb = 0; rb < nrb; ++rb) {
        if (!mbar_wait(kvempty(stage), phase ^ 1u, abort_flag, err, 21)) break;
        mbar_arrive_expect_tx(kvfull(stage), kv_bytes);
        for (int c = 0; c < p.kc; ++c)
          tma_load_3d(kv(stage) + c * CHUNK_BYTES, &tm_kt, kvfull(stage), c * 64, rb * TILE, bh);
        for (int c = 0; c < dc; ++c)
          tma_load_3d(kv(stage) + (p.kc + c) * CHUNK_BYTES, &tm_vt, kvfull(stage), c * 64, rb * TILE, bh);
        ++issued;
        if (++stage == static_cast<uint32_t>(nst)) {
          stage = 0;
          phase ^= 1u;
        }
      }
      wait_drain(smem_u32(&bars->qfull), 0);
      uint32_t st = stage, ph = phase;
      for (uint32_t j = 0; j < (issued < static_cast<uint32_t>(nst) ? issued : static_cast<uint32_t>(nst)); ++j) {
        if (st == 0) {
          st = nst - 1;
          ph ^= 1u;
        } else {
          --st;
        }
        wait_drain(kvfull(st), ph);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    constexpr uint32_t idesc_s = idesc_bf16_f32(TILE, TILE, false, false);
    const uint32_t idesc_o = idesc_bf16_f32(TILE, p.D, false, true);
    bool ok = nrb == 0 || mbar_wait_warp(smem_u32(&bars->qfull), 0, abort_flag, err, 22);
    // O += P(r) V_T(r)
    auto pv = [&](int r) -> bool {
      const uint32_t b = r & 1, pph = (r >> 1) & 1;
      const uint32_t st = r % nst;
      if (!mbar_wait_warp(pfull(b), pph, abort_flag, err, 23)) return false;
      tc_fence_after();
      if (lane == 0) {
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint64_t ad = sdesc_sw128(pbuf(b) + (kk / 4) * CHUNK_BYTES + (kk % 4) * 32, 16, 1024);
          const uint64_t bd = sdesc_sw128(kv(st) + p.kc * CHUNK_BYTES + kk * 16 * 128, CHUNK_BYTES, 1024);
          mma_f16_ss(o_tmem, ad, bd, idesc_o, (r | kk) != 0 ? 1u : 0u);
        }
        mma_commit(kvempty(st));
        mma_commit(pempty(b));
      }
      __syncwarp();
      return true;
    };
    for (int rb = 0; ok && rb < nrb; ++rb) {
      const uint32_t b = rb & 1, sph = (rb >> 1) & 1;
      const uint32_t st = rb % nst, kph = (rb / nst) & 1;
      // with a single key/value stage, block rb can only be loaded once the
      // PV product of rb-1 has released the stage: issue that product first
      if (nst == 1 && rb >= 1 && !pv(rb - 1)) {
        ok = false;
        break;
      }
      if (!mbar_wait_warp(kvfull(st), kph, abort_flag, err, 24)) {
        ok = false;
        break;
      }
      if (!mbar_wait_warp(sempty(b), sph ^ 1u, abort_flag, err, 25)) {
        ok = false;
        break;
      }
      tc_fence_after();
      if (lane == 0) {
        for (int c = 0; c < p.kc; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(q_tile + c * CHUNK_BYTES + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kv(st) + c * CHUNK_BYTES + kk * 32, 16, 1024);
            mma_f16_ss(tmem_base + b * TILE, ad, bd, idesc_s, (c | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(sfull(b));
      }
      __syncwarp();
      if (nst > 1 && rb >= 1 && !pv(rb - 1)) ok = false;
    }
    if (ok && nrb > 0) ok = pv(nrb - 1);
    if (lane == 0) {
      if (nrb > 0) mma_commit(smem_u32(&bars->ofull));
      mma_commit(smem_u32(&bars->drain));
      wait_drain(smem_u32(&bars->drain), 0);
    }
    __syncwarp();
  } else {
    const int qtr = warp & 3;
    const int r = qtr * 32 + lane;
    const int i = qb * TILE + r;
    const uint32_t lane_off = static_cast<uint32_t>(qtr * 32) << 16;
    const float L2 = i < p.S ? lse[static_cast<int64_t>(bh) * p.S + i] * kLog2e : 0.f;
    const int32_t* pos_bh = pos + static_cast<int64_t>(bh) * p.kt;
    bool ok = true;
    for (int rb = 0; rb < nrb; ++rb) {
      const uint32_t b = rb & 1, sph = (rb >> 1) & 1;
      int* psh = bars->pos[qtr];
      __syncwarp();
#pragma unroll
      for (int u = 0; u < 4; ++u) {
        const int kr = rb * TILE + u * 32 + lane;
        psh[u * 32 + lane] = kr < p.kt ? __ldg(pos_bh + kr) : 0x7FFFFFFF;
      }
      __syncwarp();
      if (!mbar_wait_warp(sfull(b), sph, abort_flag, err, 26) ||
          !mbar_wait_warp(pempty(b), sph ^ 1u, abort_flag, err, 27)) {
        ok = false;
        break;
      }
      tc_fence_after();
      uint8_t* prow = smem + (pbuf(b) - base) + r * 128;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(tmem_base + b * TILE + cc * 32 + lane_off, v);
        tmem_wait_ld();
        uint32_t w[16];
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          const int q0 = cc * 32 + 2 * e;
          const float p0 = psh[q0] <= i ? fast_exp2(__uint_as_float(v[2 * e]) * p.scale_log2 - L2) : 0.f;
          const float p1 = psh[q0 + 1] <= i ? fast_exp2(__uint_as_float(v[2 * e + 1]) * p.scale_log2 - L2) : 0.f;
          w[e] = pack_bf16x2(p0, p1);
        }
        // columns cc*32 .. cc*32+31: chunk cc/2, 16-byte pieces (cc%2)*4 .. +3, swizzled by row
        uint8_t* crow = prow + (cc >> 1) * CHUNK_BYTES;
#pragma unroll
        for (int q = 0; q < 4; ++q) {
          const int piece = (cc & 1) * 4 + q;
          *reinterpret_cast<uint4*>(crow + ((piece ^ (r & 7)) << 4)) =
              make_uint4(w[4 * q], w[4 * q + 1], w[4 * q + 2], w[4 * q + 3]);
        }
      }
      tc_fence_before();
      fence_proxy_async_smem();  // P is read by the tensor core (async proxy)
      __syncwarp();
      if (lane == 0) {
        mbar_arrive(sempty(b));
        mbar_arrive(pfull(b));
      }
    }
    // epilogue: O row i.  Every lane of the warp takes part in the tensor-memory
    // loads (warp-synchronous); only rows i < S are stored.
    const bool have = ok && nrb > 0 && mbar_wait_warp(smem_u32(&bars->ofull), 0, abort_flag, err, 28);
    if (have) tc_fence_after();
    for (int cc = 0; cc < p.D / 32; ++cc) {
      uint32_t v[32];
      if (have) {
        tmem_ld32(o_tmem + cc * 32 + lane_off, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (i >= p.S) continue;
      const int64_t off = (static_cast<int64_t>(bh) * p.S + i) * p.D + cc * 32;
      if (p.out_f32) {
        float4* y = reinterpret_cast<float4*>(static_cast<float*>(O) + off);
#pragma unroll
        for (int q = 0; q < 8; ++q)
          y[q] = make_float4(__uint_as_float(v[4 * q]), __uint_as_float(v[4 * q + 1]), __uint_as_float(v[4 * q + 2]),
                             __uint_as_float(v[4 * q + 3]));
      } else {
        uint4* y = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(O) + off);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          y[q] = make_uint4(pack_bf16x2(__uint_as_float(v[8 * q]), __uint_as_float(v[8 * q + 1])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 2]), __uint_as_float(v[8 * q + 3])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 4]), __uint_as_float(v[8 * q + 5])),
                            pack_bf16x2(__uint_as_float(v[8 * q + 6]), __uint_as_float(v[8 * q + 7])));
      }
    }
    tc_fence_before();
  }

  __syncthreads();
  if (warp == 1) {
    tc_fence_after();
    tmem_dealloc(tmem_base, 512);
  }
}

// ------------------------------------------------------------------ host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* ptr = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &ptr, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(ptr);
  });
  return fn;
}

// 3-D bf16 map over [heads][rows][pitch] with logical row length `cols`;
// boxes of 64 columns x 128 rows x 1 head, 128-byte swizzle.
bool encode_heads(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int64_t heads, int64_t pitch) {
  EncodeTiledFn encode = encode_fn();
  if (!encode) {
    set_error("rmm_attention: cuTensorMapEncodeTiled entry point unavailable");
    return false;
  }
  const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(pitch) * 2, static_cast<cuuint64_t>(pitch * rows) * 2};
  const cuuint32_t box[3] = {64, TILE, 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 3, const_cast<void*>(ptr), gdim, gstride, box,
                            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("rmm_attention: cuTensorMapEncodeTiled failed (CUresult %d)", static_cast<int>(r));
    return false;
  }
  return true;
}

struct AttnWs {
  size_t ss, score, idx_d, qi, ki, lse, tsc, idx_t, nvalid, kt_rows, vt_rows, total;
  int64_t ldk;
};

AttnWs attn_ws(int64_t B, int64_t Hq, int64_t S, int64_t D, int64_t kd, int64_t kt) {
  AttnWs w{};
  const int64_t BH = B * Hq;
  w.ldk = (kd + 7) / 8 * 8;
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t o = off;
    off += align_up(bytes, kWsAlign);
    return o;
  };
  w.ss = take(static_cast<size_t>(BH) * D * 4);
  w.score = take(score_workspace_bytes(1, BH, S, D));
  w.idx_d = take(static_cast<size_t>(BH) * kd * 4);
  w.qi = take(static_cast<size_t>(BH) * S * w.ldk * 2);
  w.ki = take(static_cast<size_t>(BH) * S * w.ldk * 2);
  w.lse = take(static_cast<size_t>(BH) * S * 4);
  w.tsc = take(static_cast<size_t>(BH) * S * 4);
  w.idx_t = take(static_cast<size_t>(BH) * kt * 4);
  w.nvalid = take(static_cast<size_t>(BH) * ((S + TILE - 1) / TILE) * 4);
  w.kt_rows = take(static_cast<size_t>(BH) * kt * w.ldk * 2);
  w.vt_rows = take(static_cast<size_t>(BH) * kt * D * 2);
  w.total = off;
  return w;
}

template <typename K>
bool set_smem(K kernel, int bytes) {
  return cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, bytes) == cudaSuccess;
}

// With RMM_DEBUG_SYNC set in the environment, every step of the attention
// pipeline is followed by a bounded wait (20 s) for the stream, and a step
// that does not finish is reported by name on stderr; the process then exits
// so the context (and any stuck kernel) is torn down.
bool debug_sync_enabled() {
  static const bool on = std::getenv("RMM_DEBUG_SYNC") != nullptr;
  return on;
}

cudaError_t debug_step(cudaStream_t stream, const char* what) {
  if (!debug_sync_enabled()) return cudaSuccess;
  const auto t0 = std::chrono::steady_clock::now();
  for (;;) {
    const cudaError_t e = cudaStreamQuery(stream);
    if (e == cudaSuccess) {
      std::fprintf(stderr, "rmm_attention: %s done\n", what);
      return cudaSuccess;
    }
    if (e != cudaErrorNotReady) {
      std::fprintf(stderr, "rmm_attention: %s failed: %s\n", what, cudaGetErrorString(e));
      return e;
    }
    if (std::chrono::steady_clock::now() - t0 > std::chrono::seconds(20)) {
      std::fprintf(stderr, "rmm_attention: %s did not finish within 20 s; exiting\n", what);
      std::fflush(stderr);
      std::_Exit(3);
    }
    std::this_thread::sleep_for(std::chrono::milliseconds(1));
  }
}

}  // namespace

size_t attention_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t S, int64_t D, int64_t kd, int64_t kt) {
  (void)Hkv;
  return attn_ws(B, Hq, S, D, kd, kt).total;
}

cudaError_t launch_attention(const void* Q, const void* K, const void* V, int64_t B, int64_t Hq, int64_t Hkv,
                             int64_t S, int64_t D, int64_t kd, int64_t kt, float scale, void* O, int out_dtype,
                             int32_t* idx_d_out, int32_t* idx_t_out, float* lse_out, float* tscore_out, void* ws,
                             unsigned* err, cudaStream_t stream) {
  const AttnWs w = attn_ws(B, Hq, S, D, kd, kt);
  const int64_t BH = B * Hq;
  char* base = static_cast<char*>(ws);
  float* ss = reinterpret_cast<float*>(base + w.ss);
  int32_t* idx_d = idx_d_out ? idx_d_out : reinterpret_cast<int32_t*>(base + w.idx_d);
  __nv_bfloat16* qi = reinterpret_cast<__nv_bfloat16*>(base + w.qi);
  __nv_bfloat16* ki = reinterpret_cast<__nv_bfloat16*>(base + w.ki);
  float* lse = lse_out ? lse_out : reinterpret_cast<float*>(base + w.lse);
  float* tsc = tscore_out ? tscore_out : reinterpret_cast<float*>(base + w.tsc);
  int32_t* idx_t = idx_t_out ? idx_t_out : reinterpret_cast<int32_t*>(base + w.idx_t);
  int* nvalid = reinterpret_cast<int*>(base + w.nvalid);
  __nv_bfloat16* kt_rows = reinterpret_cast<__nv_bfloat16*>(base + w.kt_rows);
  __nv_bfloat16* vt_rows = reinterpret_cast<__nv_bfloat16*>(base + w.vt_rows);
  const int nqb = static_cast<int>((S + TILE - 1) / TILE);
  const int kc = static_cast<int>((kd + 63) / 64);

  // 1. head_dim scores on Q and selection
  cudaError_t e = launch_score(Q, 1, BH, S, D, D, S * D, ss, D, 0, base + w.score, stream);
  if (e != cudaSuccess) return e;
  e = launch_topk(ss, BH, D, D, kd, idx_d, kd, stream);
  if (e != cudaSuccess || (e = debug_step(stream, "head_dim scores and top-k")) != cudaSuccess) return e;
  // 2. compacted Q_I and K_I per q-head
  {
    const int64_t items = S * ((kd + 7) / 8);
    const dim3 grid(static_cast<unsigned>((items + 255) / 256), static_cast<unsigned>(BH));
    compact_heads_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(Q), static_cast<int>(Hq),
                                                   static_cast<int>(Hq), static_cast<int>(S), static_cast<int>(D),
                                                   idx_d, static_cast<int>(kd), qi, static_cast<int>(w.ldk));
    compact_heads_kernel<<<grid, 256, 0, stream>>>(static_cast<const __nv_bfloat16*>(K), static_cast<int>(Hq),
                                                   static_cast<int>(Hkv), static_cast<int>(S), static_cast<int>(D),
                                                   idx_d, static_cast<int>(kd), ki, static_cast<int>(w.ldk));
    e = cudaGetLastError();
    if (e != cudaSuccess || (e = debug_step(stream, "compaction of Q and K")) != cudaSuccess) return e;
  }
  CUtensorMap tm_q, tm_k, tm_kt, tm_vt;
  if (!encode_heads(&tm_q, qi, kd, S, BH, w.ldk) || !encode_heads(&tm_k, ki, kd, S, BH, w.ldk) ||
      !encode_heads(&tm_kt, kt_rows, kd, kt, BH, w.ldk) || !encode_heads(&tm_vt, vt_rows, D, kt, BH, D))
    return cudaErrorInvalidValue;
  AttnParams prm{};
  prm.S = static_cast<int>(S);
  prm.kc = kc;
  prm.D = static_cast<int>(D);
  prm.kt = static_cast<int>(kt);
  prm.nqb = nqb;
  prm.out_f32 = out_dtype == 0 ? 1 : 0;
  prm.scale_log2 = scale * kLog2e;
  // 3-4. passes A and B
  // at least 80 KB so no more than two of these CTAs (256 TMEM columns each)
  // share an SM: a third would wait in tcgen05.alloc
  const int qk_smem = std::max((1 + QK_STAGES) * kc * CHUNK_BYTES + static_cast<int>(sizeof(QkBars)) + 1024,
                               80 * 1024);
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set_smem(attn_qk_kernel<kLse>, qk_smem) || !set_smem(attn_qk_kernel<kColScore>, qk_smem)) {
      set_error("rmm_attention: cannot set %d bytes of shared memory for passes A/B", qk_smem);
      return cudaErrorInvalidValue;
    }
  }
  const dim3 grid_qk(static_cast<unsigned>(nqb), static_cast<unsigned>(BH));
  attn_qk_kernel<kLse><<<grid_qk, ATT_THREADS, qk_smem, stream>>>(tm_q, tm_k, lse, tsc, prm, err);
  if ((e = cudaGetLastError()) != cudaSuccess || (e = debug_step(stream, "pass A (lse)")) != cudaSuccess) return e;
  attn_qk_kernel<kColScore><<<grid_qk, ATT_THREADS, qk_smem, stream>>>(tm_q, tm_k, lse, tsc, prm, err);
  if ((e = cudaGetLastError()) != cudaSuccess || (e = debug_step(stream, "pass B (token scores)")) != cudaSuccess)
    return e;
  // 5. token selection and causal prefixes
  e = launch_topk(tsc, BH, S, S, kt, idx_t, kt, stream);
  if (e != cudaSuccess) return e;
  attn_prefix_kernel<<<static_cast<unsigned>((BH * nqb + 255) / 256), 256, 0, stream>>>(
      idx_t, static_cast<int>(BH), static_cast<int>(kt), static_cast<int>(S), nqb, nvalid);
  if ((e = cudaGetLastError()) != cudaSuccess || (e = debug_step(stream, "token top-k and prefixes")) != cudaSuccess)
    return e;
  // 6. kept rows of K_I and V
  {
    const dim3 grid(static_cast<unsigned>((kt + 7) / 8), static_cast<unsigned>(BH));
    gather_heads_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(ki), static_cast<int>(Hq),
                                                  static_cast<int>(Hq), static_cast<int>(S),
                                                  static_cast<int>(w.ldk / 8), idx_t, static_cast<int>(kt),
                                                  static_cast<int>(w.ldk / 8), reinterpret_cast<uint4*>(kt_rows),
                                                  static_cast<int>(w.ldk / 8));
    gather_heads_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(V), static_cast<int>(Hq),
                                                  static_cast<int>(Hkv), static_cast<int>(S),
                                                  static_cast<int>(D / 8), idx_t, static_cast<int>(kt),
                                                  static_cast<int>(D / 8), reinterpret_cast<uint4*>(vt_rows),
                                                  static_cast<int>(D / 8));
    e = cudaGetLastError();
    if (e != cudaSuccess || (e = debug_step(stream, "row gathers")) != cudaSuccess) return e;
  }
  // 7. pass C
  auto out_smem_for = [&](int stages) {
    return kc * CHUNK_BYTES + stages * (kc + static_cast<int>(D / 64)) * CHUNK_BYTES + 4 * CHUNK_BYTES +
           static_cast<int>(sizeof(OutBars)) + 1024;
  };
  int dev = 0, max_smem = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return e;
  prm.c_stages = out_smem_for(C_STAGES) <= max_smem ? C_STAGES : 1;
  const int out_smem = out_smem_for(prm.c_stages);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set_smem(attn_out_kernel, out_smem)) {
      set_error("rmm_attention: cannot set %d bytes of shared memory for pass C", out_smem);
      return cudaErrorInvalidValue;
    }
  }
  attn_out_kernel<<<grid_qk, ATT_THREADS, out_smem, stream>>>(tm_q, tm_kt, tm_vt, lse, idx_t, nvalid, O, prm, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  return debug_step(stream, "pass C (output)");
}

}  // namespace rmm
