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
// with S_ij = scale * Q_I[i] . K_I[j].  Passes A-C are tcgen05 kernels with
// a TMA warp, an MMA warp and two softmax groups of four warps that take
// alternate 128 x 128 logit tiles from tensor memory.  Pass C rounds
// P' = 2^15 P to fp16 (11 significant bits; the power-of-two scale keeps the
// small weights of long rows out of fp16's subnormal range), multiplies it
// with V_T gathered as fp16 (exact for bf16 values of magnitude <= 65504) and
// scales the fp32 accumulator back by 2^-15, an exact step.  Exponentials use the hardware ex2; the
// scale is folded into packed (f32x2) FMAs; only tiles on the causal
// diagonal or past the sequence end are masked.
#include <cuda.h>
#include <cuda_bf16.h>

#include <algorithm>
#include <cmath>
#include <cstdio>
#include <cstdlib>
#include <mutex>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int TILE = 128;                 // rows of every tile (queries or keys)
constexpr int CHUNK_BYTES = TILE * 128;   // one [128 x 64] bf16 tile, 128-byte rows: 16 KB
constexpr int ATT_THREADS = 320;          // warp 0 TMA, warp 1 MMA, warps 2-9 softmax (two groups of four)
constexpr int SOFTMAX_THREADS = 256;
// pass C on SM pairs: warp 0 TMA, warp 1 issues the logit MMAs, warps 2-9
// softmax (two groups of four), warp 10 issues the P V MMAs
constexpr int PAIR_THREADS = 352;
constexpr int PAIR_PV_WARP = 10;
constexpr float kLog2e = 1.4426950408889634f;
constexpr float kLn2 = 0.6931471805599453f;
// Pass C multiplies P by 2^kPScaleLog2 before rounding it to fp16: P <= 1, so
// P' <= 32768 stays below fp16's largest finite value (65504), and every
// weight above 2^-29 is an fp16 normal with 11 significant bits.
constexpr float kPScaleLog2 = 15.f;
constexpr float kPScaleInv = 1.f / 32768.f;

struct AttnParams {
  int S;            // tokens
  int kc;           // 64-column chunks of Q_I / K_I rows (ceil(k_d / 64))
  int D;            // head dim of V and O (64 or 128)
  int kt;           // kept tokens
  int nqb;          // query (= key) blocks of 128
  int out_f32;      // O written as fp32 (else bf16)
  int c_ks;         // pass C key ring depth (as shared memory allows)
  int c_vs;         // pass C value ring depth (as shared memory allows)
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

// The same row gather for V, widened from bf16 to fp16 for pass C's product:
// exact for magnitudes in [2^-14, 65504] (bf16 keeps 8 significant bits, fp16
// 11); smaller ones round to fp16 subnormals (absolute error <= 2^-25).
// Values beyond 65504 (or NaN) are saturated and flagged in the error word.
__global__ void __launch_bounds__(256) gather_v_f16_kernel(const uint4* __restrict__ src, int Hq, int Hsrc, int S,
                                                           int src_ld_vec, const int32_t* __restrict__ idx, int kt,
                                                           int row_vecs, uint4* __restrict__ dst, int dst_ld_vec,
                                                           unsigned* err) {
  const int bh = blockIdx.y, b = bh / Hq, h = bh % Hq, g = (h * Hsrc) / Hq;
  const int r = blockIdx.x * 8 + (threadIdx.x >> 5), lane = threadIdx.x & 31;
  if (r >= kt) return;
  const int j = __ldg(idx + static_cast<int64_t>(bh) * kt + r);
  const uint4* s = src + ((static_cast<int64_t>(b) * Hsrc + g) * S + j) * src_ld_vec;
  uint4* d = dst + (static_cast<int64_t>(bh) * kt + r) * dst_ld_vec;
  bool bad = false;
  for (int v = lane; v < row_vecs; v += 32) {
    const uint4 x = __ldg(s + v);
    const uint32_t w[4] = {x.x, x.y, x.z, x.w};
    uint32_t o[4];
#pragma unroll
    for (int e = 0; e < 4; ++e) {
      float lo = __uint_as_float(w[e] << 16), hi = __uint_as_float(w[e] & 0xFFFF0000u);
      bad |= !(fabsf(lo) <= 65504.f) || !(fabsf(hi) <= 65504.f);
      lo = fminf(fmaxf(lo, -65504.f), 65504.f);
      hi = fminf(fmaxf(hi, -65504.f), 65504.f);
      o[e] = pack_f16x2(lo, hi);
    }
    d[v] = make_uint4(o[0], o[1], o[2], o[3]);
  }
  if (bad) record_error(err, kDevErrFp16Range);
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
  float lsh[8][TILE];  // pass B, per softmax warp: -2 lse log2(e) of the current query block
  float cmb[2][TILE];  // the second softmax group's per-row state, handed to the first
};

// Pass A (kLse): CTA = one query block; the Q tile is loaded once and key
//   blocks 0..qb stream through the ring; a softmax thread owns query row r
//   and keeps a running max / sum in the log2 domain.
// Pass B (kColScore): CTA = one key block; the K tile is loaded once and query
//   blocks kb..nqb-1 stream through; the tile in tensor memory is S^T (lane =
//   key), so a softmax thread owns key r and sums exp(2 (S_ij - lse_i)) over
//   its queries with no cross-thread reduction.
// Two softmax groups of four warps take alternate stream blocks (group g
// the blocks g, g+2, ..., in tensor-memory buffer g); at the end group 1
// hands its per-row state to group 0 through shared memory.  Only blocks on
// the causal diagonal or past the sequence end are masked.
template <int MODE>
__global__ void __launch_bounds__(ATT_THREADS, 2)
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
  // grid (heads, blocks): the hardware hands out x fastest, so every head's
  // heaviest block goes out before any lighter one (no heavy tail)
  const int bh = blockIdx.x;
  // pass A: heaviest query blocks first; pass B: key block kb (kb = 0 is the heaviest)
  const int fixed_blk = MODE == kLse ? p.nqb - 1 - static_cast<int>(blockIdx.y) : static_cast<int>(blockIdx.y);
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
    const int g = (warp - 2) >> 2;                  // softmax group
    const int qtr = warp & 3;                       // tensor-memory lane quarter of this warp
    const int r = qtr * 32 + lane;                  // TMEM lane = tile row
    const int own = fixed_blk * TILE + r;           // this thread's query (A) or key (B)
    const uint32_t lane_off = static_cast<uint32_t>(qtr * 32) << 16;
    const float sl = p.scale_log2;
    float m = -INFINITY, l = 0.f;                   // pass A state (log2 domain)
    float total = 0.f;                              // pass B state
    float* nl = bars->lsh[warp - 2];
    for (int it = g; it < n_stream; it += 2) {
      const uint32_t b = it & 1, sph = (it >> 1) & 1;
      const int sbase = (first_stream + it) * TILE;
      const bool masked = first_stream + it == fixed_blk || sbase + TILE > p.S;
      if (MODE == kColScore) {
        // each warp keeps its own copy of the block's 128 lse values, so only
        // warp-level synchronisation is needed
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int q = sbase + u * 32 + lane;
          nl[u * 32 + lane] = q < p.S ? -2.f * kLog2e * lse[static_cast<int64_t>(bh) * p.S + q] : 0.f;
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(sfull(b), sph, abort_flag, err, 15)) break;
      tc_fence_after();
      float blk = 0.f;
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        __syncwarp();  // the tensor-memory load is warp-synchronous: reconverge first
        tmem_ld32(tmem_base + b * TILE + cc * 32 + lane_off, v);
        tmem_wait_ld();
        if (masked) {
          // pass A keeps keys j <= own, pass B queries i >= own; both j, i < S
          const int c0 = sbase + cc * 32;
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int j = c0 + e;
            const bool keep = (MODE == kLse ? j <= own : j >= own) && j < p.S;
            if (!keep) v[e] = __float_as_uint(-INFINITY);
          }
        }
        uint64_t acc0 = f2_pack(0.f, 0.f), acc1 = acc0;
        if (MODE == kLse) {
          const float mx = max_of32(v) * sl;
          if (mx > -INFINITY) {  // else nothing is kept in this chunk (lane-divergent; ALU work only)
            if (mx > m) {
              l *= fast_exp2(m - mx);
              m = mx;
            }
            const uint64_t slp = f2_pack(sl, sl), nm = f2_pack(-m, -m);
#pragma unroll
            for (int e = 0; e < 16; ++e) {
              float x0, x1;
              f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), slp, nm), x0, x1);
              const uint64_t ex = f2_pack(fast_exp2(x0), fast_exp2(x1));
              if (e & 1) {
                acc1 = f2_add(acc1, ex);
              } else {
                acc0 = f2_add(acc0, ex);
              }
            }
          }
        } else {
          const uint64_t sl2 = f2_pack(2.f * sl, 2.f * sl);
          const float2* nlc = reinterpret_cast<const float2*>(nl + cc * 32);
#pragma unroll
          for (int e = 0; e < 16; ++e) {
            const float2 q = nlc[e];
            float x0, x1;
            f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), sl2,
                             f2_pack(q.x, q.y)),
                      x0, x1);
            const uint64_t ex = f2_pack(fast_exp2(x0), fast_exp2(x1));
            if (e & 1) {
              acc1 = f2_add(acc1, ex);
            } else {
              acc0 = f2_add(acc0, ex);
            }
          }
        }
        float s0, s1;
        f2_unpack(f2_add(acc0, acc1), s0, s1);
        if (MODE == kLse) {
          l += s0 + s1;
        } else {
          blk += s0 + s1;
        }
      }
      total += blk;
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(sempty(b));
    }
    // group 1 hands its state to group 0; every softmax warp reaches this
    // barrier exactly once (also after an aborted wait)
    if (g == 1) {
      bars->cmb[0][r] = MODE == kLse ? m : total;
      bars->cmb[1][r] = l;
    }
    named_barrier(1, SOFTMAX_THREADS);
    if (g == 0 && own < p.S) {
      if (MODE == kLse) {
        const float m1 = bars->cmb[0][r], l1 = bars->cmb[1][r];
        const float mm = fmaxf(m, m1);
        const float ll = (m > -INFINITY ? l * fast_exp2(m - mm) : 0.f) + (m1 > -INFINITY ? l1 * fast_exp2(m1 - mm) : 0.f);
        lse[static_cast<int64_t>(bh) * p.S + own] = (mm + log2f(ll)) * kLn2;
      } else {
        tsc[static_cast<int64_t>(bh) * p.S + own] = total + bars->cmb[0][r];
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

constexpr int C_MAX_KS = 4;  // key ring depth of pass C (at most)
constexpr int C_MAX_VS = 4;  // value ring depth (at most)
constexpr int C_SBUF = 3;    // logit / P buffers in tensor memory

struct OutBars {
  uint64_t kfull[C_MAX_KS], kempty[C_MAX_KS];
  uint64_t vfull[C_MAX_VS], vempty[C_MAX_VS];
  uint64_t qfull;
  uint64_t sfull[C_SBUF], pfull[C_SBUF];
  uint64_t ofull;
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
  int pos[8][TILE];  // per softmax warp: token positions of the current kept block
};

// Waits, with a bounded wall time, for the last min(issued, n) loads of a
// ring of n stages to land (load t used stage t % n, phase (t / n) & 1).
__device__ __forceinline__ void drain_ring(const uint64_t* full, int issued, int n) {
  for (int t = issued - 1; t >= 0 && t >= issued - n; --t) wait_drain(smem_u32(&full[t % n]), (t / n) & 1);
}

// CTA = one query block.  Kept tokens are processed 128 at a time (only the
// blocks that hold a kept position <= the block's last query): S = Q_I K_T^T
// into tensor memory; the softmax warps turn row i into P'_ir = 2^15 exp(S_ir -
// lse_i) for kept positions <= i (else 0) and write it as fp16 back into the
// same tensor-memory buffer (two per column, over the logits already read);
// the MMA lane accumulates O += P' V_T with P' read from tensor memory and
// V_T (fp16, MN-major) from shared memory; the epilogue scales O by 2^-15.
//   Tensor memory (512 columns): three logit / P buffers of 128 columns and O.
//   - kept block j uses buffer j % 3; the MMA lane issues PV(j) as soon as
//     softmax(j) is done and then S(j+3) into the same buffer: tcgen05 MMAs
//     of one thread run in issue order, so PV(j) has read P(j) before S(j+3)
//     writes there, and each softmax group finds its next logits ready;
//   - two softmax groups of four warps take alternate kept blocks;
//   - one producer lane streams keys, another values, each into its own ring;
//   - the MMA role runs on one lane (it has no warp-synchronous instruction).
// Only kept blocks that reach past the first query of this block are masked;
// the two groups split the output columns in the epilogue.
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
  const int ks = p.c_ks, vs = p.c_vs;
  const int q_bytes = p.kc * CHUNK_BYTES;
  const int k_bytes = p.kc * CHUNK_BYTES;
  const int v_bytes = dc * CHUNK_BYTES;
  const uint32_t q_tile = base;
  auto kst = [&](int s) { return base + q_bytes + s * k_bytes; };
  auto vst = [&](int s) { return base + q_bytes + ks * k_bytes + s * v_bytes; };
  OutBars* bars = reinterpret_cast<OutBars*>(smem + q_bytes + ks * k_bytes + vs * v_bytes);
  volatile int* abort_flag = &bars->abort_flag;
  auto kfull = [&](int s) { return smem_u32(&bars->kfull[s]); };
  auto kempty = [&](int s) { return smem_u32(&bars->kempty[s]); };
  auto vfull = [&](int s) { return smem_u32(&bars->vfull[s]); };
  auto vempty = [&](int s) { return smem_u32(&bars->vempty[s]); };
  auto sfull = [&](int b) { return smem_u32(&bars->sfull[b]); };
  auto pfull = [&](int b) { return smem_u32(&bars->pfull[b]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int bh = blockIdx.x;                                 // grid (heads, blocks)
  const int qb = p.nqb - 1 - static_cast<int>(blockIdx.y);  // heaviest blocks first
  const int nv = __ldg(nvalid + static_cast<int64_t>(bh) * p.nqb + qb);
  const int nrb = (nv + TILE - 1) / TILE;
  // kept positions before this block's first query: kept blocks made only of
  // those need no causal mask
  const int nbefore = qb > 0 ? __ldg(nvalid + static_cast<int64_t>(bh) * p.nqb + qb - 1) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ks; ++s) {
      mbar_init(kfull(s), 1);
      mbar_init(kempty(s), 1);
    }
    for (int s = 0; s < vs; ++s) {
      mbar_init(vfull(s), 1);
      mbar_init(vempty(s), 1);
    }
    mbar_init(smem_u32(&bars->qfull), 1);
    for (int b = 0; b < C_SBUF; ++b) {
      mbar_init(sfull(b), 1);  // commit of S
      mbar_init(pfull(b), 4);  // one arrival per warp of the softmax group
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
  const uint32_t o_tmem = tmem_base + C_SBUF * TILE;
  auto buf_tmem = [&](int b) { return tmem_base + b * TILE; };

  if (warp == 0) {
    // lane 0: Q, then the key ring; lane 1: the value ring
    if (lane == 0 && nrb > 0) {
      mbar_arrive_expect_tx(smem_u32(&bars->qfull), q_bytes);
      for (int c = 0; c < p.kc; ++c)
        tma_load_3d(q_tile + c * CHUNK_BYTES, &tm_q, smem_u32(&bars->qfull), c * 64, qb * TILE, bh);
      int n = 0;
      for (int t = 0; t < nrb; ++t) {
        const int st = t % ks;
        if (!mbar_wait(kempty(st), ((t / ks) & 1) ^ 1u, abort_flag, err, 21)) break;
        mbar_arrive_expect_tx(kfull(st), k_bytes);
        for (int c = 0; c < p.kc; ++c) tma_load_3d(kst(st) + c * CHUNK_BYTES, &tm_kt, kfull(st), c * 64, t * TILE, bh);
        ++n;
      }
      wait_drain(smem_u32(&bars->qfull), 0);
      drain_ring(bars->kfull, n, ks);
    } else if (lane == 1 && nrb > 0) {
      int n = 0;
      for (int t = 0; t < nrb; ++t) {
        const int st = t % vs;
        if (!mbar_wait(vempty(st), ((t / vs) & 1) ^ 1u, abort_flag, err, 29)) break;
        mbar_arrive_expect_tx(vfull(st), v_bytes);
        for (int c = 0; c < dc; ++c) tma_load_3d(vst(st) + c * CHUNK_BYTES, &tm_vt, vfull(st), c * 64, t * TILE, bh);
        ++n;
      }
      drain_ring(bars->vfull, n, vs);
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(TILE, TILE, false, false);
      const uint32_t idesc_o = idesc_f16_f32(TILE, p.D, false, true);
      bool ok = nrb == 0 || mbar_wait(smem_u32(&bars->qfull), 0, abort_flag, err, 22);
      // S(t) = Q_I K_T(t)^T into buffer t % 3
      auto issue_s = [&](int t) -> bool {
        const int st = t % ks;
        if (!mbar_wait(kfull(st), (t / ks) & 1, abort_flag, err, 24)) return false;
        tc_fence_after();
        for (int c = 0; c < p.kc; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(q_tile + c * CHUNK_BYTES + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kst(st) + c * CHUNK_BYTES + kk * 32, 16, 1024);
            mma_f16_ss(buf_tmem(t % C_SBUF), ad, bd, idesc_s, (c | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit(kempty(st));
        mma_commit(sfull(t % C_SBUF));
        return true;
      };
      // O += P(t) V_T(t), P from the first 64 columns of buffer t % 3
      auto issue_pv = [&](int t) -> bool {
        const int st = t % vs;
        if (!mbar_wait(vfull(st), (t / vs) & 1, abort_flag, err, 30)) return false;
        tc_fence_after();
        const uint32_t pt = buf_tmem(t % C_SBUF);
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(vst(st) + kk * 16 * 128, CHUNK_BYTES, 1024);
          mma_f16_ts(o_tmem, pt + kk * 8, bd, idesc_o, (t | kk) != 0 ? 1u : 0u);
        }
        mma_commit(vempty(st));
        return true;
      };
      for (int t = 0; ok && t < C_SBUF && t < nrb; ++t) ok = issue_s(t);
      for (int j = 0; ok && j < nrb; ++j) {
        ok = mbar_wait(pfull(j % C_SBUF), (j / C_SBUF) & 1, abort_flag, err, 23);
        if (ok) tc_fence_after();
        ok = ok && issue_pv(j);
        if (ok && j + C_SBUF < nrb) ok = issue_s(j + C_SBUF);
      }
      if (ok && nrb > 0) mma_commit(smem_u32(&bars->ofull));
      mma_commit(smem_u32(&bars->drain));
      wait_drain(smem_u32(&bars->drain), 0);
    }
    __syncwarp();
  } else {
    const int g = (warp - 2) >> 2;  // softmax group
    const int qtr = warp & 3;       // tensor-memory lane quarter of this warp
    const int r = qtr * 32 + lane;
    const int i = qb * TILE + r;
    const uint32_t lane_off = static_cast<uint32_t>(qtr * 32) << 16;
    // exponent of P' = 2^15 P
    const float L2 = i < p.S ? lse[static_cast<int64_t>(bh) * p.S + i] * kLog2e - kPScaleLog2 : 0.f;
    const int32_t* pos_bh = pos + static_cast<int64_t>(bh) * p.kt;
    const uint64_t slp = f2_pack(p.scale_log2, p.scale_log2), nl2 = f2_pack(-L2, -L2);
    int* psh = bars->pos[warp - 2];
    bool ok = true;
    for (int rb = g; ok && rb < nrb; rb += 2) {
      const int b = rb % C_SBUF;
      const uint32_t sph = (rb / C_SBUF) & 1;
      const bool masked = rb * TILE + TILE > nbefore;
      if (masked) {
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int kr = rb * TILE + u * 32 + lane;
          psh[u * 32 + lane] = kr < p.kt ? __ldg(pos_bh + kr) : 0x7FFFFFFF;
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(sfull(b), sph, abort_flag, err, 26)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // P goes over the logits of the same buffer: chunk cc's P (16 columns
      // from 16 cc) only covers logits already read
      const uint32_t s_addr = buf_tmem(b) + lane_off;
      const uint32_t p_addr = s_addr;
      // P for the 32 kept columns of chunk cc from the scores in v, packed two
      // per tensor-memory column
      auto exps = [&](int cc, const uint32_t (&v)[32], uint32_t (&w)[16]) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), slp, nl2), x0, x1);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          if (masked) {
            if (psh[cc * 32 + 2 * e] > i) p0 = 0.f;
            if (psh[cc * 32 + 2 * e + 1] > i) p1 = 0.f;
          }
          w[e] = pack_f16x2(p0, p1);
        }
      };
      uint32_t va[32], vb[32], w[16];
      __syncwarp();  // tensor-memory accesses are warp-synchronous: reconverge first
      tmem_ld32(s_addr, va);
      tmem_wait_ld_into(va);
      tmem_ld32(s_addr + 32, vb);
      exps(0, va, w);
      tmem_st16(p_addr, w);
      tmem_wait_ld_into(vb);
      __syncwarp();
      tmem_ld32(s_addr + 64, va);
      exps(1, vb, w);
      tmem_st16(p_addr + 16, w);
      tmem_wait_ld_into(va);
      __syncwarp();
      tmem_ld32(s_addr + 96, vb);
      exps(2, va, w);
      tmem_st16(p_addr + 32, w);
      tmem_wait_ld_into(vb);
      exps(3, vb, w);
      tmem_st16(p_addr + 48, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(pfull(b));
    }
    // epilogue: O row i, columns [g D/2, (g+1) D/2).  Every lane of the warp
    // takes part in the tensor-memory loads (warp-synchronous); only rows
    // i < S are stored.
    const bool have = ok && nrb > 0 && mbar_wait_warp(smem_u32(&bars->ofull), 0, abort_flag, err, 28);
    if (have) tc_fence_after();
    const int ncc = p.D / 64;  // 32-column chunks per group
    for (int cc = g * ncc; cc < (g + 1) * ncc; ++cc) {
      uint32_t v[32];
      if (have) {
        __syncwarp();
        tmem_ld32(o_tmem + cc * 32 + lane_off, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (i >= p.S) continue;
      const int64_t off = (static_cast<int64_t>(bh) * p.S + i) * p.D + cc * 32;
      float o[32];  // undo the 2^15 of P' (exact)
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(v[e]) * kPScaleInv;
      if (p.out_f32) {
        float4* y = reinterpret_cast<float4*>(static_cast<float*>(O) + off);
#pragma unroll
        for (int q = 0; q < 8; ++q) y[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      } else {
        uint4* y = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(O) + off);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          y[q] = make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                            pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
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

// ------------------------------------------------------------------ pass C on SM pairs
//
// The same product for two adjacent query blocks on a pair of SMs (a 2-CTA
// cluster) with tcgen05.mma.cta_group::2 (M = 256): measured on B200, an
// M256 N128 K16 pair step takes ~68 cycles against ~114 for M128 N128 on
// one SM, and each SM loads only half of every key block and half of every
// value block (no multicast: each CTA loads its own halves).
//   - the leader (rank 0) takes the heavier query block; both CTAs walk the
//     leader's kept blocks (the lighter block's extra ones are fully masked);
//   - S = Q_I K_T^T: each CTA's A is its own 128 query rows, its B the 64
//     keys [j*128 + rank*64, +64) of kept block j; each CTA's tensor memory
//     gets its 128 rows x 128 keys;
//   - P' (fp16) goes back into each CTA's tensor memory over the logits it
//     came from (two per column); O += P V_T takes A = P' from both CTAs'
//     tensor memory and B = each CTA's 64 of V's 128 columns, each CTA's
//     tensor memory gets its rows of O.  (With P' in shared memory each
//     CTA moved ~128 KB per kept block through shared memory, and back-to-back
//     pair MMAs were accepted every ~147 cycles against ~68 alone: the P
//     write and the P operand read were half of that traffic);
//   - every load signals the leader's barriers; the leader's MMA lane waits
//     on them, and its commits reach both CTAs (multicast); the softmax
//     groups of both CTAs arrive on the leader's P barrier;
//   - two issuing lanes in the leader: warp 1 issues the logit MMAs, warp 10
//     the P V MMAs (one issuing thread spent ~120-150 cycles per M256 N128 K16
//     pair MMA, about twice the tensor pipe's time for it, so a single issuer
//     left the pipe idle two thirds of the time);
//   - three logit / P' buffers: once both CTAs have written P'(j) the P V
//     issuer issues PV(j); once PV(j) is done the logit issuer puts S(j+3)
//     into buffer j % 3;
//   - key stage j % 3 is free when S(j) is done and value stage j % 3 when
//     PV(j) is done, so the producers wait on the logit and P V commits
//     (one commit each per kept block).
// Every wait is bounded; every path reaches the final cluster barrier.
constexpr int CP_KS = C_SBUF;  // key ring depth = logit buffers (a key stage is freed with its logits)
constexpr int CP_VS = C_SBUF;  // value ring depth = logit/P buffers (a value stage is freed with its P V)
constexpr int CP_HALF_ROWS = TILE / 2;                 // keys of a kept block per CTA
constexpr int CP_KCHUNK_BYTES = CP_HALF_ROWS * 128;    // [64 x 64] bf16, 128-byte rows: 8 KB
// one CTA per SM: each holds all 512 tensor-memory columns, so a second one
// would wait in tcgen05.alloc while its cluster partner holds another SM's
constexpr int CP_MIN_SMEM = 116 * 1024;

struct PairOutBars {
  uint64_t kfull[CP_KS];
  uint64_t vfull[CP_VS];
  uint64_t qfull;
  uint64_t sfull[C_SBUF];   // multicast commit: S(t) is in buffer t % 3
  uint64_t pfull[C_SBUF];   // leader: both CTAs' softmax groups wrote P'(t) over buffer t % 3
  uint64_t pvdone[C_SBUF];  // multicast commit: PV(t) is done, so buffer t % 3 and value stage t % 3 are free
  uint64_t ofull;
  uint64_t drain, drain_pv;
  uint32_t tmem_slot;
  int abort_flag;
  int pos[8][TILE];
};

__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(PAIR_THREADS, 1)
    attn_out_pair_kernel(const __grid_constant__ CUtensorMap tm_q, const __grid_constant__ CUtensorMap tm_kh,
                         const __grid_constant__ CUtensorMap tm_vt, const float* __restrict__ lse,
                         const int32_t* __restrict__ pos, const int* __restrict__ nvalid, void* __restrict__ O,
                         AttnParams p, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t base = smem_u32(smem);
  constexpr int ks = CP_KS, vs = CP_VS;
  const int q_bytes = p.kc * CHUNK_BYTES;
  const int k_bytes = p.kc * CP_KCHUNK_BYTES;  // this CTA's half of a key block
  const int v_bytes = CHUNK_BYTES;             // this CTA's 64 columns of a value block
  const uint32_t q_tile = base;
  auto kst = [&](int s) { return base + q_bytes + s * k_bytes; };
  auto vst = [&](int s) { return base + q_bytes + ks * k_bytes + s * v_bytes; };
  PairOutBars* bars = reinterpret_cast<PairOutBars*>(smem + q_bytes + ks * k_bytes + vs * v_bytes);
  volatile int* abort_flag = &bars->abort_flag;
  auto kfull = [&](int s) { return smem_u32(&bars->kfull[s]); };
  auto vfull = [&](int s) { return smem_u32(&bars->vfull[s]); };
  auto sfull = [&](int b) { return smem_u32(&bars->sfull[b]); };
  auto pfull = [&](int b) { return smem_u32(&bars->pfull[b]); };
  auto pvdone = [&](int b) { return smem_u32(&bars->pvdone[b]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int bh = static_cast<int>(blockIdx.x) >> 1;  // grid (2 x heads, pairs): heaviest pairs of all heads first
  const int pair = static_cast<int>(blockIdx.y);
  const int qb0 = p.nqb - 1 - 2 * pair;                   // the leader's (heavier) block
  const int qb = qb0 - static_cast<int>(rank);            // this CTA's block (-1: none)
  const int* nv_bh = nvalid + static_cast<int64_t>(bh) * p.nqb;
  const int nrb = (__ldg(nv_bh + qb0) + TILE - 1) / TILE;  // kept blocks both CTAs walk
  const int nbefore = qb > 0 ? __ldg(nv_bh + qb - 1) : 0;

  if (threadIdx.x == 0) {
    for (int s = 0; s < ks; ++s) mbar_init(kfull(s), 1);  // leader: its producer's arrive + both CTAs' bytes
    for (int s = 0; s < vs; ++s) mbar_init(vfull(s), 1);
    mbar_init(smem_u32(&bars->qfull), 1);
    for (int b = 0; b < C_SBUF; ++b) {
      mbar_init(sfull(b), 1);   // multicast commit
      mbar_init(pfull(b), 8);   // leader: four warps of a softmax group in each CTA
      mbar_init(pvdone(b), 1);  // multicast commit
    }
    mbar_init(smem_u32(&bars->ofull), 1);
    mbar_init(smem_u32(&bars->drain), 1);
    mbar_init(smem_u32(&bars->drain_pv), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&bars->tmem_slot), 512);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_slot;
  const uint32_t o_tmem = tmem_base + C_SBUF * TILE;
  auto buf_tmem = [&](int b) { return tmem_base + b * TILE; };

  if (warp == 0) {
    // lane 0: Q, then this CTA's key halves; lane 1: its value halves.  The
    // leader's lanes register both CTAs' bytes on its barriers.
    if (lane == 0 && nrb > 0) {
      const uint32_t qf = mapa_shared(smem_u32(&bars->qfull), 0);
      if (leader) mbar_arrive_expect_tx(smem_u32(&bars->qfull), 2 * q_bytes);
      for (int c = 0; c < p.kc; ++c) tma_load_3d_pair(q_tile + c * CHUNK_BYTES, &tm_q, qf, c * 64, qb * TILE, bh);
      int n = 0;
      for (int t = 0; t < nrb; ++t) {
        const int st = t % ks;  // freed by S(t - 3): the logits of buffer st
        if (!mbar_wait(sfull(st), ((t / ks) & 1) ^ 1u, abort_flag, err, 31)) break;
        const uint32_t kf = mapa_shared(kfull(st), 0);
        if (leader) mbar_arrive_expect_tx(kfull(st), 2 * k_bytes);
        for (int c = 0; c < p.kc; ++c)
          tma_load_3d_pair(kst(st) + c * CP_KCHUNK_BYTES, &tm_kh, kf, c * 64,
                           t * TILE + static_cast<int>(rank) * CP_HALF_ROWS, bh);
        ++n;
      }
      if (leader) {
        wait_drain(smem_u32(&bars->qfull), 0);
        drain_ring(bars->kfull, n, ks);
      }
    } else if (lane == 1 && nrb > 0) {
      int n = 0;
      for (int t = 0; t < nrb; ++t) {
        const int st = t % vs;  // freed by PV(t - 3)
        if (!mbar_wait(pvdone(st), ((t / vs) & 1) ^ 1u, abort_flag, err, 32)) break;
        const uint32_t vf = mapa_shared(vfull(st), 0);
        if (leader) mbar_arrive_expect_tx(vfull(st), 2 * v_bytes);
        tma_load_3d_pair(vst(st), &tm_vt, vf, static_cast<int>(rank) * 64, t * TILE, bh);
        ++n;
      }
      if (leader) drain_ring(bars->vfull, n, vs);
    }
    __syncwarp();
  } else if (warp == 1) {
    // logit MMAs: S(t) into buffer t % 3 once PV(t - 3) has read P'(t - 3) there
    if (leader && lane == 0) {
      constexpr uint32_t idesc_s = idesc_bf16_f32(2 * TILE, TILE, false, false);
      bool ok = nrb == 0 || mbar_wait(smem_u32(&bars->qfull), 0, abort_flag, err, 33);
      for (int t = 0; ok && t < nrb; ++t) {
        const int st = t % ks, b = t % C_SBUF;
        if (t >= C_SBUF) ok = mbar_wait(pvdone(b), ((t - C_SBUF) / C_SBUF) & 1, abort_flag, err, 40);
        ok = ok && mbar_wait(kfull(st), (t / ks) & 1, abort_flag, err, 34);
        if (!ok) break;
        tc_fence_after();
        for (int c = 0; c < p.kc; ++c) {
#pragma unroll
          for (int kk = 0; kk < 4; ++kk) {
            const uint64_t ad = sdesc_sw128(q_tile + c * CHUNK_BYTES + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(kst(st) + c * CP_KCHUNK_BYTES + kk * 32, 16, 1024);
            mma_f16_ss_pair(buf_tmem(b), ad, bd, idesc_s, (c | kk) != 0 ? 1u : 0u);
          }
        }
        mma_commit_pair_multicast(sfull(b), 0x3);
      }
      mma_commit_pair_multicast(smem_u32(&bars->drain), 0x1);
      wait_drain(smem_u32(&bars->drain), 0);
    }
    __syncwarp();
  } else if (warp == PAIR_PV_WARP) {
    // P V MMAs: PV(j) with P'(j) read from both CTAs' tensor memory (buffer
    // j % 3) once both have written it and V(j) has landed
    if (leader && lane == 0) {
      const uint32_t idesc_o = idesc_f16_f32(2 * TILE, p.D, false, true);
      bool ok = true;
      for (int j = 0; ok && j < nrb; ++j) {
        const int b = j % C_SBUF, st = j % vs;
        ok = mbar_wait(pfull(b), (j / C_SBUF) & 1, abort_flag, err, 36) &&
             mbar_wait(vfull(st), (j / vs) & 1, abort_flag, err, 35);
        if (!ok) break;
        tc_fence_after();
#pragma unroll
        for (int kk = 0; kk < TILE / 16; ++kk) {
          const uint64_t bd = sdesc_sw128(vst(st) + kk * 16 * 128, CHUNK_BYTES, 1024);
          mma_f16_ts_pair(o_tmem, buf_tmem(b) + kk * 8, bd, idesc_o, (j | kk) != 0 ? 1u : 0u);
        }
        mma_commit_pair_multicast(pvdone(b), 0x3);
      }
      if (ok && nrb > 0) mma_commit_pair_multicast(smem_u32(&bars->ofull), 0x3);
      mma_commit_pair_multicast(smem_u32(&bars->drain_pv), 0x1);
      wait_drain(smem_u32(&bars->drain_pv), 0);
    }
    __syncwarp();
  } else {
    const int g = (warp - 2) >> 2;  // softmax group
    const int qtr = warp & 3;       // tensor-memory lane quarter of this warp
    const int r = qtr * 32 + lane;
    const int i = qb * TILE + r;    // this thread's query (negative for the spare CTA of an odd count)
    const bool row_ok = i >= 0 && i < p.S;
    const uint32_t lane_off = static_cast<uint32_t>(qtr * 32) << 16;
    // exponent of P' = 2^15 P
    const float L2 = row_ok ? lse[static_cast<int64_t>(bh) * p.S + i] * kLog2e - kPScaleLog2 : 0.f;
    const int32_t* pos_bh = pos + static_cast<int64_t>(bh) * p.kt;
    const uint64_t slp = f2_pack(p.scale_log2, p.scale_log2), nl2 = f2_pack(-L2, -L2);
    int* psh = bars->pos[warp - 2];
    bool ok = true;
    for (int rb = g; ok && rb < nrb; rb += 2) {
      const int b = rb % C_SBUF;
      const uint32_t sph = (rb / C_SBUF) & 1;
      const bool masked = rb * TILE + TILE > nbefore;
      if (masked) {
        __syncwarp();
#pragma unroll
        for (int u = 0; u < 4; ++u) {
          const int kr = rb * TILE + u * 32 + lane;
          psh[u * 32 + lane] = kr < p.kt ? __ldg(pos_bh + kr) : 0x7FFFFFFF;
        }
        __syncwarp();
      }
      if (!mbar_wait_warp(sfull(b), sph, abort_flag, err, 37)) {
        ok = false;
        break;
      }
      tc_fence_after();
      // P' goes over the logits of the same buffer, two fp16 per column: chunk
      // cc's P' (16 columns from 16 cc) only covers logits already loaded
      const uint32_t s_addr = buf_tmem(b) + lane_off;
      const uint32_t p_addr = s_addr;
      auto exps = [&](int cc, const uint32_t (&v)[32], uint32_t (&w)[16]) {
#pragma unroll
        for (int e = 0; e < 16; ++e) {
          float x0, x1;
          f2_unpack(f2_fma(f2_pack(__uint_as_float(v[2 * e]), __uint_as_float(v[2 * e + 1])), slp, nl2), x0, x1);
          float p0 = fast_exp2(x0), p1 = fast_exp2(x1);
          if (masked) {
            if (psh[cc * 32 + 2 * e] > i) p0 = 0.f;
            if (psh[cc * 32 + 2 * e + 1] > i) p1 = 0.f;
          }
          w[e] = pack_f16x2(p0, p1);
        }
      };
      uint32_t va[32], vb[32], w[16];
      __syncwarp();  // tensor-memory accesses are warp-synchronous: reconverge first
      tmem_ld32(s_addr, va);
      tmem_wait_ld_into(va);
      tmem_ld32(s_addr + 32, vb);
      exps(0, va, w);
      tmem_st16(p_addr, w);
      tmem_wait_ld_into(vb);
      __syncwarp();
      tmem_ld32(s_addr + 64, va);
      exps(1, vb, w);
      tmem_st16(p_addr + 16, w);
      tmem_wait_ld_into(va);
      __syncwarp();
      tmem_ld32(s_addr + 96, vb);
      exps(2, va, w);
      tmem_st16(p_addr + 32, w);
      tmem_wait_ld_into(vb);
      exps(3, vb, w);
      tmem_st16(p_addr + 48, w);
      tmem_wait_st();
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(pfull(b), 0));
    }
    // epilogue: O row i, columns [g D/2, (g+1) D/2)
    const bool have = ok && nrb > 0 && mbar_wait_warp(smem_u32(&bars->ofull), 0, abort_flag, err, 39);
    if (have) tc_fence_after();
    const int ncc = p.D / 64;
    for (int cc = g * ncc; cc < (g + 1) * ncc; ++cc) {
      uint32_t v[32];
      if (have) {
        __syncwarp();
        tmem_ld32(o_tmem + cc * 32 + lane_off, v);
        tmem_wait_ld();
      } else {
#pragma unroll
        for (int e = 0; e < 32; ++e) v[e] = 0u;
      }
      if (!row_ok) continue;
      const int64_t off = (static_cast<int64_t>(bh) * p.S + i) * p.D + cc * 32;
      float o[32];  // undo the 2^15 of P' (exact)
#pragma unroll
      for (int e = 0; e < 32; ++e) o[e] = __uint_as_float(v[e]) * kPScaleInv;
      if (p.out_f32) {
        float4* y = reinterpret_cast<float4*>(static_cast<float*>(O) + off);
#pragma unroll
        for (int q = 0; q < 8; ++q) y[q] = make_float4(o[4 * q], o[4 * q + 1], o[4 * q + 2], o[4 * q + 3]);
      } else {
        uint4* y = reinterpret_cast<uint4*>(static_cast<__nv_bfloat16*>(O) + off);
#pragma unroll
        for (int q = 0; q < 4; ++q)
          y[q] = make_uint4(pack_bf16x2(o[8 * q], o[8 * q + 1]), pack_bf16x2(o[8 * q + 2], o[8 * q + 3]),
                            pack_bf16x2(o[8 * q + 4], o[8 * q + 5]), pack_bf16x2(o[8 * q + 6], o[8 * q + 7]));
      }
    }
    tc_fence_before();
  }

  tc_fence_before();
  cluster_sync();  // all MMAs, copies and remote arrivals of the pair are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, 512);
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

// 3-D map of 16-bit elements (bf16, or fp16 for V_T) over
// [heads][rows][pitch] with logical row length `cols`; boxes of 64 columns x
// box_rows rows x 1 head, 128-byte swizzle.
bool encode_heads(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int64_t heads, int64_t pitch,
                  int box_rows = TILE, CUtensorMapDataType dt = CU_TENSOR_MAP_DATA_TYPE_BFLOAT16) {
  EncodeTiledFn encode = encode_fn();
  if (!encode) {
    set_error("rmm_attention: cuTensorMapEncodeTiled entry point unavailable");
    return false;
  }
  const cuuint64_t gdim[3] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows),
                              static_cast<cuuint64_t>(heads)};
  const cuuint64_t gstride[2] = {static_cast<cuuint64_t>(pitch) * 2, static_cast<cuuint64_t>(pitch * rows) * 2};
  const cuuint32_t box[3] = {64, static_cast<cuuint32_t>(box_rows), 1};
  const cuuint32_t estride[3] = {1, 1, 1};
  const CUresult r = encode(map, dt, 3, const_cast<void*>(ptr), gdim, gstride, box,
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
  __half* vt_rows = reinterpret_cast<__half*>(base + w.vt_rows);  // fp16 rows of V
  const int nqb = static_cast<int>((S + TILE - 1) / TILE);
  const int kc = static_cast<int>((kd + 63) / 64);

  // 1. head_dim scores on Q and selection
  cudaError_t e = launch_score(Q, 1, BH, S, D, D, S * D, ss, D, 0, base + w.score, stream);
  if (e != cudaSuccess) return e;
  e = launch_topk(ss, BH, D, D, kd, idx_d, kd, stream);
  if (e != cudaSuccess) return e;
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
    if (e != cudaSuccess) return e;
  }
  CUtensorMap tm_q, tm_k, tm_kt, tm_vt;
  if (!encode_heads(&tm_q, qi, kd, S, BH, w.ldk) || !encode_heads(&tm_k, ki, kd, S, BH, w.ldk) ||
      !encode_heads(&tm_kt, kt_rows, kd, kt, BH, w.ldk) ||
      !encode_heads(&tm_vt, vt_rows, D, kt, BH, D, TILE, CU_TENSOR_MAP_DATA_TYPE_FLOAT16))
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
  if (nqb > 65535) return cudaErrorInvalidConfiguration;
  const dim3 grid_qk(static_cast<unsigned>(BH), static_cast<unsigned>(nqb));
  attn_qk_kernel<kLse><<<grid_qk, ATT_THREADS, qk_smem, stream>>>(tm_q, tm_k, lse, tsc, prm, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  attn_qk_kernel<kColScore><<<grid_qk, ATT_THREADS, qk_smem, stream>>>(tm_q, tm_k, lse, tsc, prm, err);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 5. token selection and causal prefixes
  e = launch_topk(tsc, BH, S, S, kt, idx_t, kt, stream);
  if (e != cudaSuccess) return e;
  attn_prefix_kernel<<<static_cast<unsigned>((BH * nqb + 255) / 256), 256, 0, stream>>>(
      idx_t, static_cast<int>(BH), static_cast<int>(kt), static_cast<int>(S), nqb, nvalid);
  if ((e = cudaGetLastError()) != cudaSuccess) return e;
  // 6. kept rows of K_I and V
  {
    const dim3 grid(static_cast<unsigned>((kt + 7) / 8), static_cast<unsigned>(BH));
    gather_heads_kernel<<<grid, 256, 0, stream>>>(reinterpret_cast<const uint4*>(ki), static_cast<int>(Hq),
                                                  static_cast<int>(Hq), static_cast<int>(S),
                                                  static_cast<int>(w.ldk / 8), idx_t, static_cast<int>(kt),
                                                  static_cast<int>(w.ldk / 8), reinterpret_cast<uint4*>(kt_rows),
                                                  static_cast<int>(w.ldk / 8));
    gather_v_f16_kernel<<<grid, 256, 0, stream>>>(static_cast<const uint4*>(V), static_cast<int>(Hq),
                                                  static_cast<int>(Hkv), static_cast<int>(S),
                                                  static_cast<int>(D / 8), idx_t, static_cast<int>(kt),
                                                  static_cast<int>(D / 8), reinterpret_cast<uint4*>(vt_rows),
                                                  static_cast<int>(D / 8), err);
    e = cudaGetLastError();
    if (e != cudaSuccess) return e;
  }
  // 7. pass C: on SM pairs when D = 128 (a pair's CTA takes 64 of V's columns)
  int dev = 0, max_smem = 0;
  if ((e = cudaGetDevice(&dev)) != cudaSuccess ||
      (e = cudaDeviceGetAttribute(&max_smem, cudaDevAttrMaxSharedMemoryPerBlockOptin, dev)) != cudaSuccess)
    return e;
  if (D == 128) {
    // key and value rings of 3 (one stage per logit / P' buffer); at least
    // CP_MIN_SMEM so a second CTA cannot share the SM's tensor memory
    const int pair_smem = std::max(kc * CHUNK_BYTES + CP_KS * kc * CP_KCHUNK_BYTES + CP_VS * CHUNK_BYTES +
                                       static_cast<int>(sizeof(PairOutBars)) + 1024,
                                   CP_MIN_SMEM);
    if (pair_smem > max_smem) return cudaErrorInvalidValue;
    CUtensorMap tm_kh;
    if (!encode_heads(&tm_kh, kt_rows, kd, kt, BH, w.ldk, CP_HALF_ROWS)) return cudaErrorInvalidValue;
    {
      std::lock_guard<std::mutex> lock(mu);
      if (!set_smem(attn_out_pair_kernel, pair_smem)) {
        set_error("rmm_attention: cannot set %d bytes of shared memory for pass C", pair_smem);
        return cudaErrorInvalidValue;
      }
    }
    const dim3 grid_pair(static_cast<unsigned>(2 * BH), static_cast<unsigned>((nqb + 1) / 2));
    attn_out_pair_kernel<<<grid_pair, PAIR_THREADS, pair_smem, stream>>>(tm_q, tm_kh, tm_vt, lse, idx_t, nvalid, O,
                                                                         prm, err);
    return cudaGetLastError();
  }
  auto out_smem_for = [&](int ks, int vs) {
    return kc * CHUNK_BYTES + ks * kc * CHUNK_BYTES + vs * static_cast<int>(D / 64) * CHUNK_BYTES +
           static_cast<int>(sizeof(OutBars)) + 1024;
  };
  // deepest key and value rings that fit (the value ring grows first)
  prm.c_ks = 2;
  prm.c_vs = 1;
  for (int d = C_MAX_VS; d >= 1; --d) {
    const int kd_ring = std::min(d, C_MAX_KS) < 2 ? 2 : std::min(d, C_MAX_KS);
    if (out_smem_for(kd_ring, d) <= max_smem) {
      prm.c_ks = kd_ring;
      prm.c_vs = d;
      break;
    }
  }
  const int out_smem = out_smem_for(prm.c_ks, prm.c_vs);
  {
    std::lock_guard<std::mutex> lock(mu);
    if (!set_smem(attn_out_kernel, out_smem)) {
      set_error("rmm_attention: cannot set %d bytes of shared memory for pass C", out_smem);
      return cudaErrorInvalidValue;
    }
  }
  attn_out_kernel<<<grid_qk, ATT_THREADS, out_smem, stream>>>(tm_q, tm_kt, tm_vt, lse, idx_t, nvalid, O, prm, err);
  return cudaGetLastError();
}

}  // namespace rmm

