// rmm_gemm_tc.cu — the reduced product Y = A_I · B_I on the 5th-generation
// tensor cores, where A_I = A[:, I] and B_I = B[I, :] are the compacted
// operands (Reduced Matrix Multiplication technical summary, Metodología ›
// Mecanismo Central: compute A_{:,I} B_{I,:} instead of AB).
//
// Persistent, warp-specialised kernel, one CTA per SM, 128 x 256 output tiles,
// 64-deep K blocks, 4-stage shared-memory ring, fp32 accumulators in tensor
// memory (two 256-column buffers, so the epilogue of one tile overlaps the
// main loop of the next).
//   warp 0     producer (one lane): per k-block, one TMA load of the A_I tile
//              (128 rows x 64, K-major) and four of the B_I tile (64 rows x 64
//              columns each, MN-major), all with 128-byte swizzle; rows and
//              columns past M, N or k read as zero.
//   warp 1     TMEM allocation; one thread issues tcgen05.mma (M=128, N=256,
//              K=16 per instruction, four per k-block) and tcgen05.commit to
//              release stages and publish finished accumulators.
//   warps 2-9  epilogue: two warps per TMEM lane quarter, each draining 128
//              of the 256 columns with tcgen05.ld, converting, and storing rows
//              of Y with 16-byte stores.  With an int8 weight (B_I widened to
//              exact bf16 integers by the gather) the epilogue multiplies each
//              column by its scale first.
// All waits are bounded (rmm_device.cuh); on a timeout the kernel records an
// error, drains its own copies and MMAs, frees TMEM and returns.
//
// Activations of 256 rows or more use the CTA-pair variant below (256 x 256
// tiles, tcgen05.mma.cta_group::2), which halves each SM's share of B and
// so cuts the operand bytes each SM pulls from L2 per MMA by a third; the
// single-CTA kernel serves smaller M.
//
// Why B_I is a copy rather than a gather in the operand path: gathering the
// k rows of B per k-block with tile::gather4 (64 four-row TMA gathers per
// stage) or with 16-byte cp.async was measured on B200 at about 2.2 TB/s of
// operand delivery, an order of magnitude short of what the tensor cores
// consume; a streaming row copy plus large-box TMA tiles is faster overall.
// The pair kernel can run that copy itself (kFused): the launch before it
// copies the column blocks its first wave of tiles reads, and four more warps
// per CTA copy the rest while the first wave multiplies (see pairk below).
#include <cuda.h>
#include <cuda_bf16.h>

#include <mutex>

#include "rmm_device.cuh"
#include "rmm_internal.h"
#include "rmm_launch.cuh"

namespace rmm {
namespace {

constexpr int BM = 128, BN = 256, BK = 64, STAGES = 4;
constexpr int A_STAGE = BM * BK * 2;   // 16 KB
constexpr int B_STAGE = BK * BN * 2;   // 32 KB
constexpr int B_CHUNK = BK * 128;      // one 64-column chunk of a B stage: 8 KB
constexpr int MMA_WARP = 1;
constexpr int EPI_WARP0 = 2;
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (EPI_WARP0 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int BAR_BYTES = 256;
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE) + BAR_BYTES + 1024;

static_assert(BK == 64 && BN == 256, "stage layout assumes 64 x 256 B stages");

struct Bars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t accfull[2];
  uint64_t accempty[2];
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};
static_assert(sizeof(Bars) <= BAR_BYTES, "barrier block");


// Multiply 32 accumulator values (columns col0 .. col0+31, masked at N) by
// their column scales (the per-column scales of an int8 weight).  Every lane
// of the warp reads the same 32 scales.
__device__ __forceinline__ void scale_row32(const float* __restrict__ col_scale, int col0, int N, uint32_t (&v)[32]) {
  if (col0 + 32 <= N && (reinterpret_cast<uintptr_t>(col_scale) & 15) == 0) {
#pragma unroll
    for (int i = 0; i < 8; ++i) {
      const float4 c = __ldg(reinterpret_cast<const float4*>(col_scale + col0) + i);
      v[4 * i] = __float_as_uint(__uint_as_float(v[4 * i]) * c.x);
      v[4 * i + 1] = __float_as_uint(__uint_as_float(v[4 * i + 1]) * c.y);
      v[4 * i + 2] = __float_as_uint(__uint_as_float(v[4 * i + 2]) * c.z);
      v[4 * i + 3] = __float_as_uint(__uint_as_float(v[4 * i + 3]) * c.w);
    }
  } else {
#pragma unroll
    for (int e = 0; e < 32; ++e)
      if (col0 + e < N) v[e] = __float_as_uint(__uint_as_float(v[e]) * __ldg(col_scale + col0 + e));
  }
}

// Store 32 fp32 accumulator values of one output row (columns col0 ..
// col0+31, masked at N) as fp32 or bf16, with 16-byte stores when aligned.
__device__ __forceinline__ void store_row32(void* Y, int out_f32, int64_t ldy, int y_vec_ok, int row, int col0, int N,
                                            const uint32_t (&v)[32]) {
  if (out_f32) {
    float* y = static_cast<float*>(Y) + static_cast<int64_t>(row) * ldy + col0;
    if (y_vec_ok && col0 + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 8; ++i)
        reinterpret_cast<float4*>(y)[i] = make_float4(__uint_as_float(v[4 * i]), __uint_as_float(v[4 * i + 1]),
                                                      __uint_as_float(v[4 * i + 2]), __uint_as_float(v[4 * i + 3]));
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (col0 + e < N) y[e] = __uint_as_float(v[e]);
    }
  } else {
    __nv_bfloat16* y = static_cast<__nv_bfloat16*>(Y) + static_cast<int64_t>(row) * ldy + col0;
    if (y_vec_ok && col0 + 32 <= N) {
#pragma unroll
      for (int i = 0; i < 4; ++i) {
        uint4 w;
        w.x = pack_bf16x2(__uint_as_float(v[8 * i + 0]), __uint_as_float(v[8 * i + 1]));
        w.y = pack_bf16x2(__uint_as_float(v[8 * i + 2]), __uint_as_float(v[8 * i + 3]));
        w.z = pack_bf16x2(__uint_as_float(v[8 * i + 4]), __uint_as_float(v[8 * i + 5]));
        w.w = pack_bf16x2(__uint_as_float(v[8 * i + 6]), __uint_as_float(v[8 * i + 7]));
        reinterpret_cast<uint4*>(y)[i] = w;
      }
    } else {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        if (col0 + e < N) y[e] = __float2bfloat16_rn(__uint_as_float(v[e]));
    }
  }
}

__global__ void __launch_bounds__(THREADS, 1)
    gemm_bf16_tc_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b, int M,
                        int N, int K, void* __restrict__ Y, int out_f32, int64_t ldy, int y_vec_ok,
                        const float* __restrict__ col_scale, unsigned* err) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t base = smem_u32(smem);
  Bars* bars = reinterpret_cast<Bars*>(smem + STAGES * (A_STAGE + B_STAGE));
  volatile int* abort_flag = &bars->abort_flag;
  auto sA = [&](uint32_t s) { return base + s * A_STAGE; };
  auto sB = [&](uint32_t s) { return base + STAGES * A_STAGE + s * B_STAGE; };
  auto full = [&](uint32_t s) { return smem_u32(&bars->full[s]); };
  auto empty = [&](uint32_t s) { return smem_u32(&bars->empty[s]); };
  auto accfull = [&](uint32_t b) { return smem_u32(&bars->accfull[b]); };
  auto accempty = [&](uint32_t b) { return smem_u32(&bars->accempty[b]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int num_m = (M + BM - 1) / BM, num_n = (N + BN - 1) / BN;
  const int num_tiles = num_m * num_n;
  const int nk = (K + BK - 1) / BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full(s), 1);   // producer: arrive + expected transaction bytes
      mbar_init(empty(s), 1);  // tcgen05.commit
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull(b), 1);           // tcgen05.commit
      mbar_init(accempty(b), EPI_WARPS);  // one arrive per epilogue warp
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == MMA_WARP) {
    tmem_alloc(smem_u32(&bars->tmem_slot), TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_slot;
  // set-up above overlaps the previous kernel's tail; operands are read after
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x) {
        const int m_blk = tile % num_m, n_blk = tile / num_m;
        const int n0 = n_blk * BN;
        const int live_chunks = min(4, (N - n0 + 63) / 64);
        const uint32_t stage_bytes = A_STAGE + static_cast<uint32_t>(live_chunks) * B_CHUNK;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, err, 1)) {
            ok = false;
            break;
          }
          mbar_arrive_expect_tx(full(stage), stage_bytes);
          tma_load_2d(sA(stage), &tmap_a, full(stage), kb * BK, m_blk * BM);
          for (int c = 0; c < live_chunks; ++c)
            tma_load_2d(sB(stage) + c * B_CHUNK, &tmap_b, full(stage), n0 + c * 64, kb * BK);
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // the copies this thread issued must land before the CTA may exit
      uint32_t st = stage, ph = phase;
      const uint32_t n = issued < STAGES ? issued : STAGES;
      for (uint32_t j = 0; j < n; ++j) {
        if (st == 0) {
          st = STAGES - 1;
          ph ^= 1u;
        } else {
          --st;
        }
        wait_drain(full(st), ph);
      }
    }
    __syncwarp();
  } else if (warp == MMA_WARP) {
    // ------------------------------------------------------------ MMA issuer
    constexpr uint32_t idesc = idesc_bf16_f32(BM, BN, /*a_mn=*/false, /*b_mn=*/true);
    uint32_t stage = 0, phase = 0;
    int it = 0;
    bool ok = true;
    for (int tile = blockIdx.x; ok && tile < num_tiles; tile += gridDim.x, ++it) {
      const uint32_t b = it & 1, acc_phase = (it >> 1) & 1;
      if (!mbar_wait_warp(accempty(b), acc_phase ^ 1u, abort_flag, err, 2)) break;
      tc_fence_after();
      const uint32_t d_tmem = tmem_base + b * BN;
      for (int kb = 0; kb < nk; ++kb) {
        if (!mbar_wait_warp(full(stage), phase, abort_flag, err, 3)) {
          ok = false;
          break;
        }
        tc_fence_after();
        if (lane == 0) {
#pragma unroll
          for (int kk = 0; kk < BK / 16; ++kk) {
            const uint64_t ad = sdesc_sw128(sA(stage) + kk * 32, 16, 1024);
            const uint64_t bd = sdesc_sw128(sB(stage) + kk * 16 * 128, B_CHUNK, 1024);
            mma_f16_ss(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
          }
          mma_commit(empty(stage));
        }
        __syncwarp();
        if (++stage == STAGES) {
          stage = 0;
          phase ^= 1u;
        }
      }
      if (!ok) break;
      if (lane == 0) mma_commit(accfull(b));
      __syncwarp();
    }
    if (lane == 0) {
      mma_commit(smem_u32(&bars->drain));
      wait_drain(smem_u32(&bars->drain), 0);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int qtr = warp & 3;                 // TMEM lanes 32*qtr ... 32*qtr+31
    const int half = (warp - EPI_WARP0) / 4;  // columns [128*half, 128*half + 128)
    int it = 0;
    for (int tile = blockIdx.x; tile < num_tiles; tile += gridDim.x, ++it) {
      const uint32_t b = it & 1, acc_phase = (it >> 1) & 1;
      if (!mbar_wait_warp(accfull(b), acc_phase, abort_flag, err, 4)) break;
      tc_fence_after();
      const int m_blk = tile % num_m, n_blk = tile / num_m;
      const int row = m_blk * BM + qtr * 32 + lane;
      const uint32_t taddr = tmem_base + b * BN + half * 128 + (static_cast<uint32_t>(qtr * 32) << 16);
#pragma unroll 1
      for (int cc = 0; cc < 4; ++cc) {
        uint32_t v[32];
        tmem_ld32(taddr + cc * 32, v);
        tmem_wait_ld();
        const int col0 = n_blk * BN + half * 128 + cc * 32;
        if (row < M && col0 < N) {
          if (col_scale) scale_row32(col_scale, col0, N, v);
          store_row32(Y, out_f32, ldy, y_vec_ok, row, col0, N, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive(accempty(b));
    }
  }

  __syncthreads();
  if (warp == MMA_WARP) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// ---------------------------------------------------------------- CTA-pair kernel
//
// Same pipeline on a pair of SMs (a 2-CTA cluster) computing 256 x 256
// tiles with tcgen05.mma.cta_group::2 (M = 256): each CTA loads 128 rows of
// A_I and 128 of the tile's 256 columns of B_I per k-block (32 KB per SM per
// stage instead of 48 KB for the same MMA work per SM), and each CTA's
// tensor memory holds its 128 rows x 256 columns of the accumulator.
//   - both CTAs' TMA loads signal the leader's (rank 0) full barrier, whose
//     expected bytes the leader registers for both halves;
//   - the leader's single MMA thread issues the pair MMAs; its commits arrive
//     on the empty / accumulator-full barriers of both CTAs (multicast);
//   - both CTAs' epilogue warps arrive on the leader's accumulator-empty
//     barrier;
//   - cluster barriers after set-up and before tensor memory is released;
//   - kFused: warps 10-13 of both CTAs copy B_I's column blocks from
//     nb_first on, 16 kept rows x 256 columns per unit, in column-block order,
//     and count finished units per block; the producer acquires an item's
//     block count before its first B load (bounded wait, site 45).  The
//     copy warps never wait, and units are handed out by a ticket counter, so
//     the copy progresses whichever CTAs are resident.
// Work items: tiles below `split_from` are whole 256 x 256 tiles; each tile
// from `split_from` on is done as two 256 x 128 halves (MMA N = 128, each
// CTA holding one 64-column chunk of B).  The host splits the tiles of a last
// partial wave when their halves still fit in one wave, so that wave ends in
// about half the time.
namespace pairk {
constexpr int BM = 256, BN = 256, BK = 64, STAGES = 6;
constexpr int A_STAGE = 128 * BK * 2;           // this CTA's 128 rows: 16 KB
constexpr int B_CHUNK = BK * 128;               // 64 columns x 64 rows: 8 KB
constexpr int B_STAGE = 2 * B_CHUNK;            // this CTA's 128 columns: 16 KB
constexpr uint32_t STAGE_TX = 2 * (A_STAGE + B_STAGE);
constexpr uint32_t STAGE_TX_HALF = 2 * (A_STAGE + B_CHUNK);
constexpr int EPI_WARPS = 8;
constexpr int THREADS = (2 + EPI_WARPS) * 32;
constexpr uint32_t TMEM_COLS = 2 * BN;
constexpr int SMEM_BYTES = STAGES * (A_STAGE + B_STAGE) + BAR_BYTES + 1024;

struct PairBars {
  uint64_t full[STAGES];
  uint64_t empty[STAGES];
  uint64_t accfull[2];
  uint64_t accempty[2];
  uint64_t drain;
  uint32_t tmem_slot;
  int abort_flag;
};
static_assert(sizeof(PairBars) <= BAR_BYTES, "barrier block");

// Fused row gather: warps [2 + EPI_WARPS, 2 + EPI_WARPS + GATHER_WARPS)
// copy units of GATHER_ROWS kept rows x BN columns of B into B_I.  Measured
// on the MLP up-projection: 16-row units beat 32-row ones (the copy of a unit
// is one round of loads), and 4 warps beat 2 or 8.
constexpr int GATHER_WARPS = 4;
constexpr int GATHER_ROWS = 16;
static_assert(GATHER_ROWS % 16 == 0 && GATHER_ROWS <= 32, "a lane holds one kept row; rows are loaded 16 at a time");
constexpr int THREADS_FUSED = THREADS + GATHER_WARPS * 32;

struct Item {
  int m_blk, n0, width;  // tile rows m_blk*256.., columns n0 .. n0+width-1
};
__device__ __forceinline__ Item item_of(int i, int split_from, int num_m) {
  if (i < split_from) return Item{i % num_m, (i / num_m) * BN, BN};
  const int j = i - split_from;
  const int tile = split_from + (j >> 1);
  return Item{tile % num_m, (tile / num_m) * BN + (j & 1) * (BN / 2), BN / 2};
}
// Device view of the fused gather.  ctr[0]: unit tickets; ctr[1]: unused;
// ctr[2 + b]: finished units of 256-column block b.
struct GatherArgs {
  const uint8_t* B;
  int64_t ldb_bytes;
  const int32_t* idx;
  int64_t d;
  uint8_t* BI;
  int64_t ldbi_bytes;
  uint32_t* ctr;
  int b_int8;
  int nb_first;  // column blocks [0, nb_first) of B_I were copied before the launch
};

// One gather warp: take units until none is left.  Unit u covers column
// block nb_first + u / chunks (BN columns; lane l copies columns 8l .. 8l+7
// of it) and kept rows [16 (u % chunks), +16) (lane l < 16 holds the source
// row of kept row l).  All sixteen rows are loaded before any is stored.  An
// out-of-range index gives a zero row and is flagged.  When a unit's stores
// are done the warp fences them (generic and async proxy) and adds one to its
// block's counter with release semantics, which the TMA producer acquires.
__device__ __forceinline__ void gather_units(const GatherArgs& g, int N, int K, unsigned* err) {
  const int lane = threadIdx.x & 31;
  const int num_n = (N + BN - 1) / BN;
  const int chunks = (K + GATHER_ROWS - 1) / GATHER_ROWS;
  const uint32_t units = static_cast<uint32_t>(num_n - g.nb_first) * static_cast<uint32_t>(chunks);
  for (;;) {
    uint32_t u = 0;
    if (lane == 0) u = atomicAdd(g.ctr, 1u);
    u = __shfl_sync(0xFFFFFFFFu, u, 0);
    if (u >= units) break;
    const int nb = g.nb_first + static_cast<int>(u / chunks), r0 = static_cast<int>(u % chunks) * GATHER_ROWS;
    const int nr = min(GATHER_ROWS, K - r0);
    const int col = nb * BN + lane * 8;
    const bool cok = col < N;  // N is a multiple of 8
    int j = lane < nr ? __ldg(g.idx + r0 + lane) : 0;
    if (lane < nr && (j < 0 || static_cast<int64_t>(j) >= g.d)) {
      record_error(err, kDevErrBadIndex);
      j = -1;
    }
    uint8_t* dst = g.BI + static_cast<int64_t>(r0) * g.ldbi_bytes + static_cast<int64_t>(col) * 2;
#pragma unroll 1
    for (int h = 0; h < GATHER_ROWS; h += 16) {
      uint4 v[16];
      if (!g.b_int8) {
        const uint8_t* src = g.B + static_cast<int64_t>(col) * 2;
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int jr = __shfl_sync(0xFFFFFFFFu, j, h + q);
          v[q] = (h + q < nr && cok && jr >= 0)
                     ? __ldcs(reinterpret_cast<const uint4*>(src + static_cast<int64_t>(jr) * g.ldb_bytes))
                     : make_uint4(0u, 0u, 0u, 0u);
        }
      } else {
        const uint8_t* src = g.B + col;
        uint2 w[16];
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          const int jr = __shfl_sync(0xFFFFFFFFu, j, h + q);
          w[q] = (h + q < nr && cok && jr >= 0)
                     ? __ldcs(reinterpret_cast<const uint2*>(src + static_cast<int64_t>(jr) * g.ldb_bytes))
                     : make_uint2(0u, 0u);
        }
#pragma unroll
        for (int q = 0; q < 16; ++q) {
          float lo[4], hi[4];
          i8x4_to_f32(w[q].x, lo);
          i8x4_to_f32(w[q].y, hi);
          v[q] = make_uint4(pack_bf16x2(lo[0], lo[1]), pack_bf16x2(lo[2], lo[3]), pack_bf16x2(hi[0], hi[1]),
                            pack_bf16x2(hi[2], hi[3]));
        }
      }
#pragma unroll
      for (int q = 0; q < 16; ++q)
        if (h + q < nr && cok) *reinterpret_cast<uint4*>(dst + static_cast<int64_t>(h + q) * g.ldbi_bytes) = v[q];
    }
    fence_proxy_async_global();
    __threadfence();
    __syncwarp();
    if (lane == 0) red_release_gpu_add(g.ctr + 2 + nb, 1u);
  }
}
}  // namespace pairk

template <bool kFused>
__global__ void __cluster_dims__(2, 1, 1) __launch_bounds__(kFused ? pairk::THREADS_FUSED : pairk::THREADS, 1)
    gemm_bf16_tc_pair_kernel(const __grid_constant__ CUtensorMap tmap_a, const __grid_constant__ CUtensorMap tmap_b,
                             int M, int N, int K, int split_from, void* __restrict__ Y, int out_f32, int64_t ldy,
                             int y_vec_ok, const float* __restrict__ col_scale, unsigned* err, pairk::GatherArgs g) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw_s = smem_u32(smem_raw);
  uint8_t* smem = smem_raw + ((1024u - (raw_s & 1023u)) & 1023u);
  const uint32_t base = smem_u32(smem);
  pairk::PairBars* bars = reinterpret_cast<pairk::PairBars*>(smem + pairk::STAGES * (pairk::A_STAGE + pairk::B_STAGE));
  volatile int* abort_flag = &bars->abort_flag;
  auto sA = [&](uint32_t s) { return base + s * pairk::A_STAGE; };
  auto sB = [&](uint32_t s) { return base + pairk::STAGES * pairk::A_STAGE + s * pairk::B_STAGE; };
  auto full = [&](uint32_t s) { return smem_u32(&bars->full[s]); };
  auto empty = [&](uint32_t s) { return smem_u32(&bars->empty[s]); };
  auto accfull = [&](uint32_t b) { return smem_u32(&bars->accfull[b]); };
  auto accempty = [&](uint32_t b) { return smem_u32(&bars->accempty[b]); };

  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const uint32_t rank = cluster_ctarank();
  const bool leader = rank == 0;
  const int cid = static_cast<int>(cluster_id_x()), ncl = static_cast<int>(nclusters_x());
  const int num_m = (M + pairk::BM - 1) / pairk::BM, num_n = (N + pairk::BN - 1) / pairk::BN;
  const int num_items = split_from + 2 * (num_m * num_n - split_from);
  const int nk = (K + pairk::BK - 1) / pairk::BK;

  if (threadIdx.x == 0) {
    for (int s = 0; s < pairk::STAGES; ++s) {
      mbar_init(full(s), 1);   // leader's producer: arrive + both CTAs' bytes
      mbar_init(empty(s), 1);  // pair commit (multicast)
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accfull(b), 1);               // pair commit (multicast)
      mbar_init(accempty(b), 2 * pairk::EPI_WARPS);  // epilogue warps of both CTAs
    }
    mbar_init(smem_u32(&bars->drain), 1);
    bars->abort_flag = 0;
    fence_mbar_init();
    prefetch_tmap(&tmap_a);
    prefetch_tmap(&tmap_b);
  }
  if (warp == 1) {
    tmem_alloc_pair(smem_u32(&bars->tmem_slot), pairk::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // barriers of both CTAs initialised before any cross-CTA signal
  tc_fence_after();
  const uint32_t tmem_base = bars->tmem_slot;
  pdl_wait();
  pdl_trigger();

  if (warp == 0) {
    // ------------------------------------------------------------ producer (both CTAs)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0, issued = 0;
      bool ok = true;
      for (int i = cid; ok && i < num_items; i += ncl) {
        const pairk::Item t = pairk::item_of(i, split_from, num_m);
        const bool whole = t.width == pairk::BN;
        if (kFused && t.n0 / pairk::BN >= g.nb_first) {
          // every unit of this tile's column block of B_I has been written
          const uint32_t chunks = static_cast<uint32_t>((K + pairk::GATHER_ROWS - 1) / pairk::GATHER_ROWS);
          if (!flag_wait_geq(g.ctr + 2 + t.n0 / pairk::BN, chunks, abort_flag, err, 45)) {
            ok = false;
            break;
          }
        }
        const int a_row = t.m_blk * pairk::BM + static_cast<int>(rank) * 128;
        const int b_col = t.n0 + static_cast<int>(rank) * (t.width / 2);
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait(empty(stage), phase ^ 1u, abort_flag, err, 41)) {
            ok = false;
            break;
          }
          const uint32_t full_leader = mapa_shared(full(stage), 0);
          if (leader) mbar_arrive_expect_tx(full(stage), whole ? pairk::STAGE_TX : pairk::STAGE_TX_HALF);
          tma_load_2d_pair(sA(stage), &tmap_a, full_leader, kb * pairk::BK, a_row);
          tma_load_2d_pair(sB(stage), &tmap_b, full_leader, b_col, kb * pairk::BK);
          if (whole)
            tma_load_2d_pair(sB(stage) + pairk::B_CHUNK, &tmap_b, full_leader, b_col + 64, kb * pairk::BK);
          ++issued;
          if (++stage == pairk::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (leader) {
        // the pair's copies for the last stages must land before either CTA exits
        uint32_t st = stage, ph = phase;
        const uint32_t n = issued < pairk::STAGES ? issued : pairk::STAGES;
        for (uint32_t j = 0; j < n; ++j) {
          if (st == 0) {
            st = pairk::STAGES - 1;
            ph ^= 1u;
          } else {
            --st;
          }
          wait_drain(full(st), ph);
        }
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (leader CTA)
    if (leader) {
      constexpr uint32_t idesc_whole = idesc_bf16_f32(pairk::BM, pairk::BN, /*a_mn=*/false, /*b_mn=*/true);
      constexpr uint32_t idesc_half = idesc_bf16_f32(pairk::BM, pairk::BN / 2, /*a_mn=*/false, /*b_mn=*/true);
      uint32_t stage = 0, phase = 0;
      int it = 0;
      bool ok = true;
      for (int i = cid; ok && i < num_items; i += ncl, ++it) {
        const uint32_t idesc = i < split_from ? idesc_whole : idesc_half;
        const uint32_t b = it & 1, acc_phase = (it >> 1) & 1;
        if (!mbar_wait_warp(accempty(b), acc_phase ^ 1u, abort_flag, err, 42)) break;
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * pairk::BN;
        for (int kb = 0; kb < nk; ++kb) {
          if (!mbar_wait_warp(full(stage), phase, abort_flag, err, 43)) {
            ok = false;
            break;
          }
          tc_fence_after();
          if (lane == 0) {
#pragma unroll
            for (int kk = 0; kk < pairk::BK / 16; ++kk) {
              const uint64_t ad = sdesc_sw128(sA(stage) + kk * 32, 16, 1024);
              const uint64_t bd = sdesc_sw128(sB(stage) + kk * 16 * 128, pairk::B_CHUNK, 1024);
              mma_f16_ss_pair(d_tmem, ad, bd, idesc, (kb | kk) != 0 ? 1u : 0u);
            }
            mma_commit_pair_multicast(empty(stage), 0x3);
          }
          __syncwarp();
          if (++stage == pairk::STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        if (lane == 0) mma_commit_pair_multicast(accfull(b), 0x3);
        __syncwarp();
      }
      if (lane == 0) {
        mma_commit_pair_multicast(smem_u32(&bars->drain), 0x1);
        wait_drain(smem_u32(&bars->drain), 0);
      }
      __syncwarp();
    }
  } else if (warp >= 2 + pairk::EPI_WARPS) {
    // ------------------------------------------------------------ fused row gather (both CTAs)
    if constexpr (kFused) pairk::gather_units(g, N, K, err);
  } else {
    // ------------------------------------------------------------ epilogue (both CTAs)
    const int qtr = warp & 3;
    const int half = (warp - 2) / 4;
    int it = 0;
    for (int i = cid; i < num_items; i += ncl, ++it) {
      const uint32_t b = it & 1, acc_phase = (it >> 1) & 1;
      if (!mbar_wait_warp(accfull(b), acc_phase, abort_flag, err, 44)) break;
      tc_fence_after();
      const pairk::Item t = pairk::item_of(i, split_from, num_m);
      const int hw = t.width / 2;  // accumulator columns per epilogue half
      const int row = t.m_blk * pairk::BM + static_cast<int>(rank) * 128 + qtr * 32 + lane;
      const uint32_t taddr = tmem_base + b * pairk::BN + half * hw + (static_cast<uint32_t>(qtr * 32) << 16);
#pragma unroll 1
      for (int cc = 0; cc < hw / 32; ++cc) {
        uint32_t v[32];
        tmem_ld32(taddr + cc * 32, v);
        tmem_wait_ld();
        const int col0 = t.n0 + half * hw + cc * 32;
        if (row < M && col0 < N) {
          if (col_scale) scale_row32(col_scale, col0, N, v);
          store_row32(Y, out_f32, ldy, y_vec_ok, row, col0, N, v);
        }
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(accempty(b), 0));
    }
  }

  tc_fence_before();
  cluster_sync();  // all MMAs, copies and remote arrivals of the pair are done
  tc_fence_after();
  if (warp == 1) tmem_dealloc_pair(tmem_base, pairk::TMEM_COLS);
}

// ---------------------------------------------------------------- host side

typedef CUresult (*EncodeTiledFn)(CUtensorMap*, CUtensorMapDataType, cuuint32_t, void*, const cuuint64_t*,
                                  const cuuint64_t*, const cuuint32_t*, const cuuint32_t*, CUtensorMapInterleave,
                                  CUtensorMapSwizzle, CUtensorMapL2promotion, CUtensorMapFloatOOBfill);

EncodeTiledFn encode_fn() {
  static EncodeTiledFn fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q{};
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<EncodeTiledFn>(p);
  });
  return fn;
}

bool configure_kernel_once() {
  static std::mutex mu;
  static bool done[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return false;
  std::lock_guard<std::mutex> lock(mu);
  if (!done[dev]) {
    if (cudaFuncSetAttribute(gemm_bf16_tc_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, SMEM_BYTES) !=
            cudaSuccess ||
        cudaFuncSetAttribute(gemm_bf16_tc_pair_kernel<false>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pairk::SMEM_BYTES) != cudaSuccess ||
        cudaFuncSetAttribute(gemm_bf16_tc_pair_kernel<true>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                             pairk::SMEM_BYTES) != cudaSuccess)
      return false;
    done[dev] = true;
  }
  return true;
}

// 2-D bf16 tensor map over a row-major [rows x cols] matrix (pitch in elements).
bool encode_2d(CUtensorMap* map, const void* ptr, int64_t cols, int64_t rows, int64_t pitch, uint32_t box_cols,
               uint32_t box_rows, const char* what) {
  EncodeTiledFn encode = encode_fn();
  if (!encode) {
    set_error("rmm_gemm: cuTensorMapEncodeTiled entry point unavailable");
    return false;
  }
  const cuuint64_t gdim[2] = {static_cast<cuuint64_t>(cols), static_cast<cuuint64_t>(rows)};
  const cuuint64_t gstride[1] = {static_cast<cuuint64_t>(pitch) * 2};
  const cuuint32_t box[2] = {box_cols, box_rows};
  const cuuint32_t estride[2] = {1, 1};
  const CUresult r = encode(map, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, 2, const_cast<void*>(ptr), gdim, gstride, box,
                            estride, CU_TENSOR_MAP_INTERLEAVE_NONE, CU_TENSOR_MAP_SWIZZLE_128B,
                            CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error("rmm_gemm: cuTensorMapEncodeTiled(%s) failed (CUresult %d)", what, static_cast<int>(r));
    return false;
  }
  return true;
}

}  // namespace

int64_t fused_gather_counter_words(int64_t N) { return 2 + (N + pairk::BN - 1) / pairk::BN; }

// Work items of the CTA-pair kernel and how many run in its first wave.
namespace {
struct PairPlan {
  int64_t split_from, items, clusters;
};
PairPlan pair_plan(int64_t M, int64_t N) {
  const int64_t tiles = ((M + pairk::BM - 1) / pairk::BM) * ((N + pairk::BN - 1) / pairk::BN);
  const int64_t pairs = device_sm_count() / 2;
  // split the tiles of a last partial wave into halves when those fit in one wave
  const int64_t rem = tiles % pairs;
  const int64_t split_from = (rem > 0 && 2 * rem <= pairs) ? tiles - rem : tiles;
  const int64_t items = split_from + 2 * (tiles - split_from);
  return PairPlan{split_from, items, items < pairs ? items : pairs};
}
}  // namespace

int64_t fused_gather_first_cols(int64_t M, int64_t N) {
  const PairPlan p = pair_plan(M, N);
  const int64_t num_m = (M + pairk::BM - 1) / pairk::BM;
  // items 0 .. clusters-1 run first; item i of a whole tile is column block i / num_m
  const int64_t first_item = p.clusters - 1;
  const int64_t nb = first_item < p.split_from ? first_item / num_m : (p.split_from + (first_item - p.split_from) / 2) / num_m;
  const int64_t cols = (nb + 1) * pairk::BN;
  return cols < N ? cols : N;
}

bool fused_gather_supported(int64_t M, int64_t N, int64_t k, const void* B, int64_t ldb, bool b_int8) {
  const int64_t belt = b_int8 ? 1 : 2;
  const int64_t units = ((N + pairk::BN - 1) / pairk::BN) * ((k + pairk::GATHER_ROWS - 1) / pairk::GATHER_ROWS);
  return M >= pairk::BM && N > 0 && N % 8 == 0 && k >= 1 && B != nullptr &&
         reinterpret_cast<uintptr_t>(B) % 16 == 0 && (ldb * belt) % 16 == 0 && units <= 0x7FFFFFFFLL;
}

cudaError_t launch_gemm_bf16_tc(const void* A_I, int64_t ld_ai, const void* B_I, int64_t ld_bi, int64_t M, int64_t N,
                                int64_t k, void* Y, int out_dtype, int64_t ldy, unsigned* err, cudaStream_t stream,
                                const float* col_scale, const FusedGather* fg) {
  if (M == 0 || N == 0) return cudaSuccess;
  if (fg && !fused_gather_supported(M, N, k, fg->B, fg->ldb, fg->b_int8)) return cudaErrorInvalidValue;
  CUtensorMap tmap_a, tmap_b;
  if (!encode_2d(&tmap_a, A_I, k, M, ld_ai, BK, BM, "A_I")) return cudaErrorInvalidValue;
  if (!encode_2d(&tmap_b, B_I, N, k, ld_bi, 64, BK, "B_I")) return cudaErrorInvalidValue;
  if (!configure_kernel_once()) {
    set_error("rmm_gemm: cannot raise the dynamic shared-memory limit to %d bytes", SMEM_BYTES);
    return cudaErrorInvalidValue;
  }
  const int sms = device_sm_count();
  const int out_f32 = out_dtype == 0 ? 1 : 0;
  const size_t oelt = out_f32 ? 4 : 2;
  const int y_vec_ok = (reinterpret_cast<uintptr_t>(Y) % 16 == 0) && ((ldy * oelt) % 16 == 0);
  if (M >= pairk::BM) {
    // 256 x 256 tiles on SM pairs: one 2-CTA cluster per pair of SMs
    const PairPlan p = pair_plan(M, N);
    if (p.items > 0x7FFFFFFFLL) return cudaErrorInvalidConfiguration;
    const int64_t split_from = p.split_from;
    const int clusters = static_cast<int>(p.clusters);
    if (fg && fg->n_ready < N) {
      const int64_t belt = fg->b_int8 ? 1 : 2;
      const pairk::GatherArgs g{static_cast<const uint8_t*>(fg->B), fg->ldb * belt, fg->idx, fg->d,
                                static_cast<uint8_t*>(const_cast<void*>(B_I)), ld_bi * 2, fg->ctr,
                                fg->b_int8 ? 1 : 0, static_cast<int>(fg->n_ready / pairk::BN)};
      return launch_pdl(gemm_bf16_tc_pair_kernel<true>, dim3(2 * clusters), dim3(pairk::THREADS_FUSED),
                        pairk::SMEM_BYTES, stream, tmap_a, tmap_b, static_cast<int>(M), static_cast<int>(N),
                        static_cast<int>(k), static_cast<int>(split_from), Y, out_f32, ldy, y_vec_ok, col_scale, err,
                        g);
    }
    return launch_pdl(gemm_bf16_tc_pair_kernel<false>, dim3(2 * clusters), dim3(pairk::THREADS), pairk::SMEM_BYTES,
                      stream, tmap_a, tmap_b, static_cast<int>(M), static_cast<int>(N), static_cast<int>(k),
                      static_cast<int>(split_from), Y, out_f32, ldy, y_vec_ok, col_scale, err, pairk::GatherArgs{});
  }
  const int64_t tiles = ((M + BM - 1) / BM) * ((N + BN - 1) / BN);
  const int grid = static_cast<int>(tiles < sms ? tiles : sms);
  return launch_pdl(gemm_bf16_tc_kernel, dim3(grid), dim3(THREADS), SMEM_BYTES, stream, tmap_a, tmap_b,
                    static_cast<int>(M), static_cast<int>(N), static_cast<int>(k), Y, out_f32, ldy, y_vec_ok, col_scale,
                    err);
}

}  // namespace rmm
