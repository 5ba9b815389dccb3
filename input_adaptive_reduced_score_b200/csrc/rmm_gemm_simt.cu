// rmm_gemm_simt.cu — fp32 reduced GEMM Y = A_I · B[I, :] with fp32 FMA
// (Reduced Matrix Multiplication technical summary, Metodología › Mecanismo
// Central).  Used for fp32 operands, where tf32 tensor cores would lose
// precision.  64 x 64 output tile per 256-thread CTA, 4 x 4 outputs per
// thread, k staged 16 at a time through shared memory with the B rows
// gathered by index.  Each output is one fma chain in ascending k order.
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

__global__ void __launch_bounds__(256) gemm_f32_simt_kernel(const float* __restrict__ AI, int64_t ld_ai,
                                                             const float* __restrict__ B, int64_t ldb,
                                                             const int32_t* __restrict__ idx, int d, int M, int N,
                                                             int K, float* __restrict__ Y, int64_t ldy,
                                                             unsigned* err) {
  __shared__ float As[TK][TM + 4];
  __shared__ float Bs[TK][TN];
  const int m0 = blockIdx.y * TM, n0 = blockIdx.x * TN;
  const int tx = threadIdx.x % 16, ty = threadIdx.x / 16;
  float acc[4][4] = {};
  bool bad = false;
  for (int k0 = 0; k0 < K; k0 += TK) {
#pragma unroll
    for (int i = 0; i < 4; ++i) {
      const int e = threadIdx.x + 256 * i;  // 0..1023
      const int mi = e / TK, ki = e % TK;   // A tile: 64 rows x 16 k
      const int m = m0 + mi, kk = k0 + ki;
      As[ki][mi] = (m < M && kk < K) ? AI[static_cast<int64_t>(m) * ld_ai + kk] : 0.f;
      const int kb = e / TN, ni = e % TN;   // B tile: 16 k x 64 cols
      const int kr = k0 + kb, n = n0 + ni;
      float bv = 0.f;
      if (kr < K && n < N) {
        const int row = __ldg(idx + kr);
        if (row >= 0 && row < d) {
          bv = B[static_cast<int64_t>(row) * ldb + n];
        } else {
          bad = true;
        }
      }
      Bs[kb][ni] = bv;
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float a[4], b[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) a[i] = As[kk][ty * 4 + i];
#pragma unroll
      for (int j = 0; j < 4; ++j) b[j] = Bs[kk][tx * 4 + j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(a[i], b[j], acc[i][j]);
    }
    __syncthreads();
  }
  if (bad) record_error(err, kDevErrBadIndex);
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int m = m0 + ty * 4 + i;
    if (m >= M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int n = n0 + tx * 4 + j;
      if (n < N) Y[static_cast<int64_t>(m) * ldy + n] = acc[i][j];
    }
  }
}

}  // namespace

cudaError_t launch_gemm_f32_simt(const float* A_I, int64_t ld_ai, const float* B, int64_t ldb, const int32_t* idx,
                                 int64_t d, int64_t M, int64_t N, int64_t k, float* Y, int64_t ldy, unsigned* err,
                                 cudaStream_t stream) {
  if (M == 0 || N == 0) return cudaSuccess;
  const dim3 grid(static_cast<unsigned>((N + TN - 1) / TN), static_cast<unsigned>((M + TM - 1) / TM));
  if (grid.y > 65535u) return cudaErrorInvalidConfiguration;
  gemm_f32_simt_kernel<<<grid, 256, 0, stream>>>(A_I, ld_ai, B, ldb, idx, static_cast<int>(d), static_cast<int>(M),
                                                  static_cast<int>(N), static_cast<int>(k), Y, ldy, err);
  return cudaGetLastError();
}

}  // namespace rmm
