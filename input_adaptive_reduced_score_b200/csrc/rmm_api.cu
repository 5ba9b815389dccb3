// rmm_api.cu — the extern "C" entry points of librmm (declared in rmm.h):
// argument validation, workspace carving, launches, error reporting.
#include <cuda_runtime.h>

#include <algorithm>
#include <cmath>
#include <cstdarg>
#include <cstdio>
#include <mutex>
#include <string>

#include "../../include/rmm.h"
#include "rmm_internal.h"

namespace rmm {

namespace {
thread_local std::string g_last_error;

// Per-device error word written by kernels (RMM_DEVERR_* codes).
__device__ unsigned g_device_error_word;
}  // namespace

void set_error(const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  g_last_error = buf;
}

void clear_error() { g_last_error.clear(); }

unsigned* device_error_word() {
  static std::mutex mu;
  static unsigned* cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) {
    set_error("no current CUDA device");
    return nullptr;
  }
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_device_error_word);
    if (e != cudaSuccess) {
      set_error("cudaGetSymbolAddress(error word): %s", cudaGetErrorString(e));
      return nullptr;
    }
    cache[dev] = static_cast<unsigned*>(p);
  }
  return cache[dev];
}

int device_sm_count() {
  static std::mutex mu;
  static int cache[64] = {};
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess || dev < 0 || dev >= 64) return 0;
  std::lock_guard<std::mutex> lock(mu);
  if (!cache[dev]) {
    int n = 0;
    if (cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev) != cudaSuccess) return 0;
    cache[dev] = n;
  }
  return cache[dev];
}

}  // namespace rmm

using namespace rmm;

namespace {

rmm_status fail(rmm_status s, const char* fmt, ...) {
  char buf[512];
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(buf, sizeof(buf), fmt, ap);
  va_end(ap);
  set_error("%s", buf);
  return s;
}

rmm_status from_cuda(cudaError_t e, const char* where) {
  if (e == cudaSuccess) return RMM_OK;
  return fail(RMM_ERR_CUDA, "%s: %s", where, cudaGetErrorString(e));
}

bool aligned16(const void* p) { return reinterpret_cast<uintptr_t>(p) % 16 == 0; }

size_t elt_size(int dtype) { return dtype == RMM_BF16 ? 2 : 4; }

bool valid_dtype(int dtype) { return dtype == RMM_F32 || dtype == RMM_BF16; }

constexpr int64_t kIntMax = 0x7FFFFFFFLL;

int64_t k_from_rho_impl(double rho, int64_t d) {
  if (!(rho > 0.0 && rho <= 1.0) || d < 1) return -1;
  const double x = rho * static_cast<double>(d) - 1e-9 * static_cast<double>(d);
  int64_t k = static_cast<int64_t>(std::ceil(x));
  if (k < 1) k = 1;
  if (k > d) k = d;
  return k;
}

int64_t round_up(int64_t x, int64_t a) { return (x + a - 1) / a * a; }

}  // namespace
extern "C" size_t rmm_gemm_workspace_size(int dtype, int64_t N, int64_t k);
namespace {

// Workspace of the bf16 product: B_I [k x round_up(N, 8)], then the counters
// of the fused row gather.
size_t gemm_bi_bytes(int64_t N, int64_t k) {
  return align_up(static_cast<size_t>(k) * static_cast<size_t>(round_up(N, 8)) * 2, kWsAlign);
}
uint32_t* gemm_counters(void* ws, int64_t N, int64_t k) {
  return reinterpret_cast<uint32_t*>(static_cast<char*>(ws) + gemm_bi_bytes(N, k));
}

// The bf16 tensor-core product with B_I = B[idx, :] filled in two parts: one
// launch copies the columns the product's first wave of tiles reads (and,
// given A, compacts A_I = A[:, idx] in the same grid) and zeroes the
// counters; then the product kernel, whose spare warps copy the remaining
// columns while the first wave multiplies.  A_I is [M x k] (ld_ai); B_I
// [k x N] (pitch round_up(N, 8)) at bi; ctr holds n_ctr zeroed words.
cudaError_t launch_fused_product(const void* A, int64_t lda, int64_t d, const void* B, int64_t ldb, bool b_int8,
                                 const int32_t* idx, int64_t k, void* ai, int64_t ld_ai, void* bi, uint32_t* ctr,
                                 int64_t n_ctr, int64_t M, int64_t N, void* Y, int out_dtype, int64_t ldy,
                                 const float* col_scale, unsigned* err, cudaStream_t s) {
  const int64_t ld_bi = round_up(N, 8);
  const int64_t n0 = fused_gather_first_cols(M, N);
  cudaError_t e = launch_compact_and_gather(A, A ? M : 0, d, A ? lda : d, B, n0, ldb, idx, k, ai, ld_ai, bi, ld_bi,
                                            err, s, b_int8, ctr, n_ctr);
  if (e != cudaSuccess) return e;
  const FusedGather fg{B, ldb, idx, d, ctr, b_int8, n0};
  return launch_gemm_bf16_tc(ai, ld_ai, bi, ld_bi, M, N, k, Y, out_dtype, ldy, err, s, col_scale, &fg);
}


struct MatmulWs {
  size_t ss, idx, score, ai, bi, total;
  int64_t k, ld_ai;
};

MatmulWs matmul_ws(int dtype, int64_t M, int64_t d, int64_t N, double rho) {
  MatmulWs w{};
  w.k = k_from_rho_impl(rho, d);
  if (w.k < 1) return w;
  w.ld_ai = round_up(w.k, 8);
  size_t off = 0;
  w.ss = off;
  off += align_up(static_cast<size_t>(d) * 4, kWsAlign);
  w.idx = off;
  off += align_up(static_cast<size_t>(w.k) * 4, kWsAlign);
  w.score = off;
  off += score_workspace_bytes(dtype, 1, M, d);
  w.ai = off;
  off += align_up(static_cast<size_t>(M) * w.ld_ai * elt_size(dtype), kWsAlign);
  w.bi = off;
  off += rmm_gemm_workspace_size(dtype, N, w.k);
  w.total = off;
  return w;
}

}  // namespace

extern "C" size_t rmm_matmul_multi_workspace_size(int64_t M, int64_t d, int64_t N_max, double rho);
extern "C" size_t rmm_silu_mul_score_workspace_size(int64_t M, int64_t N);
namespace {
struct MlpWs {
  size_t u, g, h, ss, inner, total;
  int64_t ld_ff;
};
MlpWs mlp_ws(int64_t M, int64_t d_model, int64_t d_ff, double rho_up, double rho_down) {
  MlpWs w{};
  w.ld_ff = round_up(d_ff, 8);
  const size_t act = align_up(static_cast<size_t>(M) * w.ld_ff * 2, kWsAlign);
  size_t off = 0;
  w.u = off;
  off += act;
  w.g = off;
  off += act;
  w.h = off;
  off += act;
  w.ss = off;
  off += align_up(static_cast<size_t>(d_ff) * 4, kWsAlign);
  w.inner = off;
  const size_t inner = std::max({rmm_matmul_multi_workspace_size(M, d_model, d_ff, rho_up),
                                 rmm_matmul_multi_workspace_size(M, d_ff, d_model, rho_down),
                                 rmm_silu_mul_score_workspace_size(M, d_ff)});
  w.total = off + inner;
  return w;
}
}  // namespace

extern "C" {

int rmm_abi_version(void) { return RMM_ABI_VERSION; }

const char* rmm_last_error(void) { return g_last_error.c_str(); }

int64_t rmm_k_from_rho(double rho, int64_t d) { return k_from_rho_impl(rho, d); }

rmm_status rmm_device_error(void* stream, int clear, unsigned* code) {
  clear_error();
  unsigned* w = device_error_word();
  if (!w) return RMM_ERR_CUDA;
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return from_cuda(e, "rmm_device_error: stream sync");
  unsigned v = 0;
  e = cudaMemcpy(&v, w, sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return from_cuda(e, "rmm_device_error: read");
  if (clear && v) {
    e = cudaMemset(w, 0, sizeof(unsigned));
    if (e != cudaSuccess) return from_cuda(e, "rmm_device_error: clear");
    e = cudaDeviceSynchronize();
    if (e != cudaSuccess) return from_cuda(e, "rmm_device_error: clear sync");
  }
  if (code) *code = v;
  if (v) return fail(RMM_ERR_DEVICE, "device error word = 0x%x", v);
  return RMM_OK;
}

size_t rmm_score_workspace_size(int dtype, int64_t batch, int64_t M, int64_t d) {
  if (!valid_dtype(dtype) || batch < 1 || M < 0 || d < 1) return 0;
  return score_workspace_bytes(dtype, batch, M, d);
}

rmm_status rmm_score(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                     int64_t batch_stride, float* ss, int64_t ld_ss, int sqrt_out, void* ws, size_t ws_bytes,
                     void* stream) {
  clear_error();
  if (!valid_dtype(dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_score: dtype %d", dtype);
  if (batch < 1 || batch > 65535 || M < 0 || d < 1 || lda < d || ld_ss < d)
    return fail(RMM_ERR_INVALID_ARG, "rmm_score: bad sizes (batch %lld M %lld d %lld lda %lld ld_ss %lld)",
                (long long)batch, (long long)M, (long long)d, (long long)lda, (long long)ld_ss);
  if (batch > 1 && batch_stride < M * lda)
    return fail(RMM_ERR_INVALID_ARG, "rmm_score: batch_stride smaller than one matrix");
  if (!ss || (M > 0 && !A)) return fail(RMM_ERR_INVALID_ARG, "rmm_score: null pointer");
  const size_t need = score_workspace_used(A, dtype, batch, M, d, lda, batch_stride);
  if (need && (!ws || ws_bytes < need))
    return fail(RMM_ERR_WORKSPACE, "rmm_score: workspace %zu < %zu bytes", ws_bytes, need);
  if (M == 0) {
    for (int64_t b = 0; b < batch; ++b) {
      cudaError_t e = cudaMemsetAsync(ss + b * ld_ss, 0, d * sizeof(float), static_cast<cudaStream_t>(stream));
      if (e != cudaSuccess) return from_cuda(e, "rmm_score: memset");
    }
    return RMM_OK;
  }
  return from_cuda(launch_score(A, dtype, batch, M, d, lda, batch_stride, ss, ld_ss, sqrt_out, ws,
                                static_cast<cudaStream_t>(stream)),
                   "rmm_score: launch");
}

rmm_status rmm_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k, int32_t* idx,
                    int64_t ld_idx, void* stream) {
  clear_error();
  if (!scores || !idx) return fail(RMM_ERR_INVALID_ARG, "rmm_topk: null pointer");
  if (batch < 1 || batch > kIntMax || d < 1 || d > kIntMax || ld_s < d)
    return fail(RMM_ERR_INVALID_ARG, "rmm_topk: bad sizes");
  if (k < 1 || k > d) return fail(RMM_ERR_INVALID_ARG, "rmm_topk: k = %lld outside [1, %lld]", (long long)k, (long long)d);
  if (ld_idx < k) return fail(RMM_ERR_INVALID_ARG, "rmm_topk: ld_idx < k");
  return from_cuda(launch_topk(scores, batch, d, ld_s, k, idx, ld_idx, static_cast<cudaStream_t>(stream)),
                   "rmm_topk: launch");
}

rmm_status rmm_compact(const void* A, int dtype, int64_t M, int64_t d, int64_t lda, const int32_t* idx, int64_t k,
                       void* A_I, int64_t ld_ai, void* stream) {
  clear_error();
  if (!valid_dtype(dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_compact: dtype %d", dtype);
  if (M < 0 || d < 1 || lda < d || k < 1 || k > d || ld_ai < k)
    return fail(RMM_ERR_INVALID_ARG, "rmm_compact: bad sizes");
  if (M > 0 && (!A || !idx || !A_I)) return fail(RMM_ERR_INVALID_ARG, "rmm_compact: null pointer");
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  return from_cuda(launch_compact(A, dtype, M, d, lda, idx, k, A_I, ld_ai, err, static_cast<cudaStream_t>(stream)),
                   "rmm_compact: launch");
}

size_t rmm_gemm_workspace_size(int dtype, int64_t N, int64_t k) {
  if (dtype != RMM_BF16 || N < 1 || k < 1) return 0;
  return gemm_bi_bytes(N, k) + align_up(static_cast<size_t>(fused_gather_counter_words(N)) * 4, kWsAlign);
}

rmm_status rmm_gather_rows(const void* B, int dtype, int64_t d, int64_t N, int64_t ldb, const int32_t* idx, int64_t k,
                           void* B_I, int64_t ld_bi, void* stream) {
  clear_error();
  if (!valid_dtype(dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_gather_rows: dtype %d", dtype);
  if (d < 1 || N < 0 || ldb < N || k < 1 || ld_bi < N)
    return fail(RMM_ERR_INVALID_ARG, "rmm_gather_rows: bad sizes");
  if (N == 0) return RMM_OK;
  if (!B || !idx || !B_I) return fail(RMM_ERR_INVALID_ARG, "rmm_gather_rows: null pointer");
  const int64_t e = static_cast<int64_t>(elt_size(dtype));
  if (!aligned16(B) || !aligned16(B_I) || (ldb * e) % 16 || (ld_bi * e) % 16)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_gather_rows: needs 16-byte aligned bases and row pitches");
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  return from_cuda(launch_gather_rows(B, d, N * e, ldb * e, idx, k, B_I, ld_bi * e, err,
                                      static_cast<cudaStream_t>(stream)),
                   "rmm_gather_rows: launch");
}

rmm_status rmm_compact_gather(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t M, int64_t d,
                              int64_t N, const int32_t* idx, int64_t k, void* A_I, int64_t ld_ai, void* B_I,
                              int64_t ld_bi, void* stream) {
  clear_error();
  if (M < 0 || N < 0 || d < 1 || lda < d || ldb < N || k < 1 || k > d || ld_ai < k || ld_bi < N || d > kIntMax)
    return fail(RMM_ERR_INVALID_ARG, "rmm_compact_gather: bad sizes");
  if (M == 0 && N == 0) return RMM_OK;
  if (!idx || (M > 0 && (!A || !A_I)) || (N > 0 && (!B || !B_I)))
    return fail(RMM_ERR_INVALID_ARG, "rmm_compact_gather: null pointer");
  if (N > 0 && (!aligned16(B) || !aligned16(B_I) || ldb % 8 || ld_bi % 8))
    return fail(RMM_ERR_UNSUPPORTED, "rmm_compact_gather: needs 16-byte aligned B/B_I, ldb and ld_bi multiples of 8");
  if (k + ((M + 7) / 8) * ((k + 63) / 64) > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "rmm_compact_gather: grid");
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  return from_cuda(launch_compact_and_gather(A, M, d, lda, B, N, ldb, idx, k, A_I, ld_ai, B_I, ld_bi, err,
                                             static_cast<cudaStream_t>(stream)),
                   "rmm_compact_gather: launch");
}

rmm_status rmm_gemm(const void* A_I, int64_t ld_ai, const void* B, int64_t ldb, const int32_t* idx, int64_t d,
                    int64_t M, int64_t N, int64_t k, int dtype, void* Y, int out_dtype, int64_t ldy, void* ws,
                    size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(dtype) || !valid_dtype(out_dtype))
    return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm: dtype %d / out dtype %d", dtype, out_dtype);
  if (M < 0 || N < 0 || d < 1 || k < 1 || k > d || ld_ai < k || ldb < N || ldy < N || M > kIntMax ||
      N > kIntMax || d > kIntMax)
    return fail(RMM_ERR_INVALID_ARG, "rmm_gemm: bad sizes");
  if (M == 0 || N == 0) return RMM_OK;
  if (!A_I || !B || !idx || !Y) return fail(RMM_ERR_INVALID_ARG, "rmm_gemm: null pointer");
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (dtype == RMM_F32) {
    if (out_dtype != RMM_F32) return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm: fp32 inputs need fp32 output");
    unsigned* err = device_error_word();
    if (!err) return RMM_ERR_CUDA;
    return from_cuda(launch_gemm_f32_simt(static_cast<const float*>(A_I), ld_ai, static_cast<const float*>(B), ldb,
                                          idx, d, M, N, k, static_cast<float*>(Y), ldy, err, s),
                     "rmm_gemm(f32): launch");
  }
  if (!aligned16(A_I) || !aligned16(B) || !aligned16(Y) || ld_ai % 8 || ldb % 8)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm(bf16): needs 16-byte aligned A_I/B/Y, ld_ai and ldb multiples of 8");
  if (((M + 127) / 128) * ((N + 255) / 256) > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm: too many tiles");
  const size_t need = rmm_gemm_workspace_size(dtype, N, k);
  if (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_gemm: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes, need);
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  if (M <= kGemvMaxM) {
    // a few rows: the kept rows of B are read in place (no gathered copy)
    const GemvPlan pl = gemv_plan(M, N, k, device_sm_count());
    if (pl.partial_bytes > ws_bytes)
      return fail(RMM_ERR_WORKSPACE, "rmm_gemm: workspace %zu < %zu bytes", ws_bytes, pl.partial_bytes);
    const cudaError_t e = launch_gemv(A_I, ld_ai, B, ldb, idx, M, d, N, k, pl, static_cast<float*>(ws), Y, out_dtype,
                                      ldy, err, s);
    return from_cuda(e, "rmm_gemm(bf16, few rows): launch");
  }
  const int64_t ld_bi = round_up(N, 8);
  cudaError_t e;
  if (fused_gather_supported(M, N, k, B, ldb, false)) {
    e = launch_fused_product(nullptr, 0, d, B, ldb, false, idx, k, const_cast<void*>(A_I), ld_ai, ws,
                             gemm_counters(ws, N, k), fused_gather_counter_words(N), M, N, Y, out_dtype, ldy, nullptr,
                             err, s);
    if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
    return from_cuda(e, "rmm_gemm(bf16): launch");
  }
  e = launch_gather_rows(B, d, N * 2, ldb * 2, idx, k, ws, ld_bi * 2, err, s);
  if (e != cudaSuccess) return from_cuda(e, "rmm_gemm: row gather launch");
  e = launch_gemm_bf16_tc(A_I, ld_ai, ws, ld_bi, M, N, k, Y, out_dtype, ldy, err, s);
  if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
  return from_cuda(e, "rmm_gemm(bf16): launch");
}

rmm_status rmm_gemm_compacted(const void* A_I, int64_t ld_ai, const void* B_I, int64_t ld_bi, int64_t M, int64_t N,
                              int64_t k, void* Y, int out_dtype, int64_t ldy, void* stream) {
  clear_error();
  if (!valid_dtype(out_dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm_compacted: out dtype %d", out_dtype);
  if (M < 0 || N < 0 || k < 1 || ld_ai < k || ld_bi < N || ldy < N || M > kIntMax || N > kIntMax || k > kIntMax)
    return fail(RMM_ERR_INVALID_ARG, "rmm_gemm_compacted: bad sizes");
  if (M == 0 || N == 0) return RMM_OK;
  if (!A_I || !B_I || !Y) return fail(RMM_ERR_INVALID_ARG, "rmm_gemm_compacted: null pointer");
  if (!aligned16(A_I) || !aligned16(B_I) || !aligned16(Y) || ld_ai % 8 || ld_bi % 8)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm_compacted: needs 16-byte aligned operands, ld_ai/ld_bi multiples of 8");
  if (((M + 127) / 128) * ((N + 255) / 256) > kIntMax)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm_compacted: too many tiles");
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  const cudaError_t e =
      launch_gemm_bf16_tc(A_I, ld_ai, B_I, ld_bi, M, N, k, Y, out_dtype, ldy, err, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
  return from_cuda(e, "rmm_gemm_compacted: launch");
}

size_t rmm_matmul_workspace_size(int dtype, int64_t M, int64_t d, int64_t N, double rho) {
  if (!valid_dtype(dtype) || M < 0 || d < 1 || N < 0) return 0;
  const MatmulWs w = matmul_ws(dtype, M, d, N, rho);
  return w.k < 1 ? 0 : w.total;
}

rmm_status rmm_matmul(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t M, int64_t d, int64_t N,
                      double rho, int dtype, void* Y, int out_dtype, int64_t ldy, int32_t* idx_out, float* ss_out,
                      void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(dtype) || !valid_dtype(out_dtype))
    return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul: dtype %d / out dtype %d", dtype, out_dtype);
  const int64_t k = k_from_rho_impl(rho, d);
  if (k < 1) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul: rho %g outside (0,1] or d < 1", rho);
  if (M < 0 || N < 0 || lda < d || ldb < N || ldy < N) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul: bad sizes");
  if (!A || !B || !Y) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul: null pointer");
  const MatmulWs w = matmul_ws(dtype, M, d, N, rho);
  if (!ws || ws_bytes < w.total || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_matmul: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes,
                w.total);
  char* base = static_cast<char*>(ws);
  float* ss = ss_out ? ss_out : reinterpret_cast<float*>(base + w.ss);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + w.idx);
  void* score_ws = base + w.score;
  void* ai = base + w.ai;
  if (dtype == RMM_BF16 && M > 0 && N > 0 && aligned16(B) && ldb % 8 == 0 && gemv_select_supported(A, M, d, lda, false)) {
    // up to 4 rows (decode): one launch whose CTAs each select the kept rows
    // and stream their share of them
    const GemvPlan pl = gemv_plan(M, N, k, device_sm_count());
    if (pl.partial_bytes <= w.total - w.bi) {
      unsigned* err = device_error_word();
      if (!err) return RMM_ERR_CUDA;
      return from_cuda(launch_gemv_select(A, lda, M, d, B, ldb, nullptr, N, k, pl, reinterpret_cast<float*>(base + w.bi),
                                          Y, out_dtype, ldy, idx, ss, err, static_cast<cudaStream_t>(stream)),
                       "rmm_matmul: fused decode launch");
    }
  }
  if (dtype == RMM_BF16 && M > 0 && N > 0 && select_rows_supported(M, d) && aligned16(B) && ldb % 8 == 0) {
    // a few rows (decode): scores, selection and A_I in one launch, then the
    // product that reads only the kept rows of B
    const cudaError_t e = launch_select_rows(A, M, d, lda, k, idx, ss, ai, w.ld_ai, static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return from_cuda(e, "rmm_matmul: row selection launch");
    return rmm_gemm(ai, w.ld_ai, B, ldb, idx, d, M, N, k, dtype, Y, out_dtype, ldy, base + w.bi, w.total - w.bi,
                    stream);
  }
  rmm_status st = rmm_score(A, dtype, 1, M, d, lda, 0, ss, d, 0, score_ws, score_workspace_bytes(dtype, 1, M, d), stream);
  if (st != RMM_OK) return st;
  st = rmm_topk(ss, 1, d, d, k, idx, k, stream);
  if (st != RMM_OK) return st;
  if (dtype == RMM_BF16 && fused_gather_supported(M, N, k, B, ldb, false)) {
    // A_I and the first columns of B_I in one launch, then the product, whose
    // spare warps copy the rest of B's kept rows while it multiplies
    if (!aligned16(Y)) return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul: needs a 16-byte aligned Y");
    if (((M + 127) / 128) * ((N + 255) / 256) > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul: too many tiles");
    unsigned* err = device_error_word();
    if (!err) return RMM_ERR_CUDA;
    cudaStream_t s = static_cast<cudaStream_t>(stream);
    void* bi = base + w.bi;
    const cudaError_t e = launch_fused_product(A, lda, d, B, ldb, false, idx, k, ai, w.ld_ai, bi,
                                               gemm_counters(bi, N, k), fused_gather_counter_words(N), M, N, Y,
                                               out_dtype, ldy, nullptr, err, s);
    if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
    return from_cuda(e, "rmm_matmul: launch");
  }
  if (dtype == RMM_BF16 && M > kGemvMaxM && N > 0 && aligned16(B) && ldb % 8 == 0) {
    // both reduced operands in one launch, then the dense product on them
    const int64_t ld_bi = round_up(N, 8);
    void* bi = base + w.bi;
    st = rmm_compact_gather(A, lda, B, ldb, M, d, N, idx, k, ai, w.ld_ai, bi, ld_bi, stream);
    if (st != RMM_OK) return st;
    return rmm_gemm_compacted(ai, w.ld_ai, bi, ld_bi, M, N, k, Y, out_dtype, ldy, stream);
  }
  st = rmm_compact(A, dtype, M, d, lda, idx, k, ai, w.ld_ai, stream);
  if (st != RMM_OK) return st;
  return rmm_gemm(ai, w.ld_ai, B, ldb, idx, d, M, N, k, dtype, Y, out_dtype, ldy, base + w.bi, w.total - w.bi,
                  stream);
}

size_t rmm_gemm_w8_workspace_size(int64_t N, int64_t k) { return rmm_gemm_workspace_size(RMM_BF16, N, k); }

rmm_status rmm_gemm_w8(const void* A_I, int64_t ld_ai, const int8_t* Bq, int64_t ldb, const float* b_scale,
                       const int32_t* idx, int64_t d, int64_t M, int64_t N, int64_t k, void* Y, int out_dtype,
                       int64_t ldy, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(out_dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm_w8: out dtype %d", out_dtype);
  if (M < 0 || N < 0 || d < 1 || k < 1 || k > d || ld_ai < k || ldb < N || ldy < N || M > kIntMax ||
      N > kIntMax || d > kIntMax)
    return fail(RMM_ERR_INVALID_ARG, "rmm_gemm_w8: bad sizes");
  if (M == 0 || N == 0) return RMM_OK;
  if (!A_I || !Bq || !b_scale || !idx || !Y) return fail(RMM_ERR_INVALID_ARG, "rmm_gemm_w8: null pointer");
  if (!aligned16(A_I) || !aligned16(Bq) || !aligned16(Y) || ld_ai % 8 || ldb % 16)
    return fail(RMM_ERR_UNSUPPORTED,
                "rmm_gemm_w8: needs 16-byte aligned A_I/Bq/Y, ld_ai a multiple of 8 and ldb of 16");
  if (((M + 127) / 128) * ((N + 255) / 256) > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm_w8: too many tiles");
  const size_t need = rmm_gemm_w8_workspace_size(N, k);
  if (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_gemm_w8: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes, need);
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M <= kGemvMaxM) {
    const GemvPlan pl = gemv_plan(M, N, k, device_sm_count());
    if (pl.partial_bytes > ws_bytes)
      return fail(RMM_ERR_WORKSPACE, "rmm_gemm_w8: workspace %zu < %zu bytes", ws_bytes, pl.partial_bytes);
    return from_cuda(launch_gemv(A_I, ld_ai, Bq, ldb, idx, M, d, N, k, pl, static_cast<float*>(ws), Y, out_dtype, ldy,
                                 err, s, b_scale),
                     "rmm_gemm_w8(few rows): launch");
  }
  const int64_t ld_bi = round_up(N, 8);
  cudaError_t e;
  if (fused_gather_supported(M, N, k, Bq, ldb, true)) {
    e = launch_fused_product(nullptr, 0, d, Bq, ldb, true, idx, k, const_cast<void*>(A_I), ld_ai, ws,
                             gemm_counters(ws, N, k), fused_gather_counter_words(N), M, N, Y, out_dtype, ldy, b_scale,
                             err, s);
    if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
    return from_cuda(e, "rmm_gemm_w8: launch");
  }
  e = launch_gather_rows_i8(Bq, d, N, ldb, idx, k, ws, ld_bi, err, s);
  if (e != cudaSuccess) return from_cuda(e, "rmm_gemm_w8: row gather launch");
  e = launch_gemm_bf16_tc(A_I, ld_ai, ws, ld_bi, M, N, k, Y, out_dtype, ldy, err, s, b_scale);
  if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
  return from_cuda(e, "rmm_gemm_w8: launch");
}

size_t rmm_matmul_w8_workspace_size(int64_t M, int64_t d, int64_t N, double rho) {
  return rmm_matmul_workspace_size(RMM_BF16, M, d, N, rho);
}

rmm_status rmm_matmul_w8(const void* A, int64_t lda, const int8_t* Bq, int64_t ldb, const float* b_scale, int64_t M,
                         int64_t d, int64_t N, double rho, void* Y, int out_dtype, int64_t ldy, int32_t* idx_out,
                         float* ss_out, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(out_dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_w8: out dtype %d", out_dtype);
  const int64_t k = k_from_rho_impl(rho, d);
  if (k < 1) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul_w8: rho %g outside (0,1] or d < 1", rho);
  if (M < 0 || N < 0 || lda < d || ldb < N || ldy < N) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul_w8: bad sizes");
  if (!A || !Bq || !b_scale || !Y) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul_w8: null pointer");
  if (!aligned16(Bq) || ldb % 16)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_w8: needs a 16-byte aligned Bq and ldb a multiple of 16");
  const MatmulWs w = matmul_ws(RMM_BF16, M, d, N, rho);
  if (!ws || ws_bytes < w.total || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_matmul_w8: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes,
                w.total);
  char* base = static_cast<char*>(ws);
  float* ss = ss_out ? ss_out : reinterpret_cast<float*>(base + w.ss);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + w.idx);
  void* ai = base + w.ai;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  if (M > 0 && N > 0 && aligned16(Bq) && ldb % 16 == 0 && b_scale && gemv_select_supported(A, M, d, lda, true)) {
    // up to 4 rows (decode): selection and product in one launch
    const GemvPlan pl = gemv_plan(M, N, k, device_sm_count());
    if (pl.partial_bytes <= w.total - w.bi) {
      unsigned* err = device_error_word();
      if (!err) return RMM_ERR_CUDA;
      return from_cuda(launch_gemv_select(A, lda, M, d, Bq, ldb, b_scale, N, k, pl,
                                          reinterpret_cast<float*>(base + w.bi), Y, out_dtype, ldy, idx, ss, err, s),
                       "rmm_matmul_w8: fused decode launch");
    }
  }
  if (M > 0 && N > 0 && select_rows_supported(M, d)) {
    const cudaError_t e = launch_select_rows(A, M, d, lda, k, idx, ss, ai, w.ld_ai, s);
    if (e != cudaSuccess) return from_cuda(e, "rmm_matmul_w8: row selection launch");
    return rmm_gemm_w8(ai, w.ld_ai, Bq, ldb, b_scale, idx, d, M, N, k, Y, out_dtype, ldy, base + w.bi,
                       w.total - w.bi, stream);
  }
  rmm_status st = rmm_score(A, RMM_BF16, 1, M, d, lda, 0, ss, d, 0, base + w.score,
                            score_workspace_bytes(RMM_BF16, 1, M, d), stream);
  if (st != RMM_OK) return st;
  st = rmm_topk(ss, 1, d, d, k, idx, k, stream);
  if (st != RMM_OK) return st;
  if (M > kGemvMaxM && N > 0) {
    // both reduced operands in one launch (the int8 rows widened to bf16),
    // then the tensor-core product with the column scales in its epilogue
    const int64_t ld_bi = round_up(N, 8);
    void* bi = base + w.bi;
    if (k + ((M + 7) / 8) * ((k + 63) / 64) > kIntMax) return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_w8: grid");
    if (((M + 127) / 128) * ((N + 255) / 256) > kIntMax)
      return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_w8: too many tiles");
    if (!aligned16(Y)) return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_w8: needs a 16-byte aligned Y");
    unsigned* err = device_error_word();
    if (!err) return RMM_ERR_CUDA;
    cudaError_t e;
    if (fused_gather_supported(M, N, k, Bq, ldb, true)) {
      // A_I and the first columns of B_I in one launch, then the product
      // with the rest of the int8 rows widened by its spare warps
      e = launch_fused_product(A, lda, d, Bq, ldb, true, idx, k, ai, w.ld_ai, bi, gemm_counters(bi, N, k),
                               fused_gather_counter_words(N), M, N, Y, out_dtype, ldy, b_scale, err, s);
      if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
      return from_cuda(e, "rmm_matmul_w8: launch");
    }
    e = launch_compact_and_gather(A, M, d, lda, Bq, N, ldb, idx, k, ai, w.ld_ai, bi, ld_bi, err, s, true);
    if (e != cudaSuccess) return from_cuda(e, "rmm_matmul_w8: compaction launch");
    e = launch_gemm_bf16_tc(ai, w.ld_ai, bi, ld_bi, M, N, k, Y, out_dtype, ldy, err, s, b_scale);
    if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
    return from_cuda(e, "rmm_matmul_w8: launch");
  }
  st = rmm_compact(A, RMM_BF16, M, d, lda, idx, k, ai, w.ld_ai, stream);
  if (st != RMM_OK) return st;
  return rmm_gemm_w8(ai, w.ld_ai, Bq, ldb, b_scale, idx, d, M, N, k, Y, out_dtype, ldy, base + w.bi, w.total - w.bi,
                     stream);
}

// ------------------------------------------------------------------ block driver

size_t rmm_silu_mul_score_workspace_size(int64_t M, int64_t N) {
  if (M < 0 || N < 1) return 0;
  return score_workspace_bytes(RMM_BF16, 1, M, N);
}

rmm_status rmm_silu_mul_score(const void* G, int64_t ldg, const void* U, int64_t ldu, int64_t M, int64_t N, void* H,
                              int64_t ldh, float* ss_out, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (M < 0 || N < 1 || ldg < N || ldu < N || ldh < N || M > kIntMax * 16)
    return fail(RMM_ERR_INVALID_ARG, "rmm_silu_mul_score: bad sizes");
  if (!G || !U || !H || !ss_out) return fail(RMM_ERR_INVALID_ARG, "rmm_silu_mul_score: null pointer");
  if (!aligned16(G) || !aligned16(U) || !aligned16(H) || ldg % 8 || ldu % 8 || ldh % 8)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_silu_mul_score: needs 16-byte aligned G/U/H and pitches multiples of 8");
  const size_t need = rmm_silu_mul_score_workspace_size(M, N);
  if (need && (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % kWsAlign))
    return fail(RMM_ERR_WORKSPACE, "rmm_silu_mul_score: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes,
                need);
  return from_cuda(launch_silu_mul_score(G, ldg, U, ldu, H, ldh, M, N, ss_out, ws, static_cast<cudaStream_t>(stream)),
                   "rmm_silu_mul_score: launch");
}

size_t rmm_matmul_multi_workspace_size(int64_t M, int64_t d, int64_t N_max, double rho) {
  return rmm_matmul_workspace_size(RMM_BF16, M, d, N_max, rho);
}

rmm_status rmm_matmul_multi(const void* A, int64_t lda, int64_t M, int64_t d, double rho, int nprod,
                            const void* const* B, const int64_t* ldb, const int64_t* N, void* const* Y,
                            const int64_t* ldy, int out_dtype, const float* ss_in, int32_t* idx_out, float* ss_out,
                            void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(out_dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_multi: out dtype %d", out_dtype);
  const int64_t k = k_from_rho_impl(rho, d);
  if (k < 1) return fail(RMM_ERR_INVALID_ARG, "rmm_matmul_multi: rho %g outside (0,1] or d < 1", rho);
  if (nprod < 1 || !B || !ldb || !N || !Y || !ldy || M < 0 || lda < d || !A)
    return fail(RMM_ERR_INVALID_ARG, "rmm_matmul_multi: bad arguments");
  int64_t nmax = 0;
  for (int i = 0; i < nprod; ++i) {
    if (!B[i] || !Y[i] || N[i] < 1 || ldb[i] < N[i] || ldy[i] < N[i])
      return fail(RMM_ERR_INVALID_ARG, "rmm_matmul_multi: bad product %d", i);
    if (!aligned16(B[i]) || ldb[i] % 8 || !aligned16(Y[i]))
      return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_multi: product %d needs 16-byte aligned B and Y, ldb % 8 == 0", i);
    nmax = std::max(nmax, N[i]);
  }
  const MatmulWs w = matmul_ws(RMM_BF16, M, d, nmax, rho);
  if (!ws || ws_bytes < w.total || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_matmul_multi: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes,
                w.total);
  char* base = static_cast<char*>(ws);
  float* ss = ss_out ? ss_out : reinterpret_cast<float*>(base + w.ss);
  int32_t* idx = idx_out ? idx_out : reinterpret_cast<int32_t*>(base + w.idx);
  void* ai = base + w.ai;
  void* bi = base + w.bi;
  const size_t bi_bytes = w.total - w.bi;
  cudaStream_t s = static_cast<cudaStream_t>(stream);
  rmm_status st = RMM_OK;
  bool compacted = false;
  if (M == 0) return RMM_OK;
  // one selection for every product
  if (ss_in) {
    st = rmm_topk(ss_in, 1, d, d, k, idx, k, stream);
  } else if (select_rows_supported(M, d)) {
    const cudaError_t e = launch_select_rows(A, M, d, lda, k, idx, ss, ai, w.ld_ai, s);
    if (e != cudaSuccess) return from_cuda(e, "rmm_matmul_multi: row selection launch");
    compacted = true;
  } else {
    st = rmm_score(A, RMM_BF16, 1, M, d, lda, 0, ss, d, 0, base + w.score, score_workspace_bytes(RMM_BF16, 1, M, d),
                   stream);
    if (st == RMM_OK) st = rmm_topk(ss, 1, d, d, k, idx, k, stream);
  }
  if (st != RMM_OK) return st;
  for (int i = 0; i < nprod; ++i) {
    if (M <= kGemvMaxM) {
      if (!compacted) {
        st = rmm_compact(A, RMM_BF16, M, d, lda, idx, k, ai, w.ld_ai, stream);
        if (st != RMM_OK) return st;
        compacted = true;
      }
      st = rmm_gemm(ai, w.ld_ai, B[i], ldb[i], idx, d, M, N[i], k, RMM_BF16, Y[i], out_dtype, ldy[i], bi, bi_bytes,
                    stream);
    } else if (fused_gather_supported(M, N[i], k, B[i], ldb[i], false)) {
      if (((M + 127) / 128) * ((N[i] + 255) / 256) > kIntMax)
        return fail(RMM_ERR_UNSUPPORTED, "rmm_matmul_multi: too many tiles");
      unsigned* err = device_error_word();
      if (!err) return RMM_ERR_CUDA;
      // A_I (first product only) and the first columns of this product's
      // B_I in one launch, then the product copying the rest
      const cudaError_t e = launch_fused_product(compacted ? nullptr : A, lda, d, B[i], ldb[i], false, idx, k, ai,
                                                 w.ld_ai, bi, gemm_counters(bi, nmax, k),
                                                 fused_gather_counter_words(nmax), M, N[i], Y[i], out_dtype, ldy[i],
                                                 nullptr, err, s);
      compacted = true;
      if (e == cudaErrorInvalidValue && !g_last_error.empty()) return RMM_ERR_CUDA;
      if (e != cudaSuccess) return from_cuda(e, "rmm_matmul_multi: product launch");
    } else {
      const int64_t ld_bi = round_up(N[i], 8);
      if (!compacted) {
        st = rmm_compact_gather(A, lda, B[i], ldb[i], M, d, N[i], idx, k, ai, w.ld_ai, bi, ld_bi, stream);
        compacted = true;
      } else {
        st = rmm_gather_rows(B[i], RMM_BF16, d, N[i], ldb[i], idx, k, bi, ld_bi, stream);
      }
      if (st == RMM_OK) st = rmm_gemm_compacted(ai, w.ld_ai, bi, ld_bi, M, N[i], k, Y[i], out_dtype, ldy[i], stream);
    }
    if (st != RMM_OK) return st;
  }
  return RMM_OK;
}


size_t rmm_mlp_block_workspace_size(int64_t M, int64_t d_model, int64_t d_ff, double rho_up, double rho_down) {
  if (M < 1 || d_model < 1 || d_ff < 1 || k_from_rho_impl(rho_up, d_model) < 1 || k_from_rho_impl(rho_down, d_ff) < 1)
    return 0;
  return mlp_ws(M, d_model, d_ff, rho_up, rho_down).total;
}

rmm_status rmm_mlp_block(const void* X, int64_t ldx, int64_t M, int64_t d_model, int64_t d_ff, const void* W_up,
                         int64_t ld_up, const void* W_gate, int64_t ld_gate, const void* W_down, int64_t ld_down,
                         double rho_up, double rho_down, void* Y, int out_dtype, int64_t ldy, int32_t* idx_up,
                         int32_t* idx_down, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (M < 1 || d_model < 1 || d_ff < 1 || !X || !W_up || !W_gate || !W_down || !Y)
    return fail(RMM_ERR_INVALID_ARG, "rmm_mlp_block: bad arguments");
  if (k_from_rho_impl(rho_up, d_model) < 1 || k_from_rho_impl(rho_down, d_ff) < 1)
    return fail(RMM_ERR_INVALID_ARG, "rmm_mlp_block: rho outside (0,1]");
  const MlpWs w = mlp_ws(M, d_model, d_ff, rho_up, rho_down);
  if (!ws || ws_bytes < w.total || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_mlp_block: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes,
                w.total);
  char* base = static_cast<char*>(ws);
  void* U = base + w.u;
  void* G = base + w.g;
  void* H = base + w.h;
  float* ssH = reinterpret_cast<float*>(base + w.ss);
  void* inner = base + w.inner;
  const size_t inner_bytes = w.total - w.inner;
  // up and gate: one selection on X for both
  const void* Bs[2] = {W_up, W_gate};
  const int64_t ldbs[2] = {ld_up, ld_gate};
  const int64_t Ns[2] = {d_ff, d_ff};
  void* Ys[2] = {U, G};
  const int64_t ldys[2] = {w.ld_ff, w.ld_ff};
  rmm_status st = rmm_matmul_multi(X, ldx, M, d_model, rho_up, 2, Bs, ldbs, Ns, Ys, ldys, RMM_BF16, nullptr, idx_up,
                                   nullptr, inner, inner_bytes, stream);
  if (st != RMM_OK) return st;
  // H = SiLU(G) * U with the down projection's column scores in the same pass
  st = rmm_silu_mul_score(G, w.ld_ff, U, w.ld_ff, M, d_ff, H, w.ld_ff, ssH, inner, inner_bytes, stream);
  if (st != RMM_OK) return st;
  // down: selection from the fused scores
  const void* Bd[1] = {W_down};
  const int64_t ldbd[1] = {ld_down};
  const int64_t Nd[1] = {d_model};
  void* Yd[1] = {Y};
  const int64_t ldyd[1] = {ldy};
  return rmm_matmul_multi(H, w.ld_ff, M, d_ff, rho_down, 1, Bd, ldbd, Nd, Yd, ldyd, out_dtype, ssH, idx_down, nullptr,
                          inner, inner_bytes, stream);
}

size_t rmm_decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t L, int64_t D, double rho_t,
                                           int with_logits, int with_idx_t) {
  const int64_t kt = k_from_rho_impl(rho_t, L);
  if (B < 1 || Hq < 1 || kt < 1 || (D != 64 && D != 128)) return 0;
  return decode_attention_workspace_bytes(B, Hq, L, D, kt, !with_logits, !with_idx_t);
}

rmm_status rmm_decode_attention(const void* q, const void* K, const void* V, int64_t B, int64_t Hq, int64_t Hkv,
                                int64_t L, int64_t Lmax, int64_t D, double rho_d, double rho_t, float scale, void* O,
                                int out_dtype, int32_t* idx_d, int32_t* idx_t, float* lse, float* logits, void* ws,
                                size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(out_dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_decode_attention: out dtype %d", out_dtype);
  if (B < 1 || Hq < 1 || Hkv < 1 || L < 1 || Lmax < L || Hq % Hkv)
    return fail(RMM_ERR_INVALID_ARG, "rmm_decode_attention: bad sizes");
  if (D != 64 && D != 128) return fail(RMM_ERR_UNSUPPORTED, "rmm_decode_attention: D must be 64 or 128");
  if (!decode_attention_group_supported(Hq / Hkv))
    return fail(RMM_ERR_UNSUPPORTED, "rmm_decode_attention: q-heads per kv-head must be 1, 2, 4, 8 or 16");
  if (B * Hq > 65535 || B * Hkv > 65535 || B * Hq * L > kIntMax || B * Hkv * Lmax * D > (int64_t{1} << 40) ||
      Lmax > kIntMax)
    return fail(RMM_ERR_UNSUPPORTED, "rmm_decode_attention: sizes beyond the kernels' grid");
  const int64_t kd = k_from_rho_impl(rho_d, D), kt = k_from_rho_impl(rho_t, L);
  if (kd < 1 || kt < 1) return fail(RMM_ERR_INVALID_ARG, "rmm_decode_attention: rho outside (0,1]");
  if (!q || !K || !V || !O) return fail(RMM_ERR_INVALID_ARG, "rmm_decode_attention: null pointer");
  if (!aligned16(q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(RMM_ERR_UNSUPPORTED, "rmm_decode_attention: q, K, V and O must be 16-byte aligned");
  const size_t need = decode_attention_workspace_bytes(B, Hq, L, D, kt, logits == nullptr, idx_t == nullptr);
  if (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_decode_attention: workspace %zu < %zu bytes or not 256-byte aligned",
                ws_bytes, need);
  const float sc = scale > 0.f ? scale : static_cast<float>(1.0 / std::sqrt(static_cast<double>(D)));
  const cudaError_t e = launch_decode_attention(q, K, V, B, Hq, Hkv, L, Lmax, D, kd, kt, sc, O, out_dtype, idx_d,
                                                idx_t, lse, logits, ws, static_cast<cudaStream_t>(stream));
  return from_cuda(e, "rmm_decode_attention: launch");
}

size_t rmm_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S, int64_t D, double rho_d,
                                    double rho_t) {
  const int64_t kd = k_from_rho_impl(rho_d, D), kt = k_from_rho_impl(rho_t, S);
  if (kd < 1 || kt < 1 || B < 1 || Hq < 1 || Hkv < 1) return 0;
  return attention_workspace_bytes(B, Hq, Hkv, S, D, kd, kt);
}

rmm_status rmm_attention(const void* Q, const void* K, const void* V, int64_t B, int64_t Hq, int64_t Hkv, int64_t S,
                         int64_t D, double rho_d, double rho_t, float scale, void* O, int out_dtype, int32_t* idx_d,
                         int32_t* idx_t, float* lse, float* tscore, void* ws, size_t ws_bytes, void* stream) {
  clear_error();
  if (!valid_dtype(out_dtype)) return fail(RMM_ERR_UNSUPPORTED, "rmm_attention: out dtype %d", out_dtype);
  if (!Q || !K || !V || !O) return fail(RMM_ERR_INVALID_ARG, "rmm_attention: null pointer");
  if (B < 1 || Hq < 1 || Hkv < 1 || Hq % Hkv || S < 1 || S > 65535LL * 128 || B * Hq > 65535)
    return fail(RMM_ERR_INVALID_ARG, "rmm_attention: bad sizes");
  if (D != 64 && D != 128) return fail(RMM_ERR_UNSUPPORTED, "rmm_attention: head_dim %lld (64 or 128 only)", (long long)D);
  const int64_t kd = k_from_rho_impl(rho_d, D), kt = k_from_rho_impl(rho_t, S);
  if (kd < 1 || kt < 1) return fail(RMM_ERR_INVALID_ARG, "rmm_attention: rho outside (0,1]");
  if (!aligned16(Q) || !aligned16(K) || !aligned16(V) || !aligned16(O))
    return fail(RMM_ERR_UNSUPPORTED, "rmm_attention: tensors must be 16-byte aligned");
  const size_t need = attention_workspace_bytes(B, Hq, Hkv, S, D, kd, kt);
  if (!ws || ws_bytes < need || reinterpret_cast<uintptr_t>(ws) % kWsAlign)
    return fail(RMM_ERR_WORKSPACE, "rmm_attention: workspace %zu < %zu bytes or not 256-byte aligned", ws_bytes,
                need);
  unsigned* err = device_error_word();
  if (!err) return RMM_ERR_CUDA;
  if (!(scale > 0.f)) scale = 1.0f / std::sqrt(static_cast<float>(D));
  const cudaError_t e = launch_attention(Q, K, V, B, Hq, Hkv, S, D, kd, kt, scale, O, out_dtype, idx_d, idx_t, lse,
                                         tscore, ws, err, static_cast<cudaStream_t>(stream));
  if (e == cudaErrorNotSupported) return fail(RMM_ERR_UNSUPPORTED, "rmm_attention: %s", g_last_error.c_str());
  return from_cuda(e, "rmm_attention: launch");
}

}  // extern "C"
