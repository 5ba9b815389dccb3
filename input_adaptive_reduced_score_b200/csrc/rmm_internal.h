// rmm_internal.h — host-side declarations shared by the librmm translation
// units (launchers, error reporting, device queries).  Not part of the ABI.
#pragma once

#include <cuda_runtime.h>

#include <cstddef>
#include <cstdint>

namespace rmm {

// Thread-local error message for rmm_last_error().
void set_error(const char* fmt, ...);
void clear_error();

// Device address of the current device's error word (nullptr on failure;
// the message is set).
unsigned* device_error_word();

// Streaming multiprocessor count of the current device (0 on failure).
int device_sm_count();

constexpr size_t kWsAlign = 256;
inline size_t align_up(size_t x, size_t a) { return (x + a - 1) / a * a; }

// ---- score (rmm_score.cu)
struct ScorePlan {
  int vec;          // elements per 16-byte vector
  int col_threads;  // threads across columns in a CTA (power of two <= 64)
  int row_groups;   // 256 / col_threads
  int64_t strips;   // column strips
  int64_t splits;   // row splits
  int64_t rows_per_split;
};
ScorePlan score_plan(int dtype, int64_t batch, int64_t M, int64_t d);
size_t score_workspace_bytes(int dtype, int64_t batch, int64_t M, int64_t d);
// Bytes of partial sums launch_score will actually write for this call: 0 when
// the one-launch kernel serves it (bf16 with 16-byte aligned base, pitch and
// batch stride) or M == 0, else score_workspace_bytes.
size_t score_workspace_used(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                            int64_t batch_stride);
cudaError_t launch_score(const void* A, int dtype, int64_t batch, int64_t M, int64_t d, int64_t lda,
                         int64_t batch_stride, float* ss, int64_t ld_ss, int sqrt_out, void* ws,
                         cudaStream_t stream);

// H = bf16(SiLU(G) * U) and ss_j = sum_i H[i,j]^2 in one pass over [M x d]
// bf16 G, U, H (16-byte aligned, pitches multiples of 8); the workspace holds
// score_workspace_bytes(1, 1, M, d) bytes of row-split partials.
cudaError_t launch_silu_mul_score(const void* G, int64_t ldg, const void* U, int64_t ldu, void* H, int64_t ldh,
                                  int64_t M, int64_t d, float* ss, void* ws, cudaStream_t stream);

// ---- top-k (rmm_topk.cu)
// CTAs per row of the top-k search (0: the row is too long to stage; it
// takes the radix pass), and the keys each CTA of such a cluster stages.
int topk_cluster_size(int64_t batch, int64_t d);
int topk_cluster_slice(int64_t d, int c);
cudaError_t launch_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k,
                        int32_t* idx, int64_t ld_idx, cudaStream_t stream);

// A few bf16 activation rows: scores, top-k and A_I = A[:, idx] in one launch
// (M <= 16, d <= 51200; A_I gets ld_ai >= k).  ss may be null.
bool select_rows_supported(int64_t M, int64_t d);
cudaError_t launch_select_rows(const void* A, int64_t M, int64_t d, int64_t lda, int64_t k, int32_t* idx, float* ss,
                               void* A_I, int64_t ld_ai, cudaStream_t stream);

// ---- compaction (rmm_compact.cu)
cudaError_t launch_compact(const void* A, int dtype, int64_t M, int64_t d, int64_t lda,
                           const int32_t* idx, int64_t k, void* A_I, int64_t ld_ai, unsigned* err,
                           cudaStream_t stream);

// Row gather B_I[r, :] = B[idx[r], :]; bases and pitches 16-byte aligned,
// row_bytes even (checked by the caller).
cudaError_t launch_gather_rows(const void* B, int64_t d, int64_t row_bytes, int64_t ldb_bytes, const int32_t* idx,
                               int64_t k, void* B_I, int64_t ldbi_bytes, unsigned* err, cudaStream_t stream);

// Both reduced operands in one launch (bf16 A): A_I = A[:, idx] and
// B_I = B[idx, :]; B, B_I bases and pitches 16-byte aligned.  b_int8: B is
// int8 [d x N] (ldb in bytes, a multiple of 16) and B_I is written as bf16.
// With M = 0 it is the row gather alone.  zero / n_zero (optional): words the
// launch sets to zero after waiting for its predecessor (the counters of a
// fused row gather).
cudaError_t launch_compact_and_gather(const void* A, int64_t M, int64_t d, int64_t lda, const void* B, int64_t N,
                                      int64_t ldb, const int32_t* idx, int64_t k, void* A_I, int64_t ld_ai,
                                      void* B_I, int64_t ld_bi, unsigned* err, cudaStream_t stream,
                                      bool b_int8 = false, uint32_t* zero = nullptr, int64_t n_zero = 0);

// Row gather of an int8 B [d x N] (ldb bytes, multiple of 16; 16-byte aligned)
// into bf16 B_I [k x N] (ld_bi elements, multiple of 8; 16-byte aligned).
cudaError_t launch_gather_rows_i8(const void* Bq, int64_t d, int64_t N, int64_t ldb, const int32_t* idx, int64_t k,
                                  void* B_I, int64_t ld_bi, unsigned* err, cudaStream_t stream);

// ---- reduced GEMM (rmm_gemm_tc.cu, rmm_gemm_simt.cu)
// Returns cudaSuccess or an error; on a driver error in tensor-map encoding
// the message is set and cudaErrorInvalidValue returned.
// Dense tcgen05 GEMM on the compacted operands: Y = A_I [M x k] · B_I [k x N].
// col_scale (may be null): fp32 [N], multiplies column n of the product
// before it is stored (the per-column scales of an int8 weight).
//
// Fused row gather (CTA-pair kernel, M >= 256): with `fg` the kernel itself
// fills columns [n_ready, N) of B_I = B[idx, :] (bf16, or int8 widened to
// exact bf16) while it multiplies: extra warps copy 16-row x 256-column units
// taken from a ticket counter and count finished units per 256-column block;
// a tile's loads of B_I wait for its block.  Columns [0, n_ready) must be in
// place before the launch: fused_gather_first_cols(M, N) is what the first
// wave of tiles reads, so that wave never waits.  fg->ctr holds
// fused_gather_counter_words(N) words that must be zero when the kernel
// starts.  With n_ready >= N the plain kernel runs.
struct FusedGather {
  const void* B;        // [d x N], row pitch ldb elements, rows 16-byte aligned
  int64_t ldb;
  const int32_t* idx;   // the k kept rows
  int64_t d;
  uint32_t* ctr;
  bool b_int8;
  int64_t n_ready;      // a multiple of 256, or N
};
int64_t fused_gather_counter_words(int64_t N);
int64_t fused_gather_first_cols(int64_t M, int64_t N);
// The fused gather applies: M >= 256, N a multiple of 8, B 16-byte aligned
// with a 16-byte multiple row pitch, and the unit count fits 31 bits.
bool fused_gather_supported(int64_t M, int64_t N, int64_t k, const void* B, int64_t ldb, bool b_int8);
cudaError_t launch_gemm_bf16_tc(const void* A_I, int64_t ld_ai, const void* B_I, int64_t ld_bi, int64_t M,
                                int64_t N, int64_t k, void* Y, int out_dtype, int64_t ldy, unsigned* err,
                                cudaStream_t stream, const float* col_scale = nullptr,
                                const FusedGather* fg = nullptr);
cudaError_t launch_gemm_f32_simt(const float* A_I, int64_t ld_ai, const float* B, int64_t ldb,
                                 const int32_t* idx, int64_t d, int64_t M, int64_t N, int64_t k,
                                 float* Y, int64_t ldy, unsigned* err, cudaStream_t stream);

// ---- reduced product for M <= 16 rows (rmm_gemv.cu): kept rows of B read in place
constexpr int64_t kGemvMaxM = 16;
struct GemvPlan {
  int64_t slices;        // column slices of 128
  int splits;            // kept-row ranges
  int rows_per_split;
  bool clustered;        // the splits of a column slice form one cluster (no partials in memory)
  size_t partial_bytes;  // fp32 partial sums in global memory (0 with one split or a cluster)
};
GemvPlan gemv_plan(int64_t M, int64_t N, int64_t k, int sms);
// A_I bf16 [M x k] (ld_ai), B bf16 [d x N] (ldb, rows 16-byte aligned), idx [k].
// b_scale non-null: B is int8 (ldb bytes, rows 16-byte aligned) and column n
// of the product is multiplied by b_scale[n].
cudaError_t launch_gemv(const void* A_I, int64_t ld_ai, const void* B, int64_t ldb, const int32_t* idx, int64_t M,
                        int64_t d, int64_t N, int64_t k, const GemvPlan& plan, float* partial, void* Y, int out_dtype,
                        int64_t ldy, unsigned* err, cudaStream_t stream, const float* b_scale = nullptr);
// The same product with the selection inside it (M <= 16): every CTA scores
// X [M x d] bf16 (16-byte aligned rows, d a multiple of 8), selects the k
// kept indices and streams its share of their rows of B; idx_out receives the
// ascending index list and ss_out (may be null) the scores.
bool gemv_select_supported(const void* X, int64_t M, int64_t d, int64_t ldx, bool b_int8);
cudaError_t launch_gemv_select(const void* X, int64_t ldx, int64_t M, int64_t d, const void* B, int64_t ldb,
                               const float* b_scale, int64_t N, int64_t k, const GemvPlan& plan, float* partial,
                               void* Y, int out_dtype, int64_t ldy, int32_t* idx_out, float* ss_out, unsigned* err,
                               cudaStream_t stream);

// ---- reduced attention (rmm_attention.cu)
size_t attention_workspace_bytes(int64_t B, int64_t Hq, int64_t Hkv, int64_t S, int64_t D, int64_t kd,
                                 int64_t kt);
cudaError_t launch_attention(const void* Q, const void* K, const void* V, int64_t B, int64_t Hq,
                             int64_t Hkv, int64_t S, int64_t D, int64_t kd, int64_t kt, float scale,
                             void* O, int out_dtype, int32_t* idx_d, int32_t* idx_t, float* lse,
                             float* tscore, void* ws, unsigned* err, cudaStream_t stream);

// ---- reduced decode attention (rmm_decode_attention.cu)
// own_logits / own_idx: the logits buffer [B*Hq, L] / token index buffer
// [B*Hq, kt] live in the workspace (the caller did not pass them).
bool decode_attention_group_supported(int64_t G);  // q-heads per kv-head: 1, 2, 4, 8 or 16
size_t decode_attention_workspace_bytes(int64_t B, int64_t Hq, int64_t L, int64_t D, int64_t kt, bool own_logits,
                                        bool own_idx);
cudaError_t launch_decode_attention(const void* q, const void* K, const void* V, int64_t B, int64_t Hq, int64_t Hkv,
                                    int64_t L, int64_t Lmax, int64_t D, int64_t kd, int64_t kt, float scale, void* O,
                                    int out_dtype, int32_t* idx_d, int32_t* idx_t, float* lse, float* logits,
                                    void* ws, cudaStream_t stream);

}  // namespace rmm
