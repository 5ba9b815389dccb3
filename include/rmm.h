/*
 * rmm.h — C ABI of librmm, a B200 (sm_100a) implementation of Reduced Matrix
 * Multiplication (RMM).
 *
 * Source page: "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
 * Reduction for LLM Inference" (technical summary; section names are those of
 * its Spanish edition).  RMM replaces a product Y = AB (A the activation, B a
 * weight or intermediate representation; Metodología) by A[:,I] B[I,:], where
 * I holds the k = ceil(rho d) contraction indices with the largest activation
 * column norms s_j = ||A[:,j]||_2 (Metodología › Mecanismo Central,
 * Estrategia de Selección).  It applies to linear projections XW, to QK^T
 * along head_dim and to PV along the token dimension (Metodología › Alcance
 * de Aplicación).
 *
 * Conventions shared by every entry point
 *  - Every data pointer is a caller-owned DEVICE pointer on the current CUDA
 *    device; the library never allocates, frees or retains memory (except
 *    the self-test rmm_selftest_timeout, which documents its own).  Scratch
 *    space ("workspace") is passed in by the caller; its size comes from the
 *    matching *_workspace_size query.  A NULL workspace with ws_bytes == 0 is
 *    allowed when the query returns 0.
 *  - Matrices are row-major with an explicit leading dimension in ELEMENTS
 *    (ld >= number of columns).  Indices are int32.
 *  - `stream` is a cudaStream_t (NULL = legacy default stream).  All work is
 *    enqueued asynchronously on it; no call synchronises unless stated.
 *  - Every call validates its arguments on the host before launching and
 *    returns an rmm_status; on failure nothing was launched and
 *    rmm_last_error() gives a message (per host thread).
 *  - Errors found on the device (an index outside [0, d), a bounded wait that
 *    ran out) are recorded in a per-device error word and reported by
 *    rmm_device_error(), which synchronises the stream.  Kernels never trap.
 *  - dtype codes: RMM_F32 (fp32) or RMM_BF16 (bf16 stored as 16-bit words).
 *    bf16 products accumulate in fp32.
 */
#ifndef RMM_H_
#define RMM_H_

#include <stddef.h>
#include <stdint.h>

#if defined(__GNUC__)
#define RMM_API __attribute__((visibility("default")))
#else
#define RMM_API
#endif

#ifdef __cplusplus
extern "C" {
#endif

typedef enum rmm_status {
  RMM_OK = 0,
  RMM_ERR_INVALID_ARG = 1,   /* null pointer, bad size, rho outside (0,1], k outside [1,d] */
  RMM_ERR_UNSUPPORTED = 2,   /* dtype, alignment or shape the kernels do not take */
  RMM_ERR_WORKSPACE = 3,     /* workspace missing or smaller than the query's size */
  RMM_ERR_CUDA = 4,          /* a CUDA runtime/driver call failed */
  RMM_ERR_DEVICE = 5         /* rmm_device_error() found a device-side error */
} rmm_status;

typedef enum rmm_dtype { RMM_F32 = 0, RMM_BF16 = 1 } rmm_dtype;

/* Device-side error codes stored in the error word (0 = none). */
#define RMM_DEVERR_BAD_INDEX 1u        /* an index outside [0, d) was read; its row/column was zero-filled */
#define RMM_DEVERR_FP16_RANGE 2u       /* rmm_attention: a kept value of V beyond fp16's range (|v| > 65504 or NaN)
                                          was saturated for the reduced P V product */
#define RMM_DEVERR_TIMEOUT_BASE 0x100u /* + site: a bounded wait ran out and the kernel returned early */

/* ABI version of this header (incremented on any incompatible change). */
#define RMM_ABI_VERSION 1
RMM_API int rmm_abi_version(void);

/* Message describing the last failing call on this host thread ("" if none).
 * The pointer stays valid until the next rmm_* call on this thread. */
RMM_API const char* rmm_last_error(void);

/* k = ceil(rho * d) (Metodología › Estrategia de Selección), computed in fp64
 * with a guard of 1e-9*d against representation error (0.3*10 gives 3) and
 * clamped to [1, d].  Returns -1 when rho is not in (0, 1] or d < 1. */
RMM_API int64_t rmm_k_from_rho(double rho, int64_t d);

/* Synchronises `stream`, then reads the current device's error word into
 * *code (may be NULL); clears it when `clear` != 0.  Returns RMM_ERR_DEVICE
 * when the word was non-zero, RMM_ERR_CUDA if the sync failed. */
RMM_API rmm_status rmm_device_error(void* stream, int clear, unsigned* code);

/* ------------------------------------------------------------------ score
 * Column scores of `batch` activation matrices (Metodología › Estrategia de
 * Selección): ss[b*ld_ss + j] = sum_i A_b[i,j]^2, with A_b = A + b*batch_stride
 * (elements) an [M x d] row-major matrix of leading dimension lda.  Squares
 * are exact in fp32; the sum is an fp32 tree in a fixed order, so results are
 * deterministic for a given shape.  With sqrt_out != 0 the output is
 * s_j = sqrt(ss_j) instead (the page's norm; ranking is identical, but the
 * square root can merge distinct scores, so rmm_topk should be given ss).
 * Layout: lda >= d; for the vectorised path A and lda*elt must be 16-byte
 * aligned (otherwise a scalar path runs).  Workspace: rmm_score_workspace_size
 * bytes (fp32 partial sums of the row splits; 0 when one split suffices), an
 * upper bound that depends on the shape only.  Calls that take the one-launch
 * path (bf16 with A, lda*2 and, for batch > 1, batch_stride*2 all multiples
 * of 16 bytes) write no partial sums and accept ws = NULL, ws_bytes = 0.
 * M == 0 gives all-zero scores. */
RMM_API size_t rmm_score_workspace_size(int dtype, int64_t batch, int64_t M, int64_t d);
RMM_API rmm_status rmm_score(const void* A, int dtype, int64_t batch, int64_t M, int64_t d,
                     int64_t lda, int64_t batch_stride, float* ss, int64_t ld_ss,
                     int sqrt_out, void* ws, size_t ws_bytes, void* stream);

/* rmm_score for callers that cannot allocate device memory: an inference-
 * engine plugin handed only its input and output buffers, or a process whose
 * device memory is all reserved up front by an external pool (where an extra
 * cudaMalloc fails, and synchronises the device even when it succeeds).  The
 * paper has no counterpart; this is a library-side convenience.
 * Same arguments and result as rmm_score, minus the workspace, and bit-equal
 * to it (same kernels, same summation order).  Inputs that rmm_score serves
 * with its one-launch kernel (bf16 with 16-byte aligned base, row pitch and
 * batch stride) need no scratch.  The others (fp32 activations, bf16 with an
 * unaligned base, pitch or batch stride) keep their row-split partial sums in
 * a fixed array of RMM_SCORE_NOALLOC_MAX_BYTES inside the library, which every
 * GPU that loads the library holds until exit; such a call whose partial sums
 * need more (rmm_score_workspace_size above the limit) is rejected with
 * RMM_ERR_INVALID_ARG and a message, before any device work.  The first call
 * in each CUDA context of a device looks up the array's device address
 * (cudaGetSymbolAddress, with that device current), so make that first call
 * before any stream capture, and again after a device reset (the new context
 * repeats the look-up).  No call allocates or frees memory.  All calls share
 * the array and each call overwrites the part it reads before reading it, so
 * nothing has to be cleared between calls; calls that overlap on the GPU
 * race on it and must be serialised by the caller. */
#define RMM_SCORE_NOALLOC_MAX_BYTES ((size_t)16 << 20)
RMM_API rmm_status rmm_score_noalloc(const void* A, int dtype, int64_t batch, int64_t M, int64_t d,
                                     int64_t lda, int64_t batch_stride, float* ss, int64_t ld_ss,
                                     int sqrt_out, void* stream);

/* ------------------------------------------------------------------ top-k
 * For each of `batch` score rows (row b at scores + b*ld_s, length d), writes
 * the k indices with the largest scores to idx + b*ld_idx, in ascending index
 * order; equal scores are taken lowest index first (Metodología › Estrategia
 * de Selección keeps the top-k; the tie rule and the order are this library's
 * reading).  Scores must be finite; -0.0 ranks equal to +0.0.  The selection
 * is exact on the fp32 bit patterns (a histogram search over the key range,
 * by one CTA or a cluster of up to eight per row, or a radix select for rows
 * longer than 409600), so the index set is the unique one defined by that
 * rule.  1 <= k <= d, ld_idx >= k, ld_s >= d.  */
RMM_API rmm_status rmm_topk(const float* scores, int64_t batch, int64_t d, int64_t ld_s, int64_t k,
                    int32_t* idx, int64_t ld_idx, void* stream);

/* ------------------------------------------------------------------ compaction
 * A_I[i, r] = A[i, idx[r]] for r < k (Metodología › Mecanismo Central: the
 * reduced operand A_{:,I}).  A is [M x d] (lda), A_I is [M x k] (ld_ai >= k).
 * Columns k..ld_ai-1 of A_I are not written.  Indices outside [0, d) are
 * replaced by zero and flagged in the device error word. */
RMM_API rmm_status rmm_compact(const void* A, int dtype, int64_t M, int64_t d, int64_t lda,
                       const int32_t* idx, int64_t k, void* A_I, int64_t ld_ai, void* stream);

/* ------------------------------------------------------------------ row gather
 * B_I[r, :] = B[idx[r], :] for r < k (Metodología › Mecanismo Central: the
 * reduced operand B_{I,:}).  B is [d x N] (ldb), B_I is [k x N] (ld_bi).
 * Rows are copied whole with 16-byte accesses: B, B_I and the row pitches in
 * bytes must be 16-byte aligned (RMM_ERR_UNSUPPORTED otherwise).  Indices outside [0, d) give a zero row
 * and are flagged in the device error word. */
RMM_API rmm_status rmm_gather_rows(const void* B, int dtype, int64_t d, int64_t N, int64_t ldb,
                                   const int32_t* idx, int64_t k, void* B_I, int64_t ld_bi, void* stream);

/* ------------------------------------------------------------------ both reduced operands
 * A_I = A[:, idx] and B_I = B[idx, :] in one launch (bf16 only): the same
 * results as rmm_compact followed by rmm_gather_rows, with the two copies
 * overlapped (Metodología › Mecanismo Central: both operands of the reduced
 * product are restricted to I).  A [M x d] (lda), B [d x N] (ldb), A_I
 * [M x k] (ld_ai >= k), B_I [k x N] (ld_bi >= N).  B, B_I 16-byte aligned and
 * ldb, ld_bi multiples of 8 (RMM_ERR_UNSUPPORTED otherwise).  Indices outside
 * [0, d) give zeros and are flagged in the device error word. */
RMM_API rmm_status rmm_compact_gather(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t M,
                                      int64_t d, int64_t N, const int32_t* idx, int64_t k, void* A_I,
                                      int64_t ld_ai, void* B_I, int64_t ld_bi, void* stream);

/* ------------------------------------------------------------------ reduced GEMM
 * Y = A_I · B[idx, :]  (Metodología › Mecanismo Central), where A_I is the
 * compacted [M x k] activation (ld_ai), B the full [d x N] row-major operand
 * (ldb >= N) whose rows idx[0..k) are the kept contraction indices, and Y is
 * [M x N] (ldy >= N) written as out_dtype (RMM_BF16 or RMM_F32).
 *  - dtype RMM_BF16, M > 16: B's kept rows are copied into workspace (B_I),
 *    and a persistent tcgen05 tensor-core kernel computes A_I · B_I with fp32
 *    accumulation in tensor memory.  From M = 256 on, with N a multiple of 8,
 *    the copy runs inside the product's kernel: spare warps copy blocks of
 *    kept rows while the tensor cores work on blocks already copied.  Below
 *    that, one streaming gather launch precedes the product.
 *  - dtype RMM_BF16, M <= 16 (decode): the kept rows of B are read in place,
 *    once each, by a row-streaming kernel with fp32 accumulation; the
 *    workspace holds fp32 partial sums over ranges of kept rows, added in a
 *    fixed order.
 *    Both bf16 forms require 16-byte aligned A_I, B, Y, and ld_ai, ldb
 *    multiples of 8 (RMM_ERR_UNSUPPORTED otherwise).  B must be finite.
 *  - dtype RMM_F32: fp32 FMA kernel (A_I, B fp32; Y fp32 only); no workspace.
 * Workspace: rmm_gemm_workspace_size(dtype, N, k) bytes, 256-byte aligned
 * (B_I, then the fused copy's counters, which the call zeroes itself).
 * Out-of-range indices contribute zero and are flagged.  k >= 1. */
RMM_API size_t rmm_gemm_workspace_size(int dtype, int64_t N, int64_t k);
RMM_API rmm_status rmm_gemm(const void* A_I, int64_t ld_ai, const void* B, int64_t ldb,
                            const int32_t* idx, int64_t d, int64_t M, int64_t N, int64_t k,
                            int dtype, void* Y, int out_dtype, int64_t ldy,
                            void* ws, size_t ws_bytes, void* stream);

/* Y = A_I · B_I on already-compacted bf16 operands: A_I [M x k] (ld_ai) and
 * B_I [k x N] (ld_bi), i.e. the tensor-core stage of rmm_gemm without its row
 * gather (Metodología › Mecanismo Central).  16-byte aligned A_I, B_I, Y;
 * ld_ai, ld_bi multiples of 8.  No workspace. */
RMM_API rmm_status rmm_gemm_compacted(const void* A_I, int64_t ld_ai, const void* B_I, int64_t ld_bi,
                                      int64_t M, int64_t N, int64_t k, void* Y, int out_dtype,
                                      int64_t ldy, void* stream);

/* ------------------------------------------------------------------ whole path
 * The method end to end on one product: ss = score(A); I = topk(ss, k) with
 * k = rmm_k_from_rho(rho, d); A_I = compact(A, I); B_I = gather_rows(B, I);
 * Y = A_I · B_I.
 * A is [M x d] (lda), B is [d x N] (ldb), Y is [M x N] (ldy).  idx_out (k
 * int32, may be NULL) and ss_out (d floats, may be NULL) receive the
 * intermediate index set and scores.  Workspace: rmm_matmul_workspace_size
 * bytes, 256-byte aligned pointer. */
RMM_API size_t rmm_matmul_workspace_size(int dtype, int64_t M, int64_t d, int64_t N, double rho);
RMM_API rmm_status rmm_matmul(const void* A, int64_t lda, const void* B, int64_t ldb,
                      int64_t M, int64_t d, int64_t N, double rho, int dtype,
                      void* Y, int out_dtype, int64_t ldy, int32_t* idx_out, float* ss_out,
                      void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ int8 weights
 * The reduced product with an int8 weight (Resultados Experimentales ›
 * Compatibilidad: the method works with INT8 weight quantisation).  The
 * page fixes no scheme; the one taken here is symmetric weight-only
 * quantisation with one fp32 scale per output column:
 *     B[j, n] = Bq[j, n] * b_scale[n],   Bq int8 [d x N] (ldb bytes),
 * so  Y = A_I · B[idx, :] = (A_I · Bq[idx, :]) * b_scale  (column-wise).
 * The selection is unchanged: it reads the activation only.
 *  - M <= 16: the kept int8 rows are read in place (half the bytes of bf16),
 *    widened exactly to fp32, and each column's sum is scaled at the end.
 *  - M > 16: the kept rows are copied into workspace as exact bf16
 *    integers (from M = 256, with N a multiple of 8, mostly by the product
 *    kernel's own spare warps, as in rmm_gemm), the tcgen05 product runs on
 *    them, and the epilogue scales each column before rounding to out_dtype.
 * A_I bf16 [M x k] (ld_ai, a multiple of 8), Bq (ldb a multiple of 16), Y
 * (ldy) 16-byte aligned, else RMM_ERR_UNSUPPORTED.  b_scale [N] fp32,
 * finite.  Workspace: rmm_gemm_w8_workspace_size(N, k) bytes, 256-byte
 * aligned.  Out-of-range indices contribute zero and are flagged. */
RMM_API size_t rmm_gemm_w8_workspace_size(int64_t N, int64_t k);
RMM_API rmm_status rmm_gemm_w8(const void* A_I, int64_t ld_ai, const int8_t* Bq, int64_t ldb, const float* b_scale,
                               const int32_t* idx, int64_t d, int64_t M, int64_t N, int64_t k, void* Y,
                               int out_dtype, int64_t ldy, void* ws, size_t ws_bytes, void* stream);

/* The whole path with an int8 weight: ss = score(A) (bf16 A [M x d], lda);
 * I = topk(ss, k), k = rmm_k_from_rho(rho, d); Y = A_I · (Bq[I, :] *
 * b_scale).  idx_out and ss_out as in rmm_matmul.  Workspace:
 * rmm_matmul_w8_workspace_size bytes, 256-byte aligned. */
RMM_API size_t rmm_matmul_w8_workspace_size(int64_t M, int64_t d, int64_t N, double rho);
RMM_API rmm_status rmm_matmul_w8(const void* A, int64_t lda, const int8_t* Bq, int64_t ldb, const float* b_scale,
                                 int64_t M, int64_t d, int64_t N, double rho, void* Y, int out_dtype, int64_t ldy,
                                 int32_t* idx_out, float* ss_out, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ block driver
 * Several products that read the same activation share one selection
 * (Metodología › Mecanismo Central: I depends on A alone), e.g. the q, k and
 * v projections of an attention input or the up and gate projections of an
 * MLP input; each component keeps its own rho, since the pages find the
 * attention-side products more reducible than the MLP ones and, within the
 * MLP, the up projection the most sensitive and the down projection the
 * most robust (Contribuciones Clave › Perspectivas Mecanísticas).
 *
 * rmm_matmul_multi: Y[i] = A[:, I] · B[i][I, :] for i < nprod with one
 * I = topk(ss(A), k), k = rmm_k_from_rho(rho, d): one score pass (or none:
 * ss_in, the d column scores of A, may be given, e.g. by
 * rmm_silu_mul_score), one top-k, one compaction of A, then per product the
 * row gather of B[i] and the product (M > 16: tcgen05 GEMM, which from
 * M = 256 copies most of B[i]'s kept rows itself as in rmm_gemm; M <= 16:
 * kept rows read in place).  A bf16 [M x d] (lda); B[i] bf16 [d x N[i]] (ldb[i] a
 * multiple of 8, 16-byte aligned); Y[i] [M x N[i]] (ldy[i], 16-byte aligned)
 * in out_dtype.  idx_out (k, may be NULL) gets I; ss_out (d, may be NULL)
 * the computed scores (not written when ss_in is given).  Workspace:
 * rmm_matmul_multi_workspace_size(M, d, max N[i], rho) bytes. */
RMM_API size_t rmm_matmul_multi_workspace_size(int64_t M, int64_t d, int64_t N_max, double rho);
RMM_API rmm_status rmm_matmul_multi(const void* A, int64_t lda, int64_t M, int64_t d, double rho, int nprod,
                                    const void* const* B, const int64_t* ldb, const int64_t* N, void* const* Y,
                                    const int64_t* ldy, int out_dtype, const float* ss_in, int32_t* idx_out,
                                    float* ss_out, void* ws, size_t ws_bytes, void* stream);

/* The activation of an MLP's down projection with its column scores in the
 * same pass: H = bf16(SiLU(G) ⊙ U), SiLU(g) = g / (1 + e^-g) in fp32, and
 * ss_out[j] = sum_i H[i,j]^2 over the stored (rounded) H, summed in fp32 in
 * an order fixed by the shape.  G (gate output), U (up output), H bf16
 * [M x N] with pitches multiples of 8, 16-byte aligned.  Workspace:
 * rmm_silu_mul_score_workspace_size(M, N) bytes (may be 0). */
RMM_API size_t rmm_silu_mul_score_workspace_size(int64_t M, int64_t N);
RMM_API rmm_status rmm_silu_mul_score(const void* G, int64_t ldg, const void* U, int64_t ldu, int64_t M, int64_t N,
                                      void* H, int64_t ldh, float* ss_out, void* ws, size_t ws_bytes, void* stream);

/* A gated MLP block with every product reduced:
 *   U = X_I W_up[I,:], G = X_I W_gate[I,:] with one I from X (rho_up);
 *   H = SiLU(G) ⊙ U with its column scores fused into the producer;
 *   Y = H_J W_down[J,:] with J = topk(ss(H)) (rho_down).
 * X bf16 [M x d_model] (ldx); W_up, W_gate bf16 [d_model x d_ff] (ld_up,
 * ld_gate multiples of 8); W_down bf16 [d_ff x d_model] (ld_down a multiple
 * of 8); Y [M x d_model] (ldy) in out_dtype; all 16-byte aligned.  U, G, H
 * are bf16 in the workspace.  idx_up (k_up) and idx_down (k_down) may be
 * NULL.  Workspace: rmm_mlp_block_workspace_size bytes. */
RMM_API size_t rmm_mlp_block_workspace_size(int64_t M, int64_t d_model, int64_t d_ff, double rho_up, double rho_down);
RMM_API rmm_status rmm_mlp_block(const void* X, int64_t ldx, int64_t M, int64_t d_model, int64_t d_ff,
                                 const void* W_up, int64_t ld_up, const void* W_gate, int64_t ld_gate,
                                 const void* W_down, int64_t ld_down, double rho_up, double rho_down, void* Y,
                                 int out_dtype, int64_t ldy, int32_t* idx_up, int32_t* idx_down, void* ws,
                                 size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ reduced attention
 * Causal attention with both reductions of Metodología › Alcance de
 * Aplicación, for Q [B, Hq, S, D] and K, V [B, Hkv, S, D] bf16, contiguous
 * row-major (Hq a multiple of Hkv; q-head h reads kv-head h*Hkv/Hq):
 *   1. per (b, h): ssq = column scores of Q_bh over its S tokens;
 *      I_d = top k_d = ceil(rho_d*D) head_dim indices (lowest index on ties);
 *   2. logits S_ij = scale * sum_{c in I_d} Q[i,c] K[j,c] for j <= i
 *      (scale <= 0 selects 1/sqrt(D), the unreduced temperature);
 *      lse_i = logsumexp_{j<=i} S_ij;  P_ij = exp(S_ij - lse_i);
 *   3. token scores t_j = sum_{i>=j} P_ij^2 (squared column norms of P);
 *      I_t = top k_t = ceil(rho_t*S) tokens;
 *   4. O_i = sum_{j in I_t, j<=i} P_ij V[j,:]  (P not renormalised; a query
 *      with no kept token in its window gets a zero row).
 * Arithmetic: logits are exact bf16 products summed in fp32; softmax and token
 * scores in fp32; the P V product takes P' = 2^15 P and the kept rows of V in
 * fp16 (11 significant bits; V's bf16 values are exact there for magnitudes
 * in [2^-14, 65504]) with fp32 accumulation, scaled back by 2^-15.  A kept
 * value beyond 65504 is saturated and sets RMM_DEVERR_FP16_RANGE.
 * O is [B, Hq, S, D] written as out_dtype.  Optional outputs (may be NULL):
 * idx_d [B*Hq, k_d], idx_t [B*Hq, k_t], lse [B*Hq, S], tscore [B*Hq, S].
 * Requires D in {64, 128}, 1 <= S <= 65535 * 128 and B * Hq <= 65535 (the
 * grids' limits; RMM_ERR_INVALID_ARG otherwise).  Workspace:
 * rmm_attention_workspace_size. */
RMM_API size_t rmm_attention_workspace_size(int64_t B, int64_t Hq, int64_t Hkv, int64_t S, int64_t D,
                                    double rho_d, double rho_t);
RMM_API rmm_status rmm_attention(const void* Q, const void* K, const void* V,
                         int64_t B, int64_t Hq, int64_t Hkv, int64_t S, int64_t D,
                         double rho_d, double rho_t, float scale,
                         void* O, int out_dtype, int32_t* idx_d, int32_t* idx_t,
                         float* lse, float* tscore, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ reduced decode attention
 * One new query token per sequence attending to a KV cache, with both
 * reductions of Metodología › Alcance de Aplicación applied to its single
 * query row (the autoregressive setting of Resultados Experimentales):
 *   1. per (b, h): I_d = top k_d = ceil(rho_d*D) of q[b,h,c]^2 (lowest index
 *      on ties);
 *   2. s_j = scale * sum_{c in I_d} q[b,h,c] K[b,g,j,c] for the L cached
 *      tokens j < L (g = h*Hkv/Hq; scale <= 0 selects 1/sqrt(D));
 *      lse = logsumexp_j s_j;  P_j = exp(s_j - lse);
 *   3. t_j = P_j^2 (squared column norms of the one-row P); I_t = top
 *      k_t = ceil(rho_t*L) tokens (lowest index on ties);
 *   4. O[b,h,:] = sum_{j in I_t} P_j V[b,g,j,:]  (P not renormalised).
 * q [B, Hq, D] and O [B, Hq, D] (out_dtype) contiguous; K, V [B, Hkv, Lmax,
 * D] bf16 contiguous caches of capacity Lmax holding L valid tokens (rows
 * L..Lmax-1 are never read).  All four 16-byte aligned.  D in {64, 128},
 * Hq = G * Hkv with G (q-heads per kv-head) in {1, 2, 4, 8, 16}, else
 * RMM_ERR_UNSUPPORTED.  Optional outputs (may be NULL): idx_d [B*Hq, k_d],
 * idx_t [B*Hq, k_t] ascending, lse [B*Hq], logits [B*Hq, L] (the s_j; when
 * given it also serves as the kernels' logit buffer).  Workspace:
 * rmm_decode_attention_workspace_size(B, Hq, L, D, rho_t, logits != NULL,
 * idx_t != NULL) bytes, 256-byte aligned. */
RMM_API size_t rmm_decode_attention_workspace_size(int64_t B, int64_t Hq, int64_t L, int64_t D, double rho_t,
                                                   int with_logits, int with_idx_t);
RMM_API rmm_status rmm_decode_attention(const void* q, const void* K, const void* V, int64_t B, int64_t Hq,
                                        int64_t Hkv, int64_t L, int64_t Lmax, int64_t D, double rho_d, double rho_t,
                                        float scale, void* O, int out_dtype, int32_t* idx_d, int32_t* idx_t,
                                        float* lse, float* logits, void* ws, size_t ws_bytes, void* stream);

/* ------------------------------------------------------------------ self-test
 * Makes one of the library's bounded waits run out on purpose and returns
 * (asynchronously, on `stream`); no fault, trap or endless loop is involved.
 * Every wait in librmm's kernels gives up after 2 s, records
 * RMM_DEVERR_TIMEOUT_BASE + site in the device error word, and lets its
 * kernel return.  Read the code with rmm_device_error() afterwards; the
 * context stays usable.
 *   which 0: an mbarrier that nothing arrives on (site 62);
 *   which 1: a global flag that nothing raises (site 63);
 *   which 2: the CTA-pair product whose spare warps copy B_I, with its copy
 *            counters preset so that nothing is copied.  Its producer, MMA
 *            and epilogue waits give up, and the kernel unwinds through its
 *            abort path (site 43, 44 or 45: whichever wait runs out first).
 * Allocates and frees about 0.25 MB on the stream (cudaMallocAsync).
 * Takes about 2 s of GPU time. */
RMM_API rmm_status rmm_selftest_timeout(int which, void* stream);

#ifdef __cplusplus
}
#endif

#endif /* RMM_H_ */
