/*
 * librmm — Reduced Matrix Multiplication (RMM) on NVIDIA B200 (sm_100a).
 *
 * The method (web pages on "Reduced Matrix Multiplication: Input-Adaptive
 * Matrix-Product Reduction for LLM Inference"; gist.science summary,
 * Resumo Técnico › Metodologia):
 *   - "Mecanismo Central": instead of Y = A·B, compute A[:, I]·B[I, :] for a
 *     subset I of the shared contraction dimension.
 *   - "Estratégia de Seleção": score every contraction slice, keep the top
 *     k = ceil(rho·K) of them, rho the user's retention ratio.
 *   - "Escopo de Aplicação": Q·Kᵀ reduced over the head dimension, P·V
 *     reduced over the key (token) dimension, X·W over the hidden dimension.
 *
 * Library defaults where the pages are silent:
 *   - score s_k = ||A[:,k]||_2 · ||B[k,:]||_2 (RMM_SCORE_PRODUCT); the pages'
 *     activation-only column norm ||A[:,k]||_2 is RMM_SCORE_A_ONLY;
 *   - ties in the score go to the lower index; kept indices are ascending;
 *   - one selection per matrix product (per batch item / attention head).
 *
 * Conventions for every call:
 *   - Pointers named A, B, C, s, idx, A_S, B_St, workspace, status_word are
 *     DEVICE pointers owned by the caller. The library never allocates.
 *   - Matrices are row-major. "ld" is the leading dimension in elements
 *     (distance between consecutive rows), "stride" the distance in elements
 *     between consecutive batch items.
 *   - bf16 data is passed as raw 16-bit words (the bits of __nv_bfloat16).
 *   - All work is enqueued on `stream` in order; no call synchronises the
 *     host except rmm_check.
 *   - A call makes the stream's device current while it runs and restores the
 *     caller's current device before it returns.
 *   - Argument errors are detected on the host, before any launch, and
 *     returned as RMM_ERR_INVALID / RMM_ERR_UNSUPPORTED. A failed CUDA
 *     runtime call returns RMM_ERR_CUDA. rmm_last_error_string() describes
 *     the most recent failure on the calling thread.
 *   - Errors found on the device (a non-finite score, a pipeline wait that
 *     ran out) are OR-ed as bits into a 32-bit status word in device memory;
 *     rmm_check() reads and clears it. No kernel traps.
 *   - M = 0, N = 0 or batch = 0 are valid and launch nothing that writes C
 *     (scores and selection are still produced when M = 0: all scores are 0).
 */
#ifndef RMM_H_
#define RMM_H_

#include <stddef.h>
#include <stdint.h>
#include <cuda_runtime_api.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  RMM_OK = 0,
  RMM_ERR_INVALID = 1,     /* bad argument (null pointer, rho outside (0,1], bad ld, small workspace) */
  RMM_ERR_NONFINITE = 2,   /* a slice score was NaN or Inf (reported by rmm_check) */
  RMM_ERR_CUDA = 3,        /* a CUDA runtime call failed */
  RMM_ERR_TIMEOUT = 4,     /* a bounded pipeline wait in a kernel gave up (reported by rmm_check) */
  RMM_ERR_UNSUPPORTED = 5  /* valid request this build does not handle (e.g. device is not sm_100) */
} rmm_status;

typedef enum { RMM_BF16 = 0, RMM_F32 = 1 } rmm_dtype;

typedef enum { RMM_SCORE_PRODUCT = 0, RMM_SCORE_A_ONLY = 1 } rmm_score_mode;

/* Device status-word bits (see rmm_check). */
#define RMM_STATUS_BIT_NONFINITE 0x1u
#define RMM_STATUS_BIT_TIMEOUT   0x2u

/* ---------------------------------------------------------------- host helpers */

/* k = ceil(rho·K) ("Estratégia de Seleção"), the IEEE double product rounded up.
 * Returns -1 unless 0 < rho <= 1 and K >= 1. Never returns 0 for valid input. */
int64_t rmm_keep_count(double rho, int64_t K);

/* Contraction extent of the packed operands: k_keep rounded up to 64, the
 * K-depth of one tensor-core pipeline stage. Padding columns hold zeros. */
int64_t rmm_padded_keep(int64_t k_keep);

/* Row pitch, in elements, of the packed N-major B operand: N rounded up to 8
 * (so that every row starts on a 16-byte boundary). */
int64_t rmm_packed_b_ld(int64_t N);

/* Bytes of workspace rmm_matmul_reduced / _batched / rmm_qk_reduced /
 * rmm_pv_reduced need for these sizes (in = input dtype). The workspace holds,
 * each 1 KiB-aligned: the status word, scores [batch][K] f32, kept indices
 * [batch][k_keep] i32, A_S [batch][M][k_pad] and the packed B operand
 * (room for [batch][k_pad][rmm_packed_b_ld(N)]). */
size_t rmm_workspace_size(int64_t batch, int64_t M, int64_t K, int64_t N, int64_t k_keep,
                          rmm_dtype in);

/* The workspace a fused call needs for the route it takes with these sizes
 * and B's layout (b_kmajor as in rmm_score; 0 for the INT8-weight call; see
 * rmm_fused_route):
 *   - gather-GEMV (M <= 16, B row-major): the status word, scores and indices
 *     only (for x[1][8192] · W[8192][28672] at rho = 0.5: 49 KiB instead of
 *     224 MiB);
 *   - stream (bf16, B row-major, N <= 128, M > 16): those plus B with its
 *     dropped rows zeroed, [batch][K][rmm_packed_b_ld(N)] (P·V at S = 32768,
 *     32 heads, rho = 0.5: 256 MiB instead of 34 GiB of packed operands). This
 *     assumes A can be streamed (16-byte aligned base, row pitch and batch
 *     stride multiples of 8 elements); an A that cannot takes the pack route,
 *     which needs rmm_workspace_size;
 *   - pack: the packed operands A_S and B_S as well.
 * The fused calls accept any workspace of at least this size; the layout of
 * what they use does not change. */
size_t rmm_workspace_size_for(int64_t batch, int64_t M, int64_t K, int64_t N, int64_t k_keep,
                              rmm_dtype in, int b_kmajor);

/* ---------------------------------------------------------------- stage calls */

/* Slice scores ("Estratégia de Seleção"; product form is the library default).
 *   A: [batch][M][K] (ld lda, batch stride strideA), dtype `in`.
 *   B: if b_kmajor == 0, [batch][K][N] (ld ldb), "row k of B" is B[k, :];
 *      if b_kmajor == 1, B is given transposed as [batch][N][K] (ld ldb), so
 *      "row k of B" is column k of that matrix (the Q·Kᵀ case, Kmat).
 *      B is not read in RMM_SCORE_A_ONLY mode and may be NULL there.
 *      strideA / strideB may be 0 to use one matrix for every batch item (a
 *      read-only input such as a weight); otherwise batch items must not
 *      overlap. The same holds for every call that takes A and B.
 *   s: [batch][K] f32 output: s_k = sqrt(sum_i A[i,k]^2) · sqrt(sum_j B[k,j]^2)
 *      (product) or sqrt(sum_i A[i,k]^2) (a_only); sums in f32 in a fixed order,
 *      so repeated calls give identical bits.
 *   status_word: nullable device u32; RMM_STATUS_BIT_NONFINITE is OR-ed in when
 *      a score is NaN/Inf (e.g. NaN inputs or f32 overflow of a sum of squares). */
rmm_status rmm_score(const void* A, int64_t lda, int64_t strideA,
                     const void* B, int64_t ldb, int64_t strideB, int b_kmajor,
                     int64_t batch, int64_t M, int64_t K, int64_t N,
                     rmm_dtype in, rmm_score_mode mode, float* s,
                     uint32_t* status_word, cudaStream_t stream);

/* Top-k selection ("Estratégia de Seleção": keep the k_keep largest scores).
 *   s: [batch][K] f32 scores; idx: [batch][k_keep] i32 output, ascending.
 *   Ties go to the lower index; -0.0 equals +0.0. Exact: the result depends
 *   only on the order of the scores, never on rounding. 1 <= k_keep <= K.
 *   A NaN or infinite score sets RMM_STATUS_BIT_NONFINITE in status_word
 *   (nullable).
 *   K is at most 2^21 (RMM_ERR_UNSUPPORTED above; the same limit applies to
 *   every call that selects). */
rmm_status rmm_select(const float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx,
                      uint32_t* status_word, cudaStream_t stream);

/* Pack the kept slices ("Mecanismo Central": A[:, I] and B[I, :]).
 *   A, B as in rmm_score (B is required here); idx: [batch][k_keep] i32 indices
 *   in [0, K) (as produced by rmm_select; 16-byte aligned for the fast path).
 *   A_S: [batch][M][k_pad] output, A_S[b][i][t] = A[b][i][idx[b][t]]
 *        (contraction dimension contiguous).
 *   B_S: if b_kmajor == 0: [batch][k_pad][ldbs], ldbs = rmm_packed_b_ld(N),
 *        B_S[b][t][j] = B[b][idx[b][t]][j] — the kept rows of B as they are;
 *        if b_kmajor == 1: [batch][N][k_pad], B_S[b][j][t] = Kmat[b][j][idx[b][t]].
 *   k_pad = rmm_padded_keep(k_keep); slices t >= k_keep (and columns j >= N of
 *   the row-major form) are written as zero. Copies bits exactly (no
 *   arithmetic). Indices outside [0, K) are a caller error that the kernels
 *   do not check; with debug checks on (rmm_set_debug) the call validates idx
 *   on the device first and returns RMM_ERR_INVALID, launching nothing that
 *   reads through it. status_word (nullable) receives RMM_STATUS_BIT_TIMEOUT
 *   if a bounded wait for a bulk copy gave up. */
rmm_status rmm_pack(const void* A, int64_t lda, int64_t strideA,
                    const void* B, int64_t ldb, int64_t strideB, int b_kmajor,
                    int64_t batch, int64_t M, int64_t K, int64_t N,
                    const int32_t* idx, int64_t k_keep, rmm_dtype in,
                    void* A_S, void* B_S, uint32_t* status_word, cudaStream_t stream);

/* Reduced product on packed operands: C[b] = A_S[b] · B_S[b] over the k_keep
 * kept slices ("Mecanismo Central"), f32 accumulation.
 *   A_S, B_S as written by rmm_pack with the same b_kmajor (zero padding,
 *   16-byte aligned base pointers).
 *   in == RMM_BF16: tcgen05 tensor-core kernel (TMA, TMEM accumulators).
 *   in == RMM_F32: CUDA-core FFMA kernel (f32 products, f32 sums).
 *   C: [batch][M][N] with ld ldc, batch stride strideC, dtype `out`
 *      (RMM_F32 or RMM_BF16, round-to-nearest-even).
 *   status_word (nullable): RMM_STATUS_BIT_TIMEOUT if a pipeline wait gave up
 *   (then C is incomplete). */
rmm_status rmm_gemm(const void* A_S, const void* B_S, int b_kmajor, int64_t batch, int64_t M,
                    int64_t N, int64_t k_keep, rmm_dtype in, void* C, int64_t ldc, int64_t strideC,
                    rmm_dtype out, uint32_t* status_word, cudaStream_t stream);

/* B_M = B with the rows outside the kept set zeroed ("Mecanismo Central":
 * A[:, I]·B[I, :] = A·B_M, since a dropped slice then contributes zero):
 *   B: [batch][K][N] row-major (ldb, strideB; strideB = 0 shares one B);
 *   idx: [batch][k_keep] ascending kept indices in [0, K) (as rmm_select
 *   writes them); B_M: [batch][K][rmm_packed_b_ld(N)] output, 16-byte aligned,
 *   B_M[b][r][j] = B[b][r][j] if r is in idx[b], else 0; columns N <= j <
 *   rmm_packed_b_ld(N) are 0. Copies bits exactly. With debug checks on,
 *   idx is validated first (see rmm_set_debug). */
rmm_status rmm_mask_rows(const void* B, int64_t ldb, int64_t strideB, int64_t batch, int64_t K, int64_t N,
                         const int32_t* idx, int64_t k_keep, rmm_dtype in, void* B_M, cudaStream_t stream);

/* C[b] = A[b] · B_M[b] over all K slices on the bf16 tensor cores (f32
 * accumulation): with B_M from rmm_mask_rows this is the reduced product
 * A[:, I]·B[I, :] computed by streaming A whole, the fused calls' route for
 * narrow products (rmm_fused_route).
 *   A: [batch][M][K] row-major, bf16, 16-byte aligned, lda and (batch > 1)
 *   strideA multiples of 8 and strideA nonzero (RMM_ERR_INVALID otherwise);
 *   B_M: [batch][K][rmm_packed_b_ld(N)], 16-byte aligned; C as in rmm_gemm.
 *   causal_off: -1 for a dense A; >= 0 declares A[i][k] = 0 for k > i +
 *   causal_off (a causal attention matrix, causal_off = S_k - S_q), and each
 *   tile of rows stops at the last key its rows see (the blocks above hold
 *   zeros and are not read).
 *   in must be RMM_BF16 (RMM_ERR_UNSUPPORTED otherwise). */
rmm_status rmm_gemm_full(const void* A, int64_t lda, int64_t strideA, const void* B_M, int64_t batch, int64_t M,
                         int64_t K, int64_t N, int64_t causal_off, rmm_dtype in, void* C, int64_t ldc, int64_t strideC,
                         rmm_dtype out, uint32_t* status_word, cudaStream_t stream);

/* Which route a fused call (rmm_matmul_reduced, _batched, _b_norms,
 * rmm_qk_reduced, rmm_pv_reduced) takes for these sizes and this A:
 *   2 = gather-GEMV (M <= 16 and B row-major: score, select, rmm_gemv_gather;
 *       when the score needs only A — B's row norms given, or the A-only
 *       score — and M <= 4, K <= 8192, the selection kernel computes the
 *       scores itself, bit-identical to rmm_score_b_norms / rmm_score, so the
 *       call launches two kernels);
 *   1 = stream (bf16, B row-major, N <= 128, M > 16, A streamable as in
 *       rmm_gemm_full: score, select, rmm_mask_rows, rmm_gemm_full). A
 *       narrow product is bound by reading A, and A's kept columns reach into
 *       nearly every 32-byte sector of A, so streaming A once beats packing
 *       it (read A, write and re-read A_S);
 *   0 = pack (score, select, rmm_pack, rmm_gemm);
 *  -1 for invalid sizes or dtype. Host only; never launches anything. */
int rmm_fused_route(int64_t batch, int64_t M, int64_t N, int b_kmajor, rmm_dtype in, const void* A, int64_t lda,
                    int64_t strideA);

/* ---------------------------------------------------------------- fused calls */

/* Y ≈ A·B with the top ceil(rho·K) contraction slices kept: score → select →
 * the product over the kept slices (pack + gemm, or the stream or
 * gather-GEMV route, see rmm_fused_route), all enqueued on `stream`.
 *   A [M][K] (ld lda), B [K][N] (ld ldb), C [M][N] (ld ldc); dtypes in/out.
 *   idx_out: nullable device [k_keep] i32 that receives the kept indices.
 *   workspace: device buffer of at least rmm_workspace_size_for(1, M, K, N, k,
 *   in, 0) bytes (rmm_workspace_size always suffices), 1 KiB-aligned; its
 *   first 4 bytes are the status word, cleared at
 *   the start of the call. Call rmm_check(workspace, stream) to learn of
 *   device-side errors. Workspace contents are scratch between calls. */
rmm_status rmm_matmul_reduced(const void* A, int64_t lda, const void* B, int64_t ldb,
                              int64_t M, int64_t K, int64_t N, double rho,
                              rmm_dtype in, rmm_score_mode mode,
                              void* C, int64_t ldc, rmm_dtype out, int32_t* idx_out,
                              void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Batched form: an independent selection per batch item. Layouts as in
 * rmm_score / rmm_pack; C [batch][M][N] (ldc, strideC); idx_out nullable
 * [batch][k_keep]. */
rmm_status rmm_matmul_reduced_batched(const void* A, int64_t lda, int64_t strideA,
                                      const void* B, int64_t ldb, int64_t strideB, int b_kmajor,
                                      int64_t batch, int64_t M, int64_t K, int64_t N, double rho,
                                      rmm_dtype in, rmm_score_mode mode,
                                      void* C, int64_t ldc, int64_t strideC, rmm_dtype out,
                                      int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream);

/* Decode-shaped reduced product without packing: C[b] = A[b][:, idx[b]] ·
 * B[b][idx[b], :] for M <= 16 rows of A (a few tokens, "Escopo de
 * Aplicação": autoregressive use), B row-major [batch][K][N]. Reads A and B
 * directly through idx (as written by rmm_select), streaming only the kept
 * rows of B; f32 products and fixed-order f32 sums (bit-reproducible); C as
 * in rmm_gemm. The fused calls take this route by themselves when M <= 16
 * and B is row-major (they then skip rmm_pack); combine with cached B norms
 * (below) or the A-only score so that scoring does not read all of B either.
 * M > 16 is RMM_ERR_INVALID. */
rmm_status rmm_gemv_gather(const void* A, int64_t lda, int64_t strideA,
                           const void* B, int64_t ldb, int64_t strideB,
                           int64_t batch, int64_t M, int64_t K, int64_t N,
                           const int32_t* idx, int64_t k_keep, rmm_dtype in,
                           void* C, int64_t ldc, int64_t strideC, rmm_dtype out,
                           cudaStream_t stream);

/* ---------------------------------------------------------------- cached B norms
 * B's factor of the product score, ||B[k,:]||_2, depends on B alone. When B is
 * a weight that is reused across calls, it can be computed once with
 * rmm_b_norms and passed to rmm_score_b_norms / rmm_matmul_reduced_b_norms,
 * which then read only A to score (the selection and the product are
 * computed as before). The cached scores agree with rmm_score's product
 * scores to f32 rounding (B's norms are the same f32 sums for b_kmajor == 0;
 * A's column sums may be grouped differently), so a near-tie can order
 * differently; the result is deterministic either way. This is an
 * implementation convenience; the pages' method has no separate step for it. */

/* b_norm[b][k] = sqrt(sum_j B[b][k][j]^2) (b_kmajor == 0, B [batch][K][N]) or
 * sqrt(sum_j Kmat[b][j][k]^2) (b_kmajor == 1, B = Kmat [batch][N][K]); f32,
 * [batch][K] contiguous. status_word (nullable) receives
 * RMM_STATUS_BIT_NONFINITE for a NaN/Inf norm. */
rmm_status rmm_b_norms(const void* B, int64_t ldb, int64_t strideB, int b_kmajor,
                       int64_t batch, int64_t K, int64_t N, rmm_dtype in, float* b_norm,
                       uint32_t* status_word, cudaStream_t stream);

/* rmm_score (product form) with B's norms given: s[b][k] = sqrt(sum_i A[b][i][k]^2)
 * · b_norm[b·b_norm_stride + k]. b_norm_stride = 0 shares one [K] vector among
 * all batch items (one weight for the whole batch), K when b_norm is
 * [batch][K]. */
rmm_status rmm_score_b_norms(const void* A, int64_t lda, int64_t strideA, const float* b_norm,
                             int64_t b_norm_stride, int64_t batch, int64_t M, int64_t K,
                             rmm_dtype in, float* s, uint32_t* status_word, cudaStream_t stream);

/* rmm_matmul_reduced_batched in product mode with cached B norms (the score
 * reads only A). Arguments as there, plus b_norm / b_norm_stride as in
 * rmm_score_b_norms; workspace sized by rmm_workspace_size as before. */
rmm_status rmm_matmul_reduced_b_norms(const void* A, int64_t lda, int64_t strideA,
                                      const void* B, int64_t ldb, int64_t strideB, int b_kmajor,
                                      const float* b_norm, int64_t b_norm_stride,
                                      int64_t batch, int64_t M, int64_t K, int64_t N, double rho,
                                      rmm_dtype in, void* C, int64_t ldc, int64_t strideC, rmm_dtype out,
                                      int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                      cudaStream_t stream);

/* ---------------------------------------------------------------- INT8 weights
 * "Resultados Experimentais" › "Compatibilidade": the method works with INT8
 * weight quantization. Read as symmetric per-output-channel quantization: the
 * weight W [K][N] is given as Wq (int8, [batch][K][ldw], batch stride strideW;
 * values in [-127, 127]) and scale (f32 [N] per batch item, scale_stride apart,
 * 0 = one vector for all items), W[k][j] = Wq[k][j] · scale[j]; the method runs
 * on that W. A stays bf16. The gather-GEMV (M <= 16) needs Wq's rows and
 * base 4-byte aligned (RMM_ERR_UNSUPPORTED otherwise); the other calls take
 * any alignment. */

/* b_norm[b][k] = ||W[b][k][:]||_2 of the dequantized weight (f32 sums), the
 * B factor of the product score, for caching while the weight is unchanged. */
rmm_status rmm_b_norms_w8(const int8_t* Wq, int64_t ldw, int64_t strideW, const float* scale,
                          int64_t scale_stride, int64_t batch, int64_t K, int64_t N, float* b_norm,
                          uint32_t* status_word, cudaStream_t stream);

/* rmm_pack for an INT8 weight: A_S as in rmm_pack; B_S [batch][k_pad][ldbs]
 * (ldbs = rmm_packed_b_ld(N)) holds bf16(Wq[idx[t]][j] · scale[j]) (round to
 * nearest even), zero padded — the operand rmm_gemm takes with b_kmajor = 0. */
rmm_status rmm_pack_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                       int64_t strideW, const float* scale, int64_t scale_stride, int64_t batch, int64_t M,
                       int64_t K, int64_t N, const int32_t* idx, int64_t k_keep, void* A_S, void* B_S,
                       uint32_t* status_word, cudaStream_t stream);

/* rmm_gemv_gather on an INT8 weight (M <= 16): C = A[:, idx] · W[idx, :] with
 * W = Wq · diag(scale), Wq's kept rows read directly (int8), products and sums
 * in f32, the column scale applied to the sums. */
rmm_status rmm_gemv_gather_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                              int64_t strideW, const float* scale, int64_t scale_stride, int64_t batch,
                              int64_t M, int64_t K, int64_t N, const int32_t* idx, int64_t k_keep, void* C,
                              int64_t ldc, int64_t strideC, rmm_dtype out, cudaStream_t stream);

/* The fused call on an INT8 weight: score with cached b_norm (product mode,
 * b_norm from rmm_b_norms_w8, b_norm_stride as in rmm_score_b_norms) or
 * A-only (mode RMM_SCORE_A_ONLY, b_norm may be NULL), select, then for
 * M <= 16 the gather-GEMV reading Wq's kept rows directly (int8 loads, f32
 * products, the column scale applied to the sums) and otherwise rmm_pack_w8 +
 * the tensor-core GEMM. in must be RMM_BF16 (A). Other arguments as in
 * rmm_matmul_reduced_batched; workspace sized by rmm_workspace_size(...,
 * RMM_BF16). */
rmm_status rmm_matmul_reduced_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                                 int64_t strideW, const float* scale, int64_t scale_stride,
                                 const float* b_norm, int64_t b_norm_stride, int64_t batch, int64_t M,
                                 int64_t K, int64_t N, double rho, rmm_dtype in, rmm_score_mode mode,
                                 void* C, int64_t ldc, int64_t strideC, rmm_dtype out, int32_t* idx_out,
                                 void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Attention scores S = Q·Kᵀ per head, reduced over the head dimension
 * ("Escopo de Aplicação": the feature dimension of QKᵀ).
 *   Q [bh][S_q][d], Kmat [bh][S_k][d] (contiguous); S_out [bh][S_q][S_k]
 *   (contiguous, dtype out). One selection of ceil(rho·d) channels per head.
 *   Workspace: rmm_workspace_size(bh, S_q, d, S_k, k, in). */
rmm_status rmm_qk_reduced(const void* Q, const void* Kmat, int64_t bh, int64_t S_q, int64_t S_k,
                          int64_t d, double rho, rmm_dtype in, rmm_score_mode mode,
                          void* S_out, rmm_dtype out, int32_t* idx_out,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* Attention output O = P·V per head, reduced over the keys ("Escopo de
 * Aplicação": the token dimension of PV, which the pages mark optional).
 *   P [bh][S_q][S_k], V [bh][S_k][d] (contiguous); O [bh][S_q][d] (contiguous,
 *   dtype out). One selection of ceil(rho·S_k) keys per head.
 *   Workspace: rmm_workspace_size(bh, S_q, S_k, d, k, in). */
rmm_status rmm_pv_reduced(const void* P, const void* V, int64_t bh, int64_t S_q, int64_t S_k,
                          int64_t d, double rho, rmm_dtype in, rmm_score_mode mode,
                          void* O, rmm_dtype out, int32_t* idx_out,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream);

/* ---------------------------------------------------------------- P·V with its softmax producer
 * "Escopo de Aplicação": P·V reduced over the keys, P the attention matrix
 * (the row softmax of the scaled logits). The key score s_k = ||P[:, k]||_2 ·
 * ||V[k, :]||_2 (product mode; ||P[:, k]||_2 in A-only mode) needs the column
 * sums of squares of P, which the kernel that writes P has in hand: P is not
 * read back to be scored.
 *   L: logits [bh][S_q][S_k] contiguous, dtype ldt (bf16 or f32); P =
 *   softmax(scale·L) per row. With causal != 0 query q sees key k only when
 *   k <= q + S_k - S_q (the last query sees every key; S_q <= S_k required)
 *   and masked entries of P are 0.
 *   P: [bh][S_q][S_k] bf16 output (round to nearest even), every entry written.
 *   V: [bh][S_k][d] bf16 contiguous. */

/* Row statistics of the softmax: stats[b][q][0] = max over the visible keys of
 * x = scale·log2(e)·L[b][q][k], stats[b][q][1] = 1 / sum exp2(x - max).
 * status_word (nullable) receives RMM_STATUS_BIT_NONFINITE for a row whose
 * statistics are not finite. */
rmm_status rmm_softmax_row_stats(const void* L, rmm_dtype ldt, float scale, int causal, int64_t bh, int64_t S_q,
                                 int64_t S_k, float* stats, uint32_t* status_word, cudaStream_t stream);

/* P from the logits and their row statistics, and (s non-null) the key scores
 * of P·V over the stored bf16 values: s[b][k] = ||P[b][:, k]||_2 ·
 * ||V[b][k, :]||_2, or ||P[b][:, k]||_2 when V is NULL (A-only). Column sums
 * in f32 in a fixed order (bit-reproducible; not the bits rmm_score gives for
 * the same P, which sums in another order). d: V's columns (ignored without
 * V). */
rmm_status rmm_softmax_score(const void* L, rmm_dtype ldt, float scale, int causal, const float* stats, const void* V,
                             int64_t d, int64_t bh, int64_t S_q, int64_t S_k, void* P, float* s,
                             uint32_t* status_word, cudaStream_t stream);

/* Workspace of rmm_pv_softmax_reduced, 1 KiB-aligned sections: the status
 * word, row statistics [bh][S_q][2] f32, scores [bh][S_k] f32, kept indices
 * [bh][k_keep] i32, and V with its dropped rows zeroed [bh][S_k][rmm_packed_b_ld(d)]. */
size_t rmm_pv_softmax_workspace_size(int64_t bh, int64_t S_q, int64_t S_k, int64_t d, int64_t k_keep);

/* O ≈ P·V with P = softmax(scale·L) produced by this call: row statistics,
 * P and the key scores in one pass over P (rmm_softmax_score), the top
 * ceil(rho·S_k) keys per head (rmm_select), V's dropped rows zeroed
 * (rmm_mask_rows) and the tensor-core GEMM over P as written (rmm_gemm_full;
 * with the causal mask it skips the key blocks above each tile's last row).
 *   P must be 16-byte aligned and S_k a multiple of 8 (RMM_ERR_UNSUPPORTED
 *   otherwise): the GEMM reads it by TMA.
 *   O: [bh][S_q][d] (contiguous, dtype out); idx_out: nullable [bh][k_keep].
 *   workspace: rmm_pv_softmax_workspace_size bytes, 1 KiB-aligned; its first
 *   4 bytes are the status word (rmm_check). */
rmm_status rmm_pv_softmax_reduced(const void* L, rmm_dtype ldt, float scale, int causal, const void* V, int64_t bh,
                                  int64_t S_q, int64_t S_k, int64_t d, double rho, rmm_score_mode mode, void* P,
                                  void* O, rmm_dtype out, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream);

/* Allocation-free form of rmm_matmul_reduced (the paper has no counterpart:
 * this is a deployment convenience of this library).
 * For callers that must not allocate device memory — for example code running
 * under another framework's memory pool or allocator hooks, a plugin that is
 * handed only its input and output buffers, or a process whose device memory
 * is reserved in full up front. Arguments are those of rmm_matmul_reduced
 * minus the workspace; the scratch (status word, scores, indices, packed
 * operands) comes from one static device array of 32 MiB that this library
 * defines. Every device on which the call has run keeps that array until the
 * process exits (with eager module loading, every device that loads the
 * library does).
 *   - Products whose rmm_workspace_size_for(1, M, K, N, k, in, 0) exceeds
 *     32 MiB (33554432 bytes) are rejected with RMM_ERR_INVALID before any
 *     launch (decode shapes, M <= 16, need only their scores and indices).
 *   - Nothing is allocated: no cudaMalloc, cudaFree or allocating library call.
 *   - The first call on a device looks up the array's device address
 *     (cudaGetSymbolAddress) with that device current; make that first call
 *     before any stream capture. A lookup that fails is not remembered: the
 *     call returns RMM_ERR_CUDA and the next call on that device tries again.
 *   - All calls share the one array and it keeps the last call's contents;
 *     the status word in it is cleared at the start of each call. Calls whose
 *     work overlaps on the GPU (different streams, or other threads) race on
 *     the array: serialise them.
 *   - status_word: nullable device u32 that receives a copy of this call's
 *     device status bits, in stream order; read it with rmm_check. */
rmm_status rmm_matmul_reduced_noalloc(const void* A, int64_t lda, const void* B, int64_t ldb,
                                      int64_t M, int64_t K, int64_t N, double rho,
                                      rmm_dtype in, rmm_score_mode mode,
                                      void* C, int64_t ldc, rmm_dtype out, int32_t* idx_out,
                                      uint32_t* status_word, cudaStream_t stream);

/* ---------------------------------------------------------------- diagnostics */

/* Synchronises `stream`, reads the status word at `status_word` (a workspace
 * base pointer works: the word is its first 4 bytes), clears it, and returns
 * RMM_OK, RMM_ERR_NONFINITE or RMM_ERR_TIMEOUT (timeout wins if both). */
rmm_status rmm_check(void* status_word, cudaStream_t stream);

/* Message for the most recent failure on the calling thread ("" if none). */
const char* rmm_last_error_string(void);

/* Upper bound, in nanoseconds, on any single pipeline wait inside the
 * tensor-core GEMM before it records RMM_STATUS_BIT_TIMEOUT and winds down
 * (default 2e9 = 2 s; 0 restores the default). Process-wide. */
void rmm_set_wait_limit_ns(uint64_t ns);

/* Test hook, process-wide: when `on` is nonzero, the next tensor-core GEMM
 * launches run with their TMA producer idle, so the MMA and epilogue waits run
 * out; the kernel then records RMM_STATUS_BIT_TIMEOUT, drains, frees its
 * tensor memory and returns. Used to test the timeout path without a fault. */
void rmm_set_stall_producer_for_test(int on);

/* Tensor-core GEMM variant, process-wide: 2 (default) runs 2-SM MMAs on CTA
 * pairs (256-row tiles, A and B halves in the two SMs' shared memory); 1 runs
 * one SM per 128-row tile. Results are identical up to f32 summation order
 * (both sum the kept slices in ascending order). Returns the previous
 * setting; values other than 1 and 2 change nothing. */
int rmm_set_gemm_cta_group(int cta_group);

/* Number of kernels this library has launched in this process. */
uint64_t rmm_launch_count(void);

/* Debug checks, process-wide; returns the previous setting. Off by default,
 * or on when the environment variable RMM_DEBUG is set to anything but "0"
 * at the first call. When on:
 *   - rmm_pack, rmm_pack_w8, rmm_gemv_gather and rmm_gemv_gather_w8 first
 *     check on the device that every kept index lies in [0, K), synchronise
 *     the stream, and return RMM_ERR_INVALID (naming the first bad entry)
 *     without launching the kernels that would read through a bad index;
 *   - the fused calls synchronise the stream after their kernels and return
 *     RMM_ERR_NONFINITE / RMM_ERR_TIMEOUT from the status word directly (the
 *     word is left set for rmm_check).
 * Calls with debug checks on share one device word for the index check and
 * must not run concurrently. Not for timed or captured work. */
int rmm_set_debug(int on);

/* Timing hook (diagnostics; no counterpart in the method). While set, every
 * GEMM launch of this process records `start` on its stream immediately
 * before the GEMM kernel and `stop` immediately after it, so that
 * cudaEventElapsedTime(start, stop) is that kernel alone (a split-K zeroing
 * kernel of rmm_gemm runs before `start`). The events are created and owned
 * by the caller; pass NULL, NULL to clear. Recording an event between two
 * kernels ends their programmatic launch overlap, so the hook perturbs the
 * timing of whatever surrounds the GEMM. Process-wide; not for concurrent
 * callers. */
void rmm_set_gemm_events(cudaEvent_t start, cudaEvent_t stop);

#ifdef __cplusplus
}
#endif

#endif /* RMM_H_ */
