// Internal host-side interface between the C ABI (api.cu) and the kernel
// launchers. Not installed; not part of the ABI.
#pragma once

#include <cstddef>
#include <cstdint>
#include <cuda_runtime.h>

namespace rmm {

enum ElemKind { kBF16 = 0, kF32 = 1 };
inline size_t elem_bytes(ElemKind e) { return e == kBF16 ? 2 : 4; }

// Strided view of a batch of row-major matrices.
struct MatView {
  const void* ptr;
  int64_t ld;       // elements between rows
  int64_t bstride;  // elements between batch items
  int64_t rows;
  int64_t cols;
};

void count_launch();

// Makes the stream's device current for the life of the guard and restores
// the caller's current device when it goes out of scope (only if it changed).
struct DeviceGuard {
  int prev = -1;
  DeviceGuard() = default;
  DeviceGuard(const DeviceGuard&) = delete;
  DeviceGuard& operator=(const DeviceGuard&) = delete;
  // Returns the CUDA error of the lookup or switch (cudaSuccess on success).
  cudaError_t bind(cudaStream_t st) {
    int dev = -1;
    cudaError_t e = cudaStreamGetDevice(st, &dev);
    if (e != cudaSuccess) return e;
    int cur = -1;
    e = cudaGetDevice(&cur);
    if (e != cudaSuccess) return e;
    if (cur != dev) {
      e = cudaSetDevice(dev);
      if (e != cudaSuccess) return e;
      if (prev < 0) prev = cur;
    }
    return cudaSuccess;
  }
  ~DeviceGuard() {
    if (prev >= 0) cudaSetDevice(prev);
  }
};

// Launch `kernel` on `st` with programmatic stream serialisation (the kernel
// calls pdl_wait before touching global memory) and, if cluster.x > 0, that
// thread-block cluster shape.
template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem, cudaStream_t st,
                       dim3 cluster, Args... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = st;
  cudaLaunchAttribute attr[2];
  unsigned n = 0;
  attr[n].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[n].val.programmaticStreamSerializationAllowed = 1;
  ++n;
  if (cluster.x > 0) {
    attr[n].id = cudaLaunchAttributeClusterDimension;
    attr[n].val.clusterDim.x = cluster.x;
    attr[n].val.clusterDim.y = cluster.y;
    attr[n].val.clusterDim.z = cluster.z;
    ++n;
  }
  cfg.attrs = attr;
  cfg.numAttrs = n;
  count_launch();
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<KArgs>(args)...);
}
// Sets the message rmm_last_error_string() returns on the calling thread.
void set_last_error(const char* msg);

// score.cu
//  s[b][k] = sqrt(sum_i A[b][i][k]^2) · (bmode 1: sqrt(sum_j B[b][k][j]^2) with B
//  row-major [K][N]; bmode 2: sqrt(sum_j B[b][j][k]^2) with B = Kmat [N][K];
//  bmode 0: 1). One launch.
//  bmode 3: s[b][k] = sqrt(sum_i A[b][i][k]^2) · bn[b * bn_stride + k] (B not read).
//  clear_status: zero *status first (the fused calls' first kernel) and leave
//  non-finite scores to the selection to report.
cudaError_t launch_score(const MatView& A, const MatView& B, int bmode, ElemKind e, int64_t batch, float* s,
                         uint32_t* status, cudaStream_t st, const float* bn = nullptr, int64_t bn_stride = 0,
                         int clear_status = 0);
//  out[b][k] = sqrt(sum_j B[b][k][j]^2) (B row-major [K][N], view rows = K) or, with
//  b_kmajor, sqrt(sum_j B[b][j][k]^2) (B = Kmat [N][K], view rows = N, cols = K).
cudaError_t launch_b_norms(const MatView& B, int b_kmajor, ElemKind e, int64_t batch, float* out, uint32_t* status,
                           cudaStream_t st);

// f32 C tiles that the tensor-core GEMM's split-K round reduce-adds into, and
// which must therefore hold zeros before it starts: `count` tiles of
// tile_rows x tile_cols starting at tile `first_tile` of the m-fastest tile
// order (tiles_m x tiles_n per batch item), clipped to M x N.
struct SplitZero {
  float* c;
  int64_t ldc, strideC;
  int64_t M, N;
  int64_t first_tile, count;
  int32_t tiles_m, tiles_n, tile_rows, tile_cols;
};

// Scores of a few rows of A (the decode shapes) that the selection computes
// itself instead of reading them: s_k = sqrt(sum_m A[m][k]^2), times bn[k]
// when B's row norms are given (bn null: the A-only score). The sums follow
// the score kernel's order for these shapes, so the scores are the same bits.
struct RowScore {
  const void* A;  // [batch][M][K] at lda / sA elements
  int64_t lda, sA;
  int32_t M;      // <= kRowScoreMaxM
  int32_t bf16;   // 1: bf16 elements, 0: f32
  int32_t a_vec;  // A's base, lda and sA allow 16-byte loads
  const float* bn;  // [batch][K] at bn_stride, or null
  int64_t bn_stride;
};
// Largest K whose selection keeps its keys in registers, and the sizes up to
// which the selection scores A's rows itself (RowScore): at most 16 keys per
// thread and 4 rows, so that all of a thread's loads fit in flight at once.
constexpr int64_t kSelectRegisterK = 512 * 64;
constexpr int64_t kRowScoreMaxK = 512 * 16;
constexpr int32_t kRowScoreMaxM = 4;

// select.cu
//  Blocks [batch, batch + zero_blocks) of the launch zero `zero`'s tiles
//  meanwhile (zero may be null); the select itself uses one block per item.
//  late_launch: release the next kernel only once the kernel before the
//  selection has completed (the fused calls' decode route, whose GEMV needs
//  whole free SMs for its clusters).
//  rows: non-null (K <= kRowScoreMaxK): compute the scores from A's rows
//  (and write them to s) instead of reading s. clear_status: the selection is
//  the call's first kernel and its only block clears the status word first.
cudaError_t launch_select(float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx,
                          uint32_t* status, cudaStream_t st, const SplitZero* zero = nullptr,
                          bool late_launch = false, const RowScore* rows = nullptr, bool clear_status = false);

// pack.cu
//  out[b][r][t] = X[b][r][idx[b][t]] for t < k_keep, 0 for k_keep <= t < k_pad.
cudaError_t launch_pack_cols(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx,
                             int64_t k_keep, int64_t k_pad, void* out, uint32_t* status, uint64_t wait_ns,
                             cudaStream_t st);
//  out[b][t][:] = X[b][idx[b][t]][:] (kept rows, row pitch ldo >= cols, zero
//  padded to ldo columns and k_pad rows).
cudaError_t launch_pack_rows(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx,
                             int64_t k_keep, int64_t k_pad, void* out, int64_t ldo, uint32_t* status,
                             uint64_t wait_ns, cudaStream_t st);

//  out[b][r][:] = X[b][r][:] for r in idx[b], zero for the other rows r < K
//  (X.rows = K), row pitch ldo >= cols, columns cols <= j < ldo zero.
cudaError_t launch_mask_rows(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx, int64_t k_keep,
                             void* out, int64_t ldo, cudaStream_t st);

//  Both packs (A's columns, B's rows) in one launch when both take the bulk
//  paths and A's rows are at most 32 KB; *handled reports whether it did.
cudaError_t launch_pack_both(const MatView& A, const MatView& B, ElemKind e, int64_t batch, const int32_t* idx,
                             int64_t k_keep, int64_t k_pad, void* a_out, void* b_out, int64_t ldo, uint32_t* status,
                             uint64_t wait_ns, cudaStream_t st, bool* handled);

// INT8 weights with one f32 scale per output column (scale[b * s_stride + j]):
//  b_norm[b][k] = ||Wq[b][k][:] · scale||_2 (score.cu) and
//  out[b][t][j] = bf16(Wq[b][idx[b][t]][j] · scale[j]) (pack.cu, zero padded).
cudaError_t launch_b_norms_w8(const int8_t* Wq, int64_t ldw, int64_t sW, const float* scale, int64_t s_stride,
                              int64_t batch, int64_t K, int64_t N, float* out, uint32_t* status, cudaStream_t st);
cudaError_t launch_pack_rows_w8(const int8_t* Wq, int64_t ldw, int64_t sW, const float* scale, int64_t s_stride,
                                int64_t batch, int64_t N, const int32_t* idx, int64_t k_keep, int64_t k_pad,
                                void* out, int64_t ldo, cudaStream_t st);

// softmax.cu: P = softmax(scale·L) row by row (causal: key k visible to query q
// when k <= q + S_k - S_q), stored bf16 [bh][S_q][S_k], L contiguous.
//  stats[b][q] = (max of scale·log2(e)·L over visible keys, 1 / sum exp2(. - max));
//  clear_status zeroes *status first (the fused call's first kernel).
cudaError_t launch_softmax_stats(const void* L, ElemKind e, int64_t bh, int64_t S_q, int64_t S_k, float scale,
                                 int causal, float* stats, uint32_t* status, int clear_status, cudaStream_t st);
//  P from L and stats; with s_out, s_out[b][k] = ||P[b][:, k]|| · (V ? ||V[b][k, :]|| : 1)
//  over the stored bf16 values (V bf16 [bh][S_k][d] contiguous, nullable).
cudaError_t launch_softmax_score(const void* L, ElemKind e, int64_t bh, int64_t S_q, int64_t S_k, float scale,
                                 int causal, const float* stats, void* P, const void* V, int64_t d, float* s_out,
                                 uint32_t* status, cudaStream_t st);

// gemm_tc.cu (bf16 tensor cores) / gemm_simt.cu (f32 CUDA cores)
struct GemmArgs {
  const void* a;  // [batch][M][k_pad] packed, or a caller's A (lda, strideA)
  const void* b;  // b_kmajor: [batch][N][k_pad]; else [batch][k_pad][ldb]
  int b_kmajor;
  int64_t ldb;    // row pitch of the N-major B operand (elements)
  void* c;        // [batch][M][N] (ldc, strideC)
  int64_t batch, M, N, k_pad, ldc, strideC;
  // A's row pitch and batch stride (elements); the packed operands have
  // lda = k_pad and strideA = M·k_pad. The tensor-core GEMM contracts over the
  // first k_pad slices; a caller's A with K not a multiple of 64 passes
  // k_pad = K (its tensor maps read zeros past K). The CUDA-core GEMM takes
  // packed operands only.
  int64_t lda, strideA;
  // >= 0: A is causal, A[i][k] = 0 for k > i + causal_off (P of a causal
  // softmax, causal_off = S_k - S_q), so a tile of rows stops at the last key
  // its rows see; -1: dense A. Tensor-core GEMM only.
  int64_t causal_off;
  ElemKind out;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int stall_producer;
  int cta_group;
  int c_zeroed;  // 1: the tiles gemm_tc_split_zero names are already zero
  cudaEvent_t ev_start, ev_stop;  // recorded around the GEMM kernel when non-null
};
//  cta_group: 2 = 2-SM MMAs on CTA pairs (default), 1 = one SM per tile.
cudaError_t launch_gemm_tc(const GemmArgs& g, cudaStream_t st, const char** why);
//  The tiles launch_gemm_tc(g) splits along K (false: it splits none).
bool gemm_tc_split_zero(const GemmArgs& g, SplitZero* z);
cudaError_t launch_gemm_simt(const GemmArgs& g, cudaStream_t st);

// gemv.cu: C[b] = A[b][:, idx[b]] · B[b][idx[b], :] read straight from A and
// B (no packed copy) for M <= kGemvMaxRows rows of A; B row-major [K][N].
constexpr int64_t kGemvMaxRows = 16;
struct GemvArgs {
  const void* a;  // [batch][M][K] (lda, strideA)
  const void* b;  // [batch][K][N] (ldb, strideB)
  int64_t lda, strideA, ldb, strideB;
  const int32_t* idx;  // [batch][k_keep]
  int64_t k_keep;
  void* c;  // [batch][M][N] (ldc, strideC)
  int64_t ldc, strideC;
  int64_t batch, M, N;
  ElemKind in, out;
};
cudaError_t launch_gemv_gather(const GemvArgs& g, cudaStream_t st);
//  B = an INT8 weight (g.b int8, rows 4-byte aligned) whose column j is scaled
//  by scale[b * s_stride + j]; A bf16.
cudaError_t launch_gemv_gather_w8(const GemvArgs& g, const float* scale, int64_t s_stride, cudaStream_t st);

}  // namespace rmm
