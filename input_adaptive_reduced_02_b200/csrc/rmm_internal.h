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
// Sets the message rmm_last_error_string() returns on the calling thread.
void set_last_error(const char* msg);

// score.cu
//  Column sums of squares of X (rows × cols, per batch item), combined per
//  `finalize`: 0 = store the sum in out; 1 = out = sqrt(sum) * sqrt(out);
//  2 = out = sqrt(sum).
cudaError_t launch_colsq(const MatView& X, ElemKind e, int64_t batch, float* out, int64_t out_bstride,
                         int finalize, uint32_t* status, cudaStream_t st);
//  Row sums of squares of X stored in out (one per row).
cudaError_t launch_rowsq(const MatView& X, ElemKind e, int64_t batch, float* out, int64_t out_bstride,
                         cudaStream_t st);

// select.cu
cudaError_t launch_select(const float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx,
                          uint32_t* status, cudaStream_t st);

// pack.cu
//  out[b][r][t] = X[b][r][idx[b][t]] for t < k_keep, 0 for k_keep <= t < k_pad.
cudaError_t launch_pack_cols(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx,
                             int64_t k_keep, int64_t k_pad, void* out, cudaStream_t st);
//  out[b][n][t] = X[b][idx[b][t]][n] (kept rows, transposed), zero padded to k_pad.
cudaError_t launch_pack_rows_t(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx,
                               int64_t k_keep, int64_t k_pad, void* out, cudaStream_t st);

// gemm_tc.cu (bf16 tensor cores) / gemm_simt.cu (f32 CUDA cores)
struct GemmArgs {
  const void* a;  // [batch][M][k_pad]
  const void* b;  // [batch][N][k_pad]
  void* c;        // [batch][M][N] (ldc, strideC)
  int64_t batch, M, N, k_pad, ldc, strideC;
  ElemKind out;
  uint32_t* status;
  uint64_t wait_limit_ns;
  int stall_producer;
};
cudaError_t launch_gemm_tc(const GemmArgs& g, cudaStream_t st, const char** why);
cudaError_t launch_gemm_simt(const GemmArgs& g, cudaStream_t st);

}  // namespace rmm
