// Reduced product in f32 on the CUDA cores ("Mecanismo Central" on the
// gist.science summary of "Reduced Matrix Multiplication: Input-Adaptive
// Matrix-Product Reduction for LLM Inference"), for f32 inputs: TF32 tensor
// cores round the operands to 10-bit mantissas, far outside a 1e-5 relative
// error budget, so the f32 path multiplies in full f32 with FFMA.
//
// 64x64 output tile per 256-thread CTA, each thread 4x4 outputs, 16-deep
// K slices of both packed operands staged in shared memory. Each output is
// a sequential f32 sum over t = 0 .. k_pad-1 (padding columns are zeros), so
// results are bit-reproducible.
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int ST = 64;   // output tile edge
constexpr int SK = 16;   // K slice

// B is K-major ([N][k_pad]) when b_kmajor, else N-major ([k_pad][ldb]).
__global__ void __launch_bounds__(256)
gemm_simt_kernel(const float* __restrict__ A, const float* __restrict__ Bp, int b_kmajor, int64_t ldb,
                 void* __restrict__ C, int64_t M, int64_t N, int64_t k_pad, int64_t ldc, int64_t strideC,
                 int out_bf16) {
  __shared__ float As[SK][ST + 4];
  __shared__ float Bs[SK][ST + 4];
  const int64_t b = blockIdx.z;
  const int64_t i0 = int64_t(blockIdx.y) * ST, j0 = int64_t(blockIdx.x) * ST;
  const float* Ab = A + b * M * k_pad;
  const float* Bb = Bp + (b_kmajor ? b * N * k_pad : b * k_pad * ldb);
  const int tx = threadIdx.x & 15, ty = threadIdx.x >> 4;
  pdl_trigger();
  pdl_wait();
  float acc[4][4];
#pragma unroll
  for (int a = 0; a < 4; ++a)
#pragma unroll
    for (int c = 0; c < 4; ++c) acc[a][c] = 0.f;

  for (int64_t k0 = 0; k0 < k_pad; k0 += SK) {
    // 64 rows x 16 k per operand: 4 elements per thread, k fastest for coalescing
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = threadIdx.x + q * 256;
      const int r = e >> 4, kk = e & 15;
      const int64_t gi = i0 + r;
      As[kk][r] = gi < M ? Ab[gi * k_pad + k0 + kk] : 0.f;
      if (b_kmajor) {
        const int64_t gj = j0 + r;
        Bs[kk][r] = gj < N ? Bb[gj * k_pad + k0 + kk] : 0.f;
      } else {
        const int kr = e >> 6, jc = e & 63;  // N fastest for coalescing
        const int64_t gj = j0 + jc;
        Bs[kr][jc] = gj < N ? Bb[(k0 + kr) * ldb + gj] : 0.f;
      }
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < SK; ++kk) {
      float a[4], bv[4];
#pragma unroll
      for (int q = 0; q < 4; ++q) {
        a[q] = As[kk][ty * 4 + q];
        bv[q] = Bs[kk][tx * 4 + q];
      }
#pragma unroll
      for (int x = 0; x < 4; ++x)
#pragma unroll
        for (int y = 0; y < 4; ++y) acc[x][y] = fmaf(a[x], bv[y], acc[x][y]);
    }
    __syncthreads();
  }

#pragma unroll
  for (int x = 0; x < 4; ++x) {
    const int64_t i = i0 + ty * 4 + x;
    if (i >= M) continue;
#pragma unroll
    for (int y = 0; y < 4; ++y) {
      const int64_t j = j0 + tx * 4 + y;
      if (j >= N) continue;
      if (out_bf16) {
        const uint32_t h = pack_bf16x2(acc[x][y], 0.f);
        static_cast<uint16_t*>(C)[b * strideC + i * ldc + j] = uint16_t(h & 0xFFFFu);
      } else {
        static_cast<float*>(C)[b * strideC + i * ldc + j] = acc[x][y];
      }
    }
  }
}

}  // namespace

cudaError_t launch_gemm_simt(const GemmArgs& g, cudaStream_t st) {
  if (g.batch == 0 || g.M == 0 || g.N == 0) return cudaSuccess;
  dim3 grid(unsigned((g.N + ST - 1) / ST), unsigned((g.M + ST - 1) / ST), unsigned(g.batch));
  if (g.ev_start) {
    cudaError_t e = cudaEventRecord(g.ev_start, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_pdl(gemm_simt_kernel, grid, dim3(256), 0, st, dim3(0, 0, 0),
                             static_cast<const float*>(g.a), static_cast<const float*>(g.b), g.b_kmajor, g.ldb, g.c,
                             g.M, g.N, g.k_pad, g.ldc, g.strideC, int(g.out == kBF16));
  if (e == cudaSuccess && g.ev_stop) e = cudaEventRecord(g.ev_stop, st);
  return e;
}

}  // namespace rmm
