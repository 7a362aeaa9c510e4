// Slice scores for RMM ("Estratégia de Seleção" on the gist.science summary of
// "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
// LLM Inference": score each contraction slice by a norm, keep the top k).
//
// One HBM-streaming launch reads every input element once. Slices are cut
// into strips of 64 (bf16) or 32 (f32) consecutive k — 128 bytes of a row. The
// CTAs of one thread-block cluster (up to 8) share a strip:
//  * each CTA sums A[i, k]^2 over its chunk of the M rows for the strip's
//    columns (8 threads cover one 128-byte row segment with 16-byte loads, 32
//    row lanes walk the chunk, 8 loads in flight per thread);
//  * in product mode each CTA also sums its share of B's part of the score:
//    whole rows B[k, :] of the strip (one warp per row), or, when B is given
//    as Kmat [N][K], Kmat's columns exactly like A's;
//  * the cluster's rank-0 CTA adds the CTAs' partial sums in rank order
//    through distributed shared memory and writes
//    s_k = sqrt(sum_i A[i,k]^2) · sqrt(sum_j B[k,j]^2)  (or sqrt of A's sum).
// Fixed summation order everywhere: bit-reproducible, no atomics, no scratch.
#include <algorithm>
#include <cooperative_groups.h>

#include "int8_convert.cuh"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace cg = cooperative_groups;

namespace rmm {
namespace {

constexpr int kScoreThreads = 256;
constexpr unsigned kMaxCluster = 8;  // CTAs sharing one strip (portable cluster size; 16 measured slower)
constexpr int kUnroll = 8;

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Add the squares of a 16-byte vector's elements to acc (one accumulator per element).
__device__ __forceinline__ void acc_sq(float (&acc)[8], uint4 u, uint16_t) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float lo = __uint_as_float(w[j] << 16);
    const float hi = __uint_as_float(w[j] & 0xFFFF0000u);
    acc[2 * j] = fmaf(lo, lo, acc[2 * j]);
    acc[2 * j + 1] = fmaf(hi, hi, acc[2 * j + 1]);
  }
}
__device__ __forceinline__ void acc_sq(float (&acc)[4], uint4 u, uint32_t) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    const float x = __uint_as_float(w[j]);
    acc[j] = fmaf(x, x, acc[j]);
  }
}

// Column sums of squares of rows [r0, r1) of a row-major matrix, for the V
// columns starting at c0 that this thread owns; rows rl, rl+32, ... in order.
template <typename T>
__device__ __forceinline__ void colsq_rows(const T* __restrict__ base, int64_t ld, int64_t r0, int64_t r1,
                                           int64_t c0, int64_t C, int rl, bool vec_ok,
                                           float (&acc)[16 / sizeof(T)]) {
  constexpr int V = 16 / sizeof(T);
  if (vec_ok && c0 + V <= C) {
    int64_t r = r0 + rl;
    for (; r + 32 * (kUnroll - 1) < r1; r += 32 * kUnroll) {
      uint4 u[kUnroll];
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) u[j] = ld_stream16(base + (r + 32 * j) * ld + c0);
#pragma unroll
      for (int j = 0; j < kUnroll; ++j) acc_sq(acc, u[j], T{});
    }
    for (; r < r1; r += 32) acc_sq(acc, ld_stream16(base + r * ld + c0), T{});
  } else {
    for (int64_t r = r0 + rl; r < r1; r += 32) {
#pragma unroll
      for (int v = 0; v < V; ++v) {
        if (c0 + v < C) {
          const float x = elem_to_f32(base[r * ld + c0 + v]);
          acc[v] = fmaf(x, x, acc[v]);
        }
      }
    }
  }
}

// Sum of squares of one row of length C (whole warp; result valid in lane 0).
template <typename T>
__device__ __forceinline__ float rowsq_warp(const T* __restrict__ row, int64_t C, bool vec_ok, int lane) {
  constexpr int V = 16 / sizeof(T);
  float a[V];
#pragma unroll
  for (int v = 0; v < V; ++v) a[v] = 0.f;
  int64_t tail = 0;
  if (vec_ok) {
    const int64_t nv = C / V;
    int64_t j = lane;
    for (; j + 32 * (kUnroll - 1) < nv; j += 32 * kUnroll) {
      uint4 u[kUnroll];
#pragma unroll
      for (int q = 0; q < kUnroll; ++q) u[q] = ld_stream16(row + (j + 32 * q) * V);
#pragma unroll
      for (int q = 0; q < kUnroll; ++q) acc_sq(a, u[q], T{});
    }
    for (; j < nv; j += 32) acc_sq(a, ld_stream16(row + j * V), T{});
    tail = nv * V;
  }
  float acc = 0.f;
#pragma unroll
  for (int v = 0; v < V; ++v) acc += a[v];
  for (int64_t c = tail + lane; c < C; c += 32) {
    const float x = elem_to_f32(row[c]);
    acc = fmaf(x, x, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  return acc;
}

// BMODE: 0 = A-only score; 1 = B row-major [K][N] (rows of the strip);
//        2 = B given as Kmat [N][K] (columns of the strip);
//        3 = B's norms given (bn[b * bn_stride + k]).
template <typename T, int BMODE>
__global__ void __launch_bounds__(kScoreThreads)
score_kernel(const T* __restrict__ A, int64_t lda, int64_t sA, int64_t M, int64_t K,
             const T* __restrict__ B, int64_t ldb, int64_t sB, int64_t N,
             const float* __restrict__ bn, int64_t bn_stride,
             float* __restrict__ s, uint32_t* status, int a_vec, int b_vec, int clear_status) {
  constexpr int V = 16 / sizeof(T);
  constexpr int CW = 8 * V;
  __shared__ float red[32][CW + 1];
  __shared__ float partA[CW];
  __shared__ float partB[CW];

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();
  const int64_t b = blockIdx.z;
  const int tid = threadIdx.x, rl = tid >> 3, cl = tid & 7;
  const int warp = tid >> 5, lane = tid & 31;
  const int64_t strip0 = int64_t(blockIdx.x) * CW;
  const int64_t c0 = strip0 + int64_t(cl) * V;
  pdl_trigger();
  pdl_wait();
  // clear_status: the first kernel of a fused call clears the status word
  // (every later kernel of the call waits for this one), and non-finite scores
  // are then reported by the selection, which reads them all
  if (clear_status && blockIdx.x == 0 && blockIdx.y == 0 && blockIdx.z == 0 && threadIdx.x == 0 && status)
    *status = 0u;

  // ---- A: column sums over this CTA's rows
  {
    const int64_t per = (M + cs - 1) / cs;
    const int64_t r0 = int64_t(crank) * per, r1 = min(M, r0 + per);
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    colsq_rows<T>(A + b * sA, lda, r0, r1, c0, K, rl, a_vec != 0, acc);
#pragma unroll
    for (int v = 0; v < V; ++v) red[rl][cl * V + v] = acc[v];
    __syncthreads();
    if (tid < CW) {
      float t = 0.f;
      for (int q = 0; q < 32; ++q) t += red[q][tid];
      partA[tid] = t;
    }
    __syncthreads();
  }
  // ---- B's share of the score
  if constexpr (BMODE == 2) {
    const int64_t per = (N + cs - 1) / cs;
    const int64_t r0 = int64_t(crank) * per, r1 = min(N, r0 + per);
    float acc[V];
#pragma unroll
    for (int v = 0; v < V; ++v) acc[v] = 0.f;
    colsq_rows<T>(B + b * sB, ldb, r0, r1, c0, K, rl, b_vec != 0, acc);
#pragma unroll
    for (int v = 0; v < V; ++v) red[rl][cl * V + v] = acc[v];
    __syncthreads();
    if (tid < CW) {
      float t = 0.f;
      for (int q = 0; q < 32; ++q) t += red[q][tid];
      partB[tid] = t;
    }
  } else if constexpr (BMODE == 1) {
    if (tid < CW) partB[tid] = 0.f;
    __syncthreads();
    // rows strip0 + j, j = crank, crank + cs, ...: one warp per row
    const T* Bb = B + b * sB;
    for (int j = int(crank) + warp * int(cs); j < CW; j += int(cs) * (kScoreThreads / 32)) {
      const int64_t k = strip0 + j;
      if (k >= K) break;
      const float t = rowsq_warp<T>(Bb + k * ldb, N, b_vec != 0, lane);
      if (lane == 0) partB[j] = t;
    }
  }
  cluster.sync();  // every CTA's partial sums are written and visible cluster-wide
  if (crank == 0 && tid < CW) {
    const int64_t c = strip0 + tid;
    float ssa = 0.f, ssb = 0.f;
    for (unsigned q = 0; q < cs; ++q) {
      ssa += cluster.map_shared_rank(partA, q)[tid];
      if constexpr (BMODE == 1 || BMODE == 2) ssb += cluster.map_shared_rank(partB, q)[tid];
    }
    if (c < K) {
      float sc = sqrtf(ssa);
      if constexpr (BMODE == 1 || BMODE == 2) sc *= sqrtf(ssb);
      if constexpr (BMODE == 3) sc *= bn[b * bn_stride + c];
      s[b * K + c] = sc;
      if (!clear_status && !isfinite(sc)) status_or(status, RMM_NONFINITE_BIT);
    }
  }
  cluster.sync();  // keep shared memory alive until rank 0 has read it
}

// b_norm[b][k] = sqrt(sum_j B[b][k][j]^2) for a row-major B: one warp per row,
// the same per-row sum as the score kernel's product mode (bit-identical).
template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
bnorm_rows_kernel(const T* __restrict__ B, int64_t ldb, int64_t sB, int64_t K, int64_t N, int b_vec,
                  float* __restrict__ out, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.y;
  constexpr int kWarps = kScoreThreads / 32;
  for (int64_t k = int64_t(blockIdx.x) * kWarps + warp; k < K; k += int64_t(gridDim.x) * kWarps) {
    const float t = rowsq_warp<T>(B + b * sB + k * ldb, N, b_vec != 0, lane);
    if (lane == 0) {
      const float v = sqrtf(t);
      out[b * K + k] = v;
      if (!isfinite(v)) status_or(status, RMM_NONFINITE_BIT);
    }
  }
}

// b_norm[b][k] = sqrt(sum_j (Wq[b][k][j] · scale[j])^2): the row norms of a
// per-column-scaled INT8 weight (one warp per row; 16 weights per load when
// the rows and the scales are 16-byte aligned).
__global__ void __launch_bounds__(kScoreThreads)
bnorm_rows_w8_kernel(const int8_t* __restrict__ Wq, int64_t ldw, int64_t sW, const float* __restrict__ scale,
                     int64_t s_stride, int64_t K, int64_t N, int vec, float* __restrict__ out, uint32_t* status) {
  pdl_trigger();
  pdl_wait();
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t b = blockIdx.y;
  constexpr int kWarps = kScoreThreads / 32;
  const float* sc = scale + b * s_stride;
  for (int64_t k = int64_t(blockIdx.x) * kWarps + warp; k < K; k += int64_t(gridDim.x) * kWarps) {
    const int8_t* row = Wq + b * sW + k * ldw;
    float acc = 0.f;
    int64_t tail = 0;
    if (vec) {
      const int64_t nv = N / 16;
      for (int64_t j = lane; j < nv; j += 32) {
        const int4 q = *reinterpret_cast<const int4*>(row + 16 * j);
        const float4* s4 = reinterpret_cast<const float4*>(sc + 16 * j);
        const uint32_t w[4] = {uint32_t(q.x), uint32_t(q.y), uint32_t(q.z), uint32_t(q.w)};
#pragma unroll
        for (int h = 0; h < 4; ++h) {
          const float4 sv = s4[h];
          float v0, v1, v2, v3;
          s8x4_to_f32(w[h], v0, v1, v2, v3);
          v0 *= sv.x, v1 *= sv.y, v2 *= sv.z, v3 *= sv.w;
          acc = fmaf(v0, v0, acc);
          acc = fmaf(v1, v1, acc);
          acc = fmaf(v2, v2, acc);
          acc = fmaf(v3, v3, acc);
        }
      }
      tail = nv * 16;
    }
    for (int64_t c = tail + lane; c < N; c += 32) {
      const float v = float(row[c]) * sc[c];
      acc = fmaf(v, v, acc);
    }
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
    if (lane == 0) {
      const float v = sqrtf(acc);
      out[b * K + k] = v;
      if (!isfinite(v)) status_or(status, RMM_NONFINITE_BIT);
    }
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

// 16-byte loads for B: base, rows and batch items 16-byte aligned.
template <typename T>
int b_vec_ok(const MatView& B, int64_t batch) {
  return aligned16(B.ptr) && (B.ld * int64_t(sizeof(T))) % 16 == 0 &&
         (batch == 1 || (B.bstride * int64_t(sizeof(T))) % 16 == 0);
}

template <typename T, int BMODE>
cudaError_t launch_t(const MatView& A, const MatView& B, int64_t batch, float* s, uint32_t* status,
                     cudaStream_t st, const float* bn = nullptr, int64_t bn_stride = 0, int clear_status = 0) {
  constexpr int V = 16 / sizeof(T);
  constexpr int CW = 8 * V;
  const int64_t K = A.cols;
  // Rows each CTA streams: A's chunk plus its share of B. Aim for >= 256 rows
  // of 128-byte segments per CTA before splitting a strip further.
  const int64_t work_rows =
      A.rows + (BMODE == 2 ? B.rows : 0) + (BMODE == 1 ? CW * B.cols * int64_t(sizeof(T)) / 128 : 0);
  unsigned cs = 1;
  while (cs < kMaxCluster && work_rows >= int64_t(cs) * 2 * 256) cs *= 2;
  const int a_vec = aligned16(A.ptr) && (A.ld * int64_t(sizeof(T))) % 16 == 0 &&
                    (batch == 1 || (A.bstride * int64_t(sizeof(T))) % 16 == 0);
  const int b_vec = (BMODE == 0 || BMODE == 3) ? 0 : b_vec_ok<T>(B, batch);
  const int64_t N = BMODE == 2 ? B.rows : B.cols;
  return launch_pdl(score_kernel<T, BMODE>, dim3(unsigned((K + CW - 1) / CW), cs, unsigned(batch)),
                    dim3(kScoreThreads), 0, st, dim3(1, cs, 1), static_cast<const T*>(A.ptr), A.ld, A.bstride, A.rows, K,
                    static_cast<const T*>(B.ptr), B.ld, B.bstride, N, bn, bn_stride, s, status, a_vec, b_vec,
                    clear_status);
}

template <typename T>
cudaError_t launch_bnorm_rows(const MatView& B, int64_t batch, float* out, uint32_t* status, cudaStream_t st) {
  constexpr int kWarps = kScoreThreads / 32;
  const int64_t ctas = std::min<int64_t>((B.rows + kWarps - 1) / kWarps, 148 * 8);
  return launch_pdl(bnorm_rows_kernel<T>, dim3(unsigned(ctas), unsigned(batch)), dim3(kScoreThreads), 0, st,
                    dim3(0, 0, 0), static_cast<const T*>(B.ptr), B.ld, B.bstride, B.rows, B.cols,
                    b_vec_ok<T>(B, batch), out, status);
}

}  // namespace

cudaError_t launch_score(const MatView& A, const MatView& B, int bmode, ElemKind e, int64_t batch, float* s,
                         uint32_t* status, cudaStream_t st, const float* bn, int64_t bn_stride, int clear_status) {
  if (batch == 0 || A.cols == 0) return cudaSuccess;
  const int cs = clear_status;
  if (e == kBF16) {
    switch (bmode) {
      case 0: return launch_t<uint16_t, 0>(A, B, batch, s, status, st, nullptr, 0, cs);
      case 1: return launch_t<uint16_t, 1>(A, B, batch, s, status, st, nullptr, 0, cs);
      case 2: return launch_t<uint16_t, 2>(A, B, batch, s, status, st, nullptr, 0, cs);
      default: return launch_t<uint16_t, 3>(A, B, batch, s, status, st, bn, bn_stride, cs);
    }
  }
  switch (bmode) {
    case 0: return launch_t<uint32_t, 0>(A, B, batch, s, status, st, nullptr, 0, cs);
    case 1: return launch_t<uint32_t, 1>(A, B, batch, s, status, st, nullptr, 0, cs);
    case 2: return launch_t<uint32_t, 2>(A, B, batch, s, status, st, nullptr, 0, cs);
    default: return launch_t<uint32_t, 3>(A, B, batch, s, status, st, bn, bn_stride, cs);
  }
}

cudaError_t launch_b_norms(const MatView& B, int b_kmajor, ElemKind e, int64_t batch, float* out, uint32_t* status,
                           cudaStream_t st) {
  if (batch == 0 || B.rows == 0 || B.cols == 0) return cudaSuccess;
  if (b_kmajor) {  // column norms of Kmat [N][K]: the A-only score of Kmat
    const MatView none{nullptr, 0, 0, 0, 0};
    return e == kBF16 ? launch_t<uint16_t, 0>(B, none, batch, out, status, st)
                      : launch_t<uint32_t, 0>(B, none, batch, out, status, st);
  }
  return e == kBF16 ? launch_bnorm_rows<uint16_t>(B, batch, out, status, st)
                    : launch_bnorm_rows<uint32_t>(B, batch, out, status, st);
}

cudaError_t launch_b_norms_w8(const int8_t* Wq, int64_t ldw, int64_t sW, const float* scale, int64_t s_stride,
                              int64_t batch, int64_t K, int64_t N, float* out, uint32_t* status, cudaStream_t st) {
  if (batch == 0 || K == 0 || N == 0) return cudaSuccess;
  constexpr int kWarps = kScoreThreads / 32;
  const int64_t ctas = std::min<int64_t>((K + kWarps - 1) / kWarps, 148 * 8);
  const int vec = aligned16(Wq) && ldw % 16 == 0 && (batch == 1 || sW % 16 == 0) && aligned16(scale) &&
                  (batch == 1 || s_stride % 4 == 0);
  return launch_pdl(bnorm_rows_w8_kernel, dim3(unsigned(ctas), unsigned(batch)), dim3(kScoreThreads), 0, st,
                    dim3(0, 0, 0), Wq, ldw, sW, scale, s_stride, K, N, vec, out, status);
}

}  // namespace rmm
