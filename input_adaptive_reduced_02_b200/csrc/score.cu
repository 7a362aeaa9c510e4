// Slice scores for RMM ("Estratégia de Seleção" on the gist.science summary of
// "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product Reduction for
// LLM Inference": score each contraction slice by a norm, keep the top k).
//
// Two HBM-streaming kernels, both reading each input element exactly once:
//  * colsq: column sums of squares of a row-major matrix (A's columns, or the
//    columns of Kmat when B = Kmatᵀ). A CTA owns a strip of 64 bf16 (128 B)
//    columns and a contiguous chunk of rows; 8 threads cover one 128-byte row
//    segment with 16-byte loads, 32 row lanes walk the chunk. The row chunks of
//    one strip form a thread-block cluster (up to 8 CTAs) and are summed
//    through distributed shared memory by the cluster's rank-0 CTA in rank
//    order, so the result is bit-reproducible without a second launch or any
//    global scratch. The same CTA applies the score's final form.
//  * rowsq: row sums of squares (rows of a row-major B), one warp per row,
//    16-byte loads, fixed-order butterfly.
// All sums are f32 in a fixed order.
#include <cooperative_groups.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace cg = cooperative_groups;

namespace rmm {
namespace {

constexpr int kScoreThreads = 256;

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Unpack a 16-byte vector into f32 values and add their squares to acc.
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

template <typename T>
__device__ __forceinline__ float vec_sumsq(uint4 u) {
  constexpr int V = 16 / sizeof(T);
  float a[V];
#pragma unroll
  for (int v = 0; v < V; ++v) a[v] = 0.f;
  acc_sq(a, u, T{});
  float s = 0.f;
#pragma unroll
  for (int v = 0; v < V; ++v) s += a[v];
  return s;
}

// FIN: 0 store the column sum of squares; 1 out = sqrt(sum)·sqrt(out) (the
// product score, out holding the other factor's sum of squares); 2 out = sqrt(sum).
template <typename T, int FIN>
__global__ void __launch_bounds__(kScoreThreads)
colsq_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
             float* __restrict__ out, int64_t out_bstride, uint32_t* status, int vec_ok) {
  constexpr int V = 16 / sizeof(T);  // elements per 16-byte load
  constexpr int CW = 8 * V;          // strip width: 8 threads x 16 B = 128 B of a row
  __shared__ float red[32][CW + 1];
  __shared__ float part[CW];

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();

  const int64_t b = blockIdx.z;
  const T* base = X + b * bstride;
  const int tid = threadIdx.x;
  const int rl = tid >> 3;  // row lane 0..31
  const int cl = tid & 7;   // 16-byte column slot 0..7
  const int64_t c0 = int64_t(blockIdx.x) * CW + int64_t(cl) * V;
  const int64_t rows_per = (R + cs - 1) / cs;
  const int64_t r0 = int64_t(crank) * rows_per;
  const int64_t r1 = min(R, r0 + rows_per);

  float acc[V];
#pragma unroll
  for (int v = 0; v < V; ++v) acc[v] = 0.f;

  if (vec_ok && c0 + V <= C) {
    int64_t r = r0 + rl;
    for (; r + 96 < r1; r += 128) {  // four rows in flight per thread
      const uint4 u0 = ld_stream16(base + r * ld + c0);
      const uint4 u1 = ld_stream16(base + (r + 32) * ld + c0);
      const uint4 u2 = ld_stream16(base + (r + 64) * ld + c0);
      const uint4 u3 = ld_stream16(base + (r + 96) * ld + c0);
      acc_sq(acc, u0, T{});
      acc_sq(acc, u1, T{});
      acc_sq(acc, u2, T{});
      acc_sq(acc, u3, T{});
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

#pragma unroll
  for (int v = 0; v < V; ++v) red[rl][cl * V + v] = acc[v];
  __syncthreads();
  if (tid < CW) {
    float s = 0.f;
#pragma unroll 8
    for (int q = 0; q < 32; ++q) s += red[q][tid];
    part[tid] = s;
  }
  cluster.sync();  // every CTA's part[] is written and visible cluster-wide
  if (crank == 0 && tid < CW) {
    float tot = 0.f;
    for (unsigned q = 0; q < cs; ++q) tot += cluster.map_shared_rank(part, q)[tid];
    const int64_t c = int64_t(blockIdx.x) * CW + tid;
    if (c < C) {
      float* o = out + b * out_bstride + c;
      if (FIN == 0) {
        *o = tot;
      } else {
        float sc = sqrtf(tot);
        if (FIN == 1) sc *= sqrtf(*o);
        *o = sc;
        if (!isfinite(sc)) status_or(status, RMM_NONFINITE_BIT);
      }
    }
  }
  cluster.sync();  // keep shared memory alive until rank 0 has read it
}

template <typename T>
__global__ void __launch_bounds__(kScoreThreads)
rowsq_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
             float* __restrict__ out, int64_t out_bstride, int vec_ok) {
  constexpr int V = 16 / sizeof(T);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const int64_t r = int64_t(blockIdx.x) * (kScoreThreads / 32) + warp;
  const int64_t b = blockIdx.y;
  if (r >= R) return;  // whole warp leaves; no block-level barrier follows
  const T* row = X + b * bstride + r * ld;
  float acc = 0.f;
  int64_t tail = 0;
  if (vec_ok) {
    const int64_t nv = C / V;
    int64_t j = lane;
    for (; j + 96 < nv; j += 128) {
      const uint4 u0 = ld_stream16(row + j * V);
      const uint4 u1 = ld_stream16(row + (j + 32) * V);
      const uint4 u2 = ld_stream16(row + (j + 64) * V);
      const uint4 u3 = ld_stream16(row + (j + 96) * V);
      acc += vec_sumsq<T>(u0);
      acc += vec_sumsq<T>(u1);
      acc += vec_sumsq<T>(u2);
      acc += vec_sumsq<T>(u3);
    }
    for (; j < nv; j += 32) acc += vec_sumsq<T>(ld_stream16(row + j * V));
    tail = nv * V;
  }
  for (int64_t c = tail + lane; c < C; c += 32) {
    const float x = elem_to_f32(row[c]);
    acc = fmaf(x, x, acc);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) acc += __shfl_xor_sync(0xffffffffu, acc, o);
  if (lane == 0) out[b * out_bstride + r] = acc;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename T>
cudaError_t launch_colsq_t(const MatView& X, int64_t batch, float* out, int64_t out_bstride, int fin,
                           uint32_t* status, cudaStream_t st) {
  constexpr int V = 16 / sizeof(T);
  constexpr int CW = 8 * V;
  unsigned cs = 1;
  while (cs < 8 && X.rows >= int64_t(cs) * 2 * 256) cs *= 2;
  const int vec_ok = aligned16(X.ptr) && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                     (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0);
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(unsigned((X.cols + CW - 1) / CW), cs, unsigned(batch));
  cfg.blockDim = dim3(kScoreThreads, 1, 1);
  cfg.dynamicSmemBytes = 0;
  cfg.stream = st;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 1;
  attr[0].val.clusterDim.y = cs;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  const T* p = static_cast<const T*>(X.ptr);
  count_launch();
  switch (fin) {
    case 0:
      return cudaLaunchKernelEx(&cfg, colsq_kernel<T, 0>, p, X.ld, X.bstride, X.rows, X.cols, out, out_bstride,
                                status, vec_ok);
    case 1:
      return cudaLaunchKernelEx(&cfg, colsq_kernel<T, 1>, p, X.ld, X.bstride, X.rows, X.cols, out, out_bstride,
                                status, vec_ok);
    default:
      return cudaLaunchKernelEx(&cfg, colsq_kernel<T, 2>, p, X.ld, X.bstride, X.rows, X.cols, out, out_bstride,
                                status, vec_ok);
  }
}

template <typename T>
cudaError_t launch_rowsq_t(const MatView& X, int64_t batch, float* out, int64_t out_bstride, cudaStream_t st) {
  const int vec_ok = aligned16(X.ptr) && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                     (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0);
  const int64_t rows_per_cta = kScoreThreads / 32;
  dim3 grid(unsigned((X.rows + rows_per_cta - 1) / rows_per_cta), unsigned(batch), 1);
  count_launch();
  rowsq_kernel<T><<<grid, kScoreThreads, 0, st>>>(static_cast<const T*>(X.ptr), X.ld, X.bstride, X.rows, X.cols,
                                                   out, out_bstride, vec_ok);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_colsq(const MatView& X, ElemKind e, int64_t batch, float* out, int64_t out_bstride, int finalize,
                         uint32_t* status, cudaStream_t st) {
  if (batch == 0 || X.cols == 0) return cudaSuccess;
  return e == kBF16 ? launch_colsq_t<uint16_t>(X, batch, out, out_bstride, finalize, status, st)
                    : launch_colsq_t<uint32_t>(X, batch, out, out_bstride, finalize, status, st);
}

cudaError_t launch_rowsq(const MatView& X, ElemKind e, int64_t batch, float* out, int64_t out_bstride,
                         cudaStream_t st) {
  if (batch == 0 || X.rows == 0) return cudaSuccess;
  return e == kBF16 ? launch_rowsq_t<uint16_t>(X, batch, out, out_bstride, st)
                    : launch_rowsq_t<uint32_t>(X, batch, out, out_bstride, st);
}

}  // namespace rmm
