// Packing the kept slices for RMM ("Mecanismo Central" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference": the reduced product is A[:, I]·B[I, :]).
//
// Both packed operands are written K-major (the kept slice index t is the
// contiguous dimension), zero-padded to k_pad = ceil(k/64)·64, which is the
// layout the tensor-core GEMM's TMA loads consume with 128-byte swizzle:
//  * pack_cols: out[r][t] = X[r][idx[t]] — column compaction of a row-major
//    matrix (A, or Kmat for Q·Kᵀ). Kept columns are spread over every 32-byte
//    sector, so a CTA streams whole rows into shared memory with 16-byte loads
//    and gathers from there; the packed rows leave as 16-byte stores.
//  * pack_rows_t: out[n][t] = X[idx[t]][n] — gather of kept rows of a
//    row-major B, transposed through a padded shared-memory tile so that both
//    the row reads and the packed writes are whole 128-byte lines.
// Pure bit copies; no arithmetic.
#include <algorithm>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kPackThreads = 256;

__device__ __forceinline__ uint4 ld_stream16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

template <typename T>
union Vec16 {
  uint4 u;
  T e[16 / sizeof(T)];
};

// rows_per_cta rows of X staged in shared memory, then gathered.
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_cols_smem_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
                      const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                      int rows_per_cta, int vec_ok) {
  constexpr int V = 16 / sizeof(T);
  extern __shared__ __align__(16) unsigned char pack_smem[];
  T* srow = reinterpret_cast<T*>(pack_smem);
  const int64_t b = blockIdx.y;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_cta;
  if (r0 >= R) return;
  const int nr = int(min(int64_t(rows_per_cta), R - r0));
  const T* src = X + b * bstride + r0 * ld;
  const int32_t* ib = idx + b * k_keep;
  T* dst = out + (b * R + r0) * k_pad;

  if (vec_ok) {  // C % V == 0 and rows 16-byte aligned
    const int64_t nvr = C / V;
    for (int rr = 0; rr < nr; ++rr) {
      const uint4* s4 = reinterpret_cast<const uint4*>(src + rr * ld);
      uint4* d4 = reinterpret_cast<uint4*>(srow + rr * C);
      for (int64_t v = threadIdx.x; v < nvr; v += kPackThreads) d4[v] = ld_stream16(s4 + v);
    }
  } else {
    for (int rr = 0; rr < nr; ++rr)
      for (int64_t c = threadIdx.x; c < C; c += kPackThreads) srow[rr * C + c] = src[rr * ld + c];
  }
  __syncthreads();

  const int64_t ng = k_pad / V;
  for (int rr = 0; rr < nr; ++rr) {
    const T* row = srow + rr * C;
    for (int64_t g = threadIdx.x; g < ng; g += kPackThreads) {
      const int64_t t0 = g * V;
      Vec16<T> v;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int64_t t = t0 + j;
        v.e[j] = t < k_keep ? row[__ldg(ib + t)] : T(0);
      }
      reinterpret_cast<uint4*>(dst + rr * k_pad)[g] = v.u;
    }
  }
}

// Rows too long for shared memory: gather straight from global memory.
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_cols_direct_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R,
                        const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out) {
  constexpr int V = 16 / sizeof(T);
  const int64_t b = blockIdx.y;
  const int64_t r = blockIdx.x;
  if (r >= R) return;
  const T* row = X + b * bstride + r * ld;
  const int32_t* ib = idx + b * k_keep;
  T* dst = out + (b * R + r) * k_pad;
  for (int64_t g = threadIdx.x; g < k_pad / V; g += kPackThreads) {
    Vec16<T> v;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int64_t t = g * V + j;
      v.e[j] = t < k_keep ? row[__ldg(ib + t)] : T(0);
    }
    reinterpret_cast<uint4*>(dst)[g] = v.u;
  }
}

// 64 kept rows x 64 columns per CTA, transposed through shared memory.
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_rows_t_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t N,
                   const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out, int vec_ok) {
  constexpr int V = 16 / sizeof(T);
  constexpr int TT = 64;      // kept rows (t) per tile
  constexpr int TN = 64;      // columns (n) per tile
  constexpr int P = TN + V;   // padded pitch, keeps rows 16-byte aligned
  __shared__ __align__(16) T tile[TT][P];
  const int64_t b = blockIdx.z;
  const int64_t t0 = int64_t(blockIdx.x) * TT;
  const int64_t n0 = int64_t(blockIdx.y) * TN;
  const T* src = X + b * bstride;
  const int32_t* ib = idx + b * k_keep;

  constexpr int TPR = TN / V;           // threads per tile row
  constexpr int RPP = kPackThreads / TPR;
  const int cq = threadIdx.x % TPR, rq = threadIdx.x / TPR;
  for (int tt = rq; tt < TT; tt += RPP) {
    const int64_t t = t0 + tt;
    const int64_t n = n0 + int64_t(cq) * V;
    Vec16<T> v;
    v.u = make_uint4(0u, 0u, 0u, 0u);
    if (t < k_keep) {
      const T* p = src + int64_t(__ldg(ib + t)) * ld + n;
      if (vec_ok && n + V <= N) {
        v.u = ld_stream16(p);
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) v.e[j] = (n + j < N) ? p[j] : T(0);
      }
    }
    *reinterpret_cast<uint4*>(&tile[tt][cq * V]) = v.u;
  }
  __syncthreads();

  constexpr int TPO = TT / V;           // threads per packed output row
  constexpr int OPP = kPackThreads / TPO;
  const int oq = threadIdx.x % TPO, orow = threadIdx.x / TPO;
  for (int nn = orow; nn < TN; nn += OPP) {
    const int64_t n = n0 + nn;
    if (n >= N) break;
    Vec16<T> v;
#pragma unroll
    for (int j = 0; j < V; ++j) v.e[j] = tile[oq * V + j][nn];
    *reinterpret_cast<uint4*>(out + (b * N + n) * k_pad + t0 + oq * V) = v.u;
  }
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

constexpr size_t kPackSmemRowsBudget = 32 * 1024;   // several short rows per CTA
constexpr size_t kPackSmemMax = 112 * 1024;         // one long row per CTA, 2 CTAs/SM

template <typename T>
cudaError_t launch_pack_cols_t(const MatView& X, int64_t batch, const int32_t* idx, int64_t k_keep,
                               int64_t k_pad, void* out, cudaStream_t st) {
  constexpr int V = 16 / sizeof(T);
  const size_t row_bytes = size_t(X.cols) * sizeof(T);
  const T* p = static_cast<const T*>(X.ptr);
  T* o = static_cast<T*>(out);
  if (row_bytes > kPackSmemMax) {
    dim3 grid(unsigned(X.rows), unsigned(batch), 1);
    count_launch();
    pack_cols_direct_kernel<T><<<grid, kPackThreads, 0, st>>>(p, X.ld, X.bstride, X.rows, idx, k_keep, k_pad, o);
    return cudaGetLastError();
  }
  int rows_per_cta = 1;
  if (row_bytes <= kPackSmemRowsBudget) rows_per_cta = int(std::min<size_t>(8, kPackSmemRowsBudget / std::max<size_t>(row_bytes, 1)));
  const size_t smem = size_t(rows_per_cta) * row_bytes;
  const int vec_ok = aligned16(X.ptr) && X.cols % V == 0 && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                     (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0);
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(pack_cols_smem_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kPackSmemMax));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  dim3 grid(unsigned((X.rows + rows_per_cta - 1) / rows_per_cta), unsigned(batch), 1);
  count_launch();
  pack_cols_smem_kernel<T><<<grid, kPackThreads, smem, st>>>(p, X.ld, X.bstride, X.rows, X.cols, idx, k_keep, k_pad,
                                                             o, rows_per_cta, vec_ok);
  return cudaGetLastError();
}

template <typename T>
cudaError_t launch_pack_rows_t_t(const MatView& X, int64_t batch, const int32_t* idx, int64_t k_keep, int64_t k_pad,
                                 void* out, cudaStream_t st) {
  const int vec_ok = aligned16(X.ptr) && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                     (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0);
  dim3 grid(unsigned(k_pad / 64), unsigned((X.cols + 63) / 64), unsigned(batch));
  count_launch();
  pack_rows_t_kernel<T><<<grid, kPackThreads, 0, st>>>(static_cast<const T*>(X.ptr), X.ld, X.bstride, X.cols, idx,
                                                        k_keep, k_pad, static_cast<T*>(out), vec_ok);
  return cudaGetLastError();
}

}  // namespace

cudaError_t launch_pack_cols(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx, int64_t k_keep,
                             int64_t k_pad, void* out, cudaStream_t st) {
  if (batch == 0 || X.rows == 0) return cudaSuccess;
  return e == kBF16 ? launch_pack_cols_t<uint16_t>(X, batch, idx, k_keep, k_pad, out, st)
                    : launch_pack_cols_t<uint32_t>(X, batch, idx, k_keep, k_pad, out, st);
}

cudaError_t launch_pack_rows_t(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx, int64_t k_keep,
                               int64_t k_pad, void* out, cudaStream_t st) {
  if (batch == 0 || X.cols == 0) return cudaSuccess;
  return e == kBF16 ? launch_pack_rows_t_t<uint16_t>(X, batch, idx, k_keep, k_pad, out, st)
                    : launch_pack_rows_t_t<uint32_t>(X, batch, idx, k_keep, k_pad, out, st);
}

}  // namespace rmm
