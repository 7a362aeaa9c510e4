// Packing the kept slices for RMM ("Mecanismo Central" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference": the reduced product is A[:, I]·B[I, :]).
//
//  * pack_cols: out[r][t] = X[r][idx[t]] — column compaction of a row-major
//    matrix (A; Kmat for Q·Kᵀ). Kept columns are spread over every 32-byte
//    sector, so whole rows are staged in shared memory by bulk-async (TMA)
//    copies, one thread issuing all of a CTA's row copies at once; the CTA
//    then gathers through idx and writes 16-byte vectors. Padding columns
//    k <= t < k_pad are written as zeros. Output is K-major, the layout the
//    tensor-core GEMM reads for A (and for B when B is given as Kmat).
//  * pack_rows: out[t][:] = X[idx[t]][:] — the kept rows of a row-major B,
//    copied as whole rows: bulk-async loads into shared memory, bulk-async
//    stores back out, no register traffic. Padding rows are zeros. The GEMM
//    reads this operand N-major.
// Pure bit copies. Rows that are not 16-byte aligned take plain-load paths.
#include <algorithm>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kPackThreads = 256;
constexpr size_t kStageBytes = 32 * 1024;   // shared-memory rows per CTA (short rows)
constexpr size_t kStageMax = 112 * 1024;    // one long row per CTA, two CTAs per SM
constexpr size_t kSmemAttr = kStageMax + kStageBytes;  // + staged kept indices

template <typename T>
union Vec16 {
  uint4 u;
  T e[16 / sizeof(T)];
};

__device__ __forceinline__ void bulk_load(void* smem_dst, const void* gsrc, uint32_t bytes, uint64_t* bar) {
  asm volatile(
      "cp.async.bulk.shared::cluster.global.mbarrier::complete_tx::bytes [%0], [%1], %2, [%3];"
      ::"r"(smem_addr(smem_dst)), "l"(gsrc), "r"(bytes), "r"(smem_addr(bar))
      : "memory");
}

__device__ __forceinline__ void bulk_store(void* gdst, const void* smem_src, uint32_t bytes) {
  asm volatile("cp.async.bulk.global.shared::cta.bulk_group [%0], [%1], %2;"
               ::"l"(gdst), "r"(smem_addr(smem_src)), "r"(bytes)
               : "memory");
}

// Wait for this CTA's bulk loads; every thread polls, bounded. On a timeout the
// status bit is set and the CTA waits once more (also bounded) so that no copy
// is still writing shared memory when it exits.
__device__ __forceinline__ bool wait_loads(uint64_t* bar, uint64_t limit_ns, uint32_t* status, int* never) {
  if (mbar_wait_bounded(bar, 0, limit_ns, never)) return true;
  if (threadIdx.x == 0) status_or(status, RMM_TIMEOUT_BIT);
  mbar_wait_bounded(bar, 0, limit_ns, never);
  return false;
}

// Gather kept columns of nr staged rows; ib points at the kept indices (in
// shared memory or global memory, 16-byte aligned).
template <typename T>
__device__ __forceinline__ void gather_rows(const T* srow, int nr, int64_t C, const int32_t* ib, int64_t k_keep,
                                            int64_t k_pad, T* dst) {
  constexpr int V = 16 / sizeof(T);
  const int64_t ng = k_pad / V;
  for (int rr = 0; rr < nr; ++rr) {
    const T* row = srow + rr * C;
    for (int64_t g = threadIdx.x; g < ng; g += kPackThreads) {
      const int64_t t0 = g * V;
      Vec16<T> v;
      if (t0 + V <= k_keep) {
        const int4 i0 = *reinterpret_cast<const int4*>(ib + t0);
        if constexpr (V == 8) {
          const int4 i1 = *reinterpret_cast<const int4*>(ib + t0 + 4);
          v.e[0] = row[i0.x]; v.e[1] = row[i0.y]; v.e[2] = row[i0.z]; v.e[3] = row[i0.w];
          v.e[4] = row[i1.x]; v.e[5] = row[i1.y]; v.e[6] = row[i1.z]; v.e[7] = row[i1.w];
        } else {
          v.e[0] = row[i0.x]; v.e[1] = row[i0.y]; v.e[2] = row[i0.z]; v.e[3] = row[i0.w];
        }
      } else {
#pragma unroll
        for (int j = 0; j < V; ++j) {
          const int64_t t = t0 + j;
          v.e[j] = t < k_keep ? row[ib[t]] : T(0);
        }
      }
      reinterpret_cast<uint4*>(dst + rr * k_pad)[g] = v.u;
    }
  }
}

// Rows (and, when idx_in_smem, the kept indices) staged by bulk-async copies
// (rows 16-byte aligned, C·e a multiple of 16; idx 16-byte aligned).
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_cols_bulk_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
                      const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                      int rows_per_cta, int idx_in_smem, uint32_t* status, uint64_t wait_ns) {
  extern __shared__ __align__(128) unsigned char pack_smem[];
  __shared__ uint64_t bar;
  __shared__ int never;
  T* srow = reinterpret_cast<T*>(pack_smem);
  int32_t* sidx = reinterpret_cast<int32_t*>(pack_smem + size_t(rows_per_cta) * C * sizeof(T));
  const int64_t b = blockIdx.y;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_cta;
  const int nr = int(min(int64_t(rows_per_cta), R - r0));
  const T* src = X + b * bstride + r0 * ld;
  const int32_t* gidx = idx + b * k_keep;
  const int64_t idx_bulk = idx_in_smem ? (k_keep & ~int64_t(3)) : 0;  // whole 16-byte groups
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    never = 0;
    fence_mbar_init();
  }
  pdl_trigger();
  pdl_wait();
  __syncthreads();
  if (threadIdx.x == 0) {
    const uint32_t row_bytes = uint32_t(C * sizeof(T));
    mbar_arrive_expect_tx(&bar, row_bytes * uint32_t(nr) + uint32_t(idx_bulk * 4));
    for (int rr = 0; rr < nr; ++rr) bulk_load(srow + rr * C, src + rr * ld, row_bytes, &bar);
    if (idx_bulk > 0) bulk_load(sidx, gidx, uint32_t(idx_bulk * 4), &bar);
  }
  if (idx_in_smem)
    for (int64_t t = idx_bulk + threadIdx.x; t < k_keep; t += kPackThreads) sidx[t] = gidx[t];
  wait_loads(&bar, wait_ns, status, &never);
  __syncthreads();
  gather_rows(srow, nr, C, idx_in_smem ? sidx : gidx, k_keep, k_pad, out + (b * R + r0) * k_pad);
}

// Any alignment: rows staged with plain loads (eight in flight per thread).
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_cols_plain_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
                       const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                       int rows_per_cta) {
  constexpr int V = 16 / sizeof(T);
  extern __shared__ __align__(128) unsigned char pack_smem[];
  T* srow = reinterpret_cast<T*>(pack_smem);
  const int64_t b = blockIdx.y;
  const int64_t r0 = int64_t(blockIdx.x) * rows_per_cta;
  const int nr = int(min(int64_t(rows_per_cta), R - r0));
  const T* src = X + b * bstride + r0 * ld;
  pdl_trigger();
  pdl_wait();
  for (int rr = 0; rr < nr; ++rr) {
    for (int64_t c0 = threadIdx.x; c0 < C; c0 += kPackThreads * 8) {
      T v[8];
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t c = c0 + int64_t(j) * kPackThreads;
        v[j] = c < C ? src[rr * ld + c] : T(0);
      }
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        const int64_t c = c0 + int64_t(j) * kPackThreads;
        if (c < C) srow[rr * C + c] = v[j];
      }
    }
  }
  __syncthreads();
  const int32_t* ib = idx + b * k_keep;
  T* dst = out + (b * R + r0) * k_pad;
  for (int rr = 0; rr < nr; ++rr) {
    const T* row = srow + rr * C;
    for (int64_t g = threadIdx.x; g < k_pad / V; g += kPackThreads) {
      Vec16<T> v;
#pragma unroll
      for (int j = 0; j < V; ++j) {
        const int64_t t = g * V + j;
        v.e[j] = t < k_keep ? row[ib[t]] : T(0);
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
  const T* row = X + b * bstride + r * ld;
  const int32_t* ib = idx + b * k_keep;
  T* dst = out + (b * R + r) * k_pad;
  pdl_trigger();
  pdl_wait();
  for (int64_t g = threadIdx.x; g < k_pad / V; g += kPackThreads) {
    Vec16<T> v;
#pragma unroll
    for (int j = 0; j < V; ++j) {
      const int64_t t = g * V + j;
      v.e[j] = t < k_keep ? row[ib[t]] : T(0);
    }
    reinterpret_cast<uint4*>(dst)[g] = v.u;
  }
}

// Kept rows of B (N·e a multiple of 16, rows 16-byte aligned): bulk-async row
// copies through shared memory. CTA x covers kept rows [x·rows, (x+1)·rows).
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_rows_bulk_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t N,
                      const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                      int64_t ldo, int rows_per_cta, uint32_t* status, uint64_t wait_ns) {
  extern __shared__ __align__(128) unsigned char pack_smem[];
  __shared__ uint64_t bar;
  __shared__ int never;
  T* srow = reinterpret_cast<T*>(pack_smem);
  const int64_t b = blockIdx.y;
  const int64_t t0 = int64_t(blockIdx.x) * rows_per_cta;
  const int nr = int(min(int64_t(rows_per_cta), k_pad - t0));
  const int nload = int(max(int64_t(0), min(int64_t(nr), k_keep - t0)));  // kept rows in this CTA
  const uint32_t row_bytes = uint32_t(N * sizeof(T));
  T* dst = out + (b * k_pad + t0) * ldo;
  if (threadIdx.x == 0) {
    mbar_init(&bar, 1);
    never = 0;
    fence_mbar_init();
  }
  pdl_trigger();
  pdl_wait();
  __syncthreads();
  if (threadIdx.x == 0 && nload > 0) {
    const int32_t* ib = idx + b * k_keep + t0;
    const T* src = X + b * bstride;
    mbar_arrive_expect_tx(&bar, row_bytes * uint32_t(nload));
    for (int rr = 0; rr < nload; ++rr) bulk_load(srow + rr * N, src + int64_t(__ldg(ib + rr)) * ld, row_bytes, &bar);
  }
  // padding rows (t >= k_keep) are zeros; padding columns N <= c < ldo too
  for (int rr = nload; rr < nr; ++rr)
    for (int64_t c = threadIdx.x; c < ldo; c += kPackThreads) dst[rr * ldo + c] = T(0);
  if (ldo > N)
    for (int rr = 0; rr < nload; ++rr)
      for (int64_t c = N + threadIdx.x; c < ldo; c += kPackThreads) dst[rr * ldo + c] = T(0);
  if (nload > 0) {
    wait_loads(&bar, wait_ns, status, &never);
    if (threadIdx.x == 0) {
      for (int rr = 0; rr < nload; ++rr) bulk_store(dst + rr * ldo, srow + rr * N, row_bytes);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // smem stays live until read
    }
  }
}

// Kept rows of B, any alignment: plain element copies.
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_rows_plain_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t N,
                       const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                       int64_t ldo) {
  const int64_t b = blockIdx.y;
  const int64_t t = blockIdx.x;
  T* dst = out + (b * k_pad + t) * ldo;
  pdl_trigger();
  pdl_wait();
  if (t >= k_keep) {
    for (int64_t c = threadIdx.x; c < ldo; c += kPackThreads) dst[c] = T(0);
    return;
  }
  const T* src = X + b * bstride + int64_t(idx[b * k_keep + t]) * ld;
  for (int64_t c = threadIdx.x; c < ldo; c += kPackThreads) dst[c] = c < N ? src[c] : T(0);
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }

template <typename K>
void set_smem_attr_once(K kernel) {
  static bool done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !done[dev]) {
    cudaFuncSetAttribute(kernel, cudaFuncAttributeMaxDynamicSharedMemorySize, int(kSmemAttr));
    done[dev] = true;
  }
}

template <typename T>
cudaError_t launch_pack_cols_t(const MatView& X, int64_t batch, const int32_t* idx, int64_t k_keep, int64_t k_pad,
                               void* out, uint32_t* status, uint64_t wait_ns, cudaStream_t st) {
  const size_t row_bytes = size_t(X.cols) * sizeof(T);
  const T* p = static_cast<const T*>(X.ptr);
  T* o = static_cast<T*>(out);
  if (row_bytes > kStageMax) {
    return launch_pdl(pack_cols_direct_kernel<T>, dim3(unsigned(X.rows), unsigned(batch)), dim3(kPackThreads), 0, st,
                      dim3(0, 0, 0), p, X.ld, X.bstride, X.rows, idx, k_keep, k_pad, o);
  }
  const int rows_per_cta =
      row_bytes <= kStageBytes ? int(std::min<size_t>(64, kStageBytes / std::max<size_t>(row_bytes, 1))) : 1;
  const size_t idx_bytes = size_t(k_keep) * 4;
  const int idx_in_smem = idx_bytes <= kStageBytes;
  const size_t smem = size_t(rows_per_cta) * row_bytes + (idx_in_smem ? (idx_bytes + 15) / 16 * 16 : 0);
  const dim3 grid(unsigned((X.rows + rows_per_cta - 1) / rows_per_cta), unsigned(batch), 1u);
  const bool bulk = aligned16(X.ptr) && row_bytes % 16 == 0 && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                    (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0) && aligned16(idx) &&
                    (batch == 1 || k_keep % 4 == 0);
  if (bulk) {
    set_smem_attr_once(pack_cols_bulk_kernel<T>);
    return launch_pdl(pack_cols_bulk_kernel<T>, grid, dim3(kPackThreads), smem, st, dim3(0, 0, 0), p, X.ld,
                      X.bstride, X.rows, X.cols, idx, k_keep, k_pad, o, rows_per_cta, idx_in_smem, status, wait_ns);
  }
  set_smem_attr_once(pack_cols_plain_kernel<T>);
  return launch_pdl(pack_cols_plain_kernel<T>, grid, dim3(kPackThreads), smem, st, dim3(0, 0, 0), p, X.ld, X.bstride, X.rows,
                    X.cols, idx, k_keep, k_pad, o, rows_per_cta);
}

template <typename T>
cudaError_t launch_pack_rows_t(const MatView& X, int64_t batch, const int32_t* idx, int64_t k_keep, int64_t k_pad,
                               void* out, int64_t ldo, uint32_t* status, uint64_t wait_ns, cudaStream_t st) {
  const size_t row_bytes = size_t(X.cols) * sizeof(T);
  const T* p = static_cast<const T*>(X.ptr);
  T* o = static_cast<T*>(out);
  const bool bulk = row_bytes > 0 && row_bytes % 16 == 0 && row_bytes <= kStageMax && aligned16(X.ptr) &&
                    aligned16(out) && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                    (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0) && (ldo * int64_t(sizeof(T))) % 16 == 0;
  if (bulk) {
    const int rows_per_cta =
        row_bytes <= kStageBytes ? int(std::min<size_t>(64, kStageBytes / row_bytes)) : 1;
    const size_t smem = size_t(rows_per_cta) * row_bytes;
    set_smem_attr_once(pack_rows_bulk_kernel<T>);
    const dim3 grid(unsigned((k_pad + rows_per_cta - 1) / rows_per_cta), unsigned(batch), 1u);
    return launch_pdl(pack_rows_bulk_kernel<T>, grid, dim3(kPackThreads), smem, st, dim3(0, 0, 0), p, X.ld, X.bstride, X.cols, idx,
                      k_keep, k_pad, o, ldo, rows_per_cta, status, wait_ns);
  }
  return launch_pdl(pack_rows_plain_kernel<T>, dim3(unsigned(k_pad), unsigned(batch)), dim3(kPackThreads), 0, st, dim3(0, 0, 0),
                    p, X.ld, X.bstride, X.cols, idx, k_keep, k_pad, o, ldo);
}

}  // namespace

cudaError_t launch_pack_cols(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx, int64_t k_keep,
                             int64_t k_pad, void* out, uint32_t* status, uint64_t wait_ns, cudaStream_t st) {
  if (batch == 0 || X.rows == 0) return cudaSuccess;
  return e == kBF16 ? launch_pack_cols_t<uint16_t>(X, batch, idx, k_keep, k_pad, out, status, wait_ns, st)
                    : launch_pack_cols_t<uint32_t>(X, batch, idx, k_keep, k_pad, out, status, wait_ns, st);
}

cudaError_t launch_pack_rows(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx, int64_t k_keep,
                             int64_t k_pad, void* out, int64_t ldo, uint32_t* status, uint64_t wait_ns,
                             cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  return e == kBF16 ? launch_pack_rows_t<uint16_t>(X, batch, idx, k_keep, k_pad, out, ldo, status, wait_ns, st)
                    : launch_pack_rows_t<uint32_t>(X, batch, idx, k_keep, k_pad, out, ldo, status, wait_ns, st);
}

}  // namespace rmm
