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
#include <atomic>

#include "int8_convert.cuh"
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kPackThreads = 256;
constexpr size_t kStageBytes = 32 * 1024;   // shared-memory rows per CTA (short rows)
constexpr size_t kStageMax = 112 * 1024;    // one long row per CTA, two CTAs per SM
constexpr size_t kSmemAttr = kStageMax + kStageBytes;  // + staged kept indices
constexpr size_t kIdxStageMax = 64 * 1024;             // kept indices a pack_cols CTA stages

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
// shared memory or global memory; read as 16-byte vectors when ib_vec, i.e.
// ib is 16-byte aligned, else one by one). The threads take the nr x (k_pad / V)
// output vectors in order, so that short output rows (few kept columns, e.g.
// a head dimension of 128) still keep every thread busy and the stores stay
// contiguous.
template <typename T>
__device__ __forceinline__ void gather_rows(const T* srow, int nr, int64_t C, const int32_t* ib, bool ib_vec,
                                            int64_t k_keep, int64_t k_pad, T* dst) {
  constexpr int V = 16 / sizeof(T);
  const int ng = int(k_pad / V);  // k_pad <= 2^21 and nr <= 64: nr · ng fits an int
  const int total = nr * ng;
  for (int e = threadIdx.x; e < total; e += kPackThreads) {
    const int rr = e / ng, g = e - rr * ng;
    const T* row = srow + rr * C;
    {
      const int64_t t0 = int64_t(g) * V;
      Vec16<T> v;
      if (ib_vec && t0 + V <= k_keep) {
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
__device__ __forceinline__ void pack_cols_bulk_body(int64_t bx, const T* __restrict__ X, int64_t ld, int64_t bstride,
                                                    int64_t R, int64_t C, const int32_t* __restrict__ idx,
                                                    int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                                                    int rows_per_cta, int idx_in_smem, uint32_t* status,
                                                    uint64_t wait_ns) {
  extern __shared__ __align__(128) unsigned char pack_smem[];
  __shared__ uint64_t bar;
  __shared__ int never;
  T* srow = reinterpret_cast<T*>(pack_smem);
  int32_t* sidx = reinterpret_cast<int32_t*>(pack_smem + size_t(rows_per_cta) * C * sizeof(T));
  const int64_t b = blockIdx.y;
  const int64_t r0 = bx * rows_per_cta;
  const int nr = int(min(int64_t(rows_per_cta), R - r0));
  const T* src = X + b * bstride + r0 * ld;
  const int32_t* gidx = idx + b * k_keep;
  const bool gidx_vec = (reinterpret_cast<uintptr_t>(gidx) & 15u) == 0;
  // whole 16-byte groups of indices by bulk copy when this item's list is aligned
  const int64_t idx_bulk = (idx_in_smem && gidx_vec) ? (k_keep & ~int64_t(3)) : 0;
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
    if (ld == C)  // contiguous rows: one copy (each copy has a fixed cost; rows can be short)
      bulk_load(srow, src, row_bytes * uint32_t(nr), &bar);
    else
      for (int rr = 0; rr < nr; ++rr) bulk_load(srow + rr * C, src + rr * ld, row_bytes, &bar);
    if (idx_bulk > 0) bulk_load(sidx, gidx, uint32_t(idx_bulk * 4), &bar);
  }
  if (idx_in_smem)
    for (int64_t t = idx_bulk + threadIdx.x; t < k_keep; t += kPackThreads) sidx[t] = gidx[t];
  wait_loads(&bar, wait_ns, status, &never);
  __syncthreads();
  gather_rows(srow, nr, C, idx_in_smem ? sidx : gidx, idx_in_smem || gidx_vec, k_keep, k_pad,
              out + (b * R + r0) * k_pad);
}

template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_cols_bulk_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
                      const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                      int rows_per_cta, int idx_in_smem, uint32_t* status, uint64_t wait_ns) {
  pack_cols_bulk_body<T>(blockIdx.x, X, ld, bstride, R, C, idx, k_keep, k_pad, out, rows_per_cta, idx_in_smem,
                         status, wait_ns);
}

// Any alignment: rows staged with plain loads (eight in flight per thread).
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_cols_plain_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t R, int64_t C,
                       const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                       int rows_per_cta) {
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
  gather_rows(srow, nr, C, ib, (reinterpret_cast<uintptr_t>(ib) & 15u) == 0, k_keep, k_pad, out + (b * R + r0) * k_pad);
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

// Kept rows of B (N·e a multiple of 16, rows 16-byte aligned): a persistent
// CTA streams its share of the kept rows through a ring of shared-memory
// buffers, one thread keeping bulk-async loads and bulk-async stores in
// flight at once; the other threads write the zero padding rows.
constexpr int kRowRing = 4;
constexpr int64_t kRowIdxStage = 8192;  // kept-row indices a CTA stages in shared memory

template <typename T>
__device__ __forceinline__ void pack_rows_bulk_body(int64_t bx, int64_t nbx, const T* __restrict__ X, int64_t ld,
                                                    int64_t bstride, int64_t N, const int32_t* __restrict__ idx,
                                                    int64_t k_keep, int64_t k_pad, T* __restrict__ out, int64_t ldo,
                                                    int rows_per_buf, int64_t seg, uint32_t* status,
                                                    uint64_t wait_ns) {
  // A chunk is rows_per_buf whole rows (seg == N) or one `seg`-element segment
  // of one row (rows_per_buf == 1, long rows).
  extern __shared__ __align__(128) unsigned char pack_smem[];
  __shared__ uint64_t bar[kRowRing];
  __shared__ int never;
  const int64_t b = blockIdx.y;
  const int64_t segs = (N + seg - 1) / seg;
  const size_t buf_elems = size_t(rows_per_buf) * seg;
  T* ring = reinterpret_cast<T*>(pack_smem);
  int32_t* sidx = reinterpret_cast<int32_t*>(pack_smem + kRowRing * buf_elems * sizeof(T));
  // this CTA's kept rows: a contiguous range of [0, k_keep), at most kRowIdxStage long
  const int64_t per = (k_keep + nbx - 1) / nbx;
  const int64_t t_begin = min(k_keep, bx * per), t_end = min(k_keep, t_begin + per);
  const int64_t nchunks = (t_end - t_begin + rows_per_buf - 1) / rows_per_buf * segs;
  T* outb = out + b * k_pad * ldo;
  if (threadIdx.x == 0) {
    for (int i = 0; i < kRowRing; ++i) mbar_init(&bar[i], 1);
    never = 0;
    fence_mbar_init();
  }
  pdl_trigger();
  pdl_wait();
  for (int64_t t = t_begin + threadIdx.x; t < t_end; t += kPackThreads) sidx[t - t_begin] = idx[b * k_keep + t];
  __syncthreads();
  // zero padding: rows k_keep <= t < k_pad (split across CTAs), and columns N <= c < ldo
  {
    const int64_t pad_rows = k_pad - k_keep;
    const int64_t pr = (pad_rows + nbx - 1) / nbx;
    const int64_t pa = k_keep + min(pad_rows, bx * pr), pb = min(k_pad, pa + pr);
    for (int64_t t = pa; t < pb; ++t)
      for (int64_t c = threadIdx.x; c < ldo; c += kPackThreads) outb[t * ldo + c] = T(0);
    if (ldo > N)
      for (int64_t t = t_begin; t < t_end; ++t)
        for (int64_t c = N + threadIdx.x; c < ldo; c += kPackThreads) outb[t * ldo + c] = T(0);
  }
  if (threadIdx.x == 0 && nchunks > 0) {
    const T* src = X + b * bstride;
    // chunk c: rows [t_begin + (c / segs)·rows_per_buf, ...), columns of
    // segment c % segs, through buffer c % kRowRing
    auto chunk = [&](int64_t c, int64_t& r0, int& nr, int64_t& c0, uint32_t& bytes) {
      r0 = (c / segs) * rows_per_buf;
      nr = int(min(int64_t(rows_per_buf), t_end - t_begin - r0));
      c0 = (c % segs) * seg;
      bytes = uint32_t(min(seg, N - c0) * int64_t(sizeof(T)));
    };
    auto issue_load = [&](int64_t c) {
      int64_t r0, c0;
      int nr;
      uint32_t bytes;
      chunk(c, r0, nr, c0, bytes);
      T* buf = ring + (c % kRowRing) * buf_elems;
      mbar_arrive_expect_tx(&bar[c % kRowRing], bytes * uint32_t(nr));
      for (int r = 0; r < nr; ++r)
        bulk_load(buf + r * seg, src + int64_t(sidx[r0 + r]) * ld + c0, bytes, &bar[c % kRowRing]);
    };
    int64_t issued = min(int64_t(kRowRing - 1), nchunks);
    for (int64_t c = 0; c < issued; ++c) issue_load(c);
    int64_t c = 0;
    for (; c < nchunks; ++c) {
      if (!mbar_wait_bounded(&bar[c % kRowRing], uint32_t((c / kRowRing) & 1), wait_ns, &never)) break;
      int64_t r0, c0;
      int nr;
      uint32_t bytes;
      chunk(c, r0, nr, c0, bytes);
      T* buf = ring + (c % kRowRing) * buf_elems;
      for (int r = 0; r < nr; ++r) bulk_store(outb + (t_begin + r0 + r) * ldo + c0, buf + r * seg, bytes);
      asm volatile("cp.async.bulk.commit_group;" ::: "memory");
      if (issued < nchunks) {
        // the buffer of chunk `issued` was last read by chunk c - 1's store
        asm volatile("cp.async.bulk.wait_group.read 1;" ::: "memory");
        issue_load(issued++);
      }
    }
    if (c < nchunks) {  // a wait ran out: record it, then let the loads in flight land
      status_or(status, RMM_TIMEOUT_BIT);
      for (int64_t d = c; d < issued; ++d)
        mbar_wait_bounded(&bar[d % kRowRing], uint32_t((d / kRowRing) & 1), wait_ns, &never);
    }
    asm volatile("cp.async.bulk.wait_group.read 0;" ::: "memory");  // smem stays live until read
  }
}

template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_rows_bulk_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t N,
                      const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, T* __restrict__ out,
                      int64_t ldo, int rows_per_buf, int64_t seg, uint32_t* status, uint64_t wait_ns) {
  pack_rows_bulk_body<T>(blockIdx.x, gridDim.x, X, ld, bstride, N, idx, k_keep, k_pad, out, ldo, rows_per_buf, seg,
                         status, wait_ns);
}

// Both packs in one launch (B row-major, both on the bulk paths): CTAs
// [0, nb) copy B's kept rows, the others gather A's columns; the two copy
// streams overlap instead of meeting at a kernel boundary.
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
pack_both_bulk_kernel(const T* __restrict__ A, int64_t lda, int64_t sA, int64_t M, int64_t K, T* __restrict__ a_out,
                      int rows_per_cta, int idx_in_smem, const T* __restrict__ B, int64_t ldb, int64_t sB, int64_t N,
                      T* __restrict__ b_out, int64_t ldo, int rows_per_buf, int64_t seg, int64_t nb,
                      const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad, uint32_t* status,
                      uint64_t wait_ns) {
  if (int64_t(blockIdx.x) < nb)
    pack_rows_bulk_body<T>(blockIdx.x, nb, B, ldb, sB, N, idx, k_keep, k_pad, b_out, ldo, rows_per_buf, seg, status,
                           wait_ns);
  else
    pack_cols_bulk_body<T>(int64_t(blockIdx.x) - nb, A, lda, sA, M, K, idx, k_keep, k_pad, a_out, rows_per_cta,
                           idx_in_smem, status, wait_ns);
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
  static std::atomic<bool> done[64];  // per device; racing first calls both set the attribute
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
  // kept indices in shared memory when they fit beside the rows (up to 64 KB;
  // beyond that the gather reads them from global memory, through L1)
  const size_t idx_bytes = (size_t(k_keep) * 4 + 15) / 16 * 16;
  const int idx_in_smem = idx_bytes <= kIdxStageMax && size_t(rows_per_cta) * row_bytes + idx_bytes <= kSmemAttr;
  const size_t smem = size_t(rows_per_cta) * row_bytes + (idx_in_smem ? idx_bytes : 0);
  const dim3 grid(unsigned((X.rows + rows_per_cta - 1) / rows_per_cta), unsigned(batch), 1u);
  // any index alignment: each CTA stages or reads its item's list as aligned allows
  const bool bulk = aligned16(X.ptr) && row_bytes % 16 == 0 && (X.ld * int64_t(sizeof(T))) % 16 == 0 &&
                    (batch == 1 || (X.bstride * int64_t(sizeof(T))) % 16 == 0);
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
    // ring of kRowRing buffers of up to 16 KB (at least one row each)
    // ring of kRowRing buffers of 16 KB: several whole rows, or a segment of a long row
    const int rows_per_buf = row_bytes <= 16384 ? int(std::min<size_t>(32, 16384 / row_bytes)) : 1;
    const int64_t seg = row_bytes <= 16384 ? X.cols : int64_t(16384 / sizeof(T));
    const size_t smem = size_t(kRowRing) * rows_per_buf * size_t(seg) * sizeof(T) + size_t(kRowIdxStage) * 4;
    if (smem <= kSmemAttr) {
      set_smem_attr_once(pack_rows_bulk_kernel<T>);
      int dev = 0, sms = 148;
      cudaGetDevice(&dev);
      cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
      // about two CTAs per SM over the whole batch, each streaming >= 4 buffers,
      // and few enough kept rows per CTA for its index stage
      const int64_t want = std::max<int64_t>(1, 2 * int64_t(sms) / std::max<int64_t>(1, batch));
      const int64_t segs = (X.cols + seg - 1) / seg;
      const int64_t by_work = std::max<int64_t>(1, k_keep * segs / (4 * rows_per_buf));
      const int64_t ctas = std::max(std::min(want, by_work), (k_keep + kRowIdxStage - 1) / kRowIdxStage);
      const dim3 grid(unsigned(ctas), unsigned(batch), 1u);
      return launch_pdl(pack_rows_bulk_kernel<T>, grid, dim3(kPackThreads), smem, st, dim3(0, 0, 0), p, X.ld,
                        X.bstride, X.cols, idx, k_keep, k_pad, o, ldo, rows_per_buf, seg, status, wait_ns);
    }
  }
  return launch_pdl(pack_rows_plain_kernel<T>, dim3(unsigned(k_pad), unsigned(batch)), dim3(kPackThreads), 0, st, dim3(0, 0, 0),
                    p, X.ld, X.bstride, X.cols, idx, k_keep, k_pad, o, ldo);
}

// Both packs in one launch when A's rows are short enough to stage several per
// CTA and both operands take the bulk paths; *handled = false otherwise.
template <typename T>
cudaError_t launch_pack_both_t(const MatView& A, const MatView& B, int64_t batch, const int32_t* idx,
                               int64_t k_keep, int64_t k_pad, void* a_out, void* b_out, int64_t ldo, uint32_t* status,
                               uint64_t wait_ns, cudaStream_t st, bool* handled) {
  *handled = false;
  const size_t a_row = size_t(A.cols) * sizeof(T), b_row = size_t(B.cols) * sizeof(T);
  const bool a_bulk = A.rows > 0 && a_row > 0 && a_row <= kStageBytes && a_row % 16 == 0 && aligned16(A.ptr) &&
                      (A.ld * int64_t(sizeof(T))) % 16 == 0 &&
                      (batch == 1 || (A.bstride * int64_t(sizeof(T))) % 16 == 0);
  const bool b_bulk = b_row > 0 && b_row % 16 == 0 && b_row <= kStageMax && aligned16(B.ptr) && aligned16(b_out) &&
                      (B.ld * int64_t(sizeof(T))) % 16 == 0 &&
                      (batch == 1 || (B.bstride * int64_t(sizeof(T))) % 16 == 0) && (ldo * int64_t(sizeof(T))) % 16 == 0;
  if (!a_bulk || !b_bulk) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  // B: as in launch_pack_rows_t, with the index stage sized to the CTA's share
  const int rows_per_buf = b_row <= 16384 ? int(std::min<size_t>(32, 16384 / b_row)) : 1;
  const int64_t seg = b_row <= 16384 ? B.cols : int64_t(16384 / sizeof(T));
  const int64_t want = std::max<int64_t>(1, 2 * int64_t(sms) / std::max<int64_t>(1, batch));
  const int64_t segs = (B.cols + seg - 1) / seg;
  const int64_t by_work = std::max<int64_t>(1, k_keep * segs / (4 * rows_per_buf));
  const int64_t nb = std::max(std::min(want, by_work), (k_keep + kRowIdxStage - 1) / kRowIdxStage);
  const int64_t per = (k_keep + nb - 1) / nb;
  const size_t b_smem = size_t(kRowRing) * rows_per_buf * size_t(seg) * sizeof(T) + size_t((per * 4 + 15) / 16 * 16);
  // A: as many whole rows per CTA as the same shared-memory size holds
  const size_t idx_bytes = (size_t(k_keep) * 4 + 15) / 16 * 16;
  const int idx_in_smem = idx_bytes <= kIdxStageMax && a_row + idx_bytes <= kSmemAttr;
  const size_t a_fixed = idx_in_smem ? idx_bytes : 0;
  const size_t budget = std::max(b_smem, a_row + a_fixed);
  const int rows_per_cta = int(std::max<size_t>(1, std::min<size_t>(64, (budget - a_fixed) / a_row)));
  const size_t smem = std::max(b_smem, size_t(rows_per_cta) * a_row + a_fixed);
  if (smem > kSmemAttr) return cudaSuccess;
  const int64_t na = (A.rows + rows_per_cta - 1) / rows_per_cta;
  set_smem_attr_once(pack_both_bulk_kernel<T>);
  *handled = true;
  return launch_pdl(pack_both_bulk_kernel<T>, dim3(unsigned(nb + na), unsigned(batch)), dim3(kPackThreads), smem, st,
                    dim3(0, 0, 0), static_cast<const T*>(A.ptr), A.ld, A.bstride, A.rows, A.cols,
                    static_cast<T*>(a_out), rows_per_cta, idx_in_smem, static_cast<const T*>(B.ptr), B.ld, B.bstride,
                    B.cols, static_cast<T*>(b_out), ldo, rows_per_buf, seg, nb, idx, k_keep, k_pad, status, wait_ns);
}

}  // namespace

cudaError_t launch_pack_both(const MatView& A, const MatView& B, ElemKind e, int64_t batch, const int32_t* idx,
                             int64_t k_keep, int64_t k_pad, void* a_out, void* b_out, int64_t ldo, uint32_t* status,
                             uint64_t wait_ns, cudaStream_t st, bool* handled) {
  *handled = false;
  if (batch == 0) return cudaSuccess;
  return e == kBF16 ? launch_pack_both_t<uint16_t>(A, B, batch, idx, k_keep, k_pad, a_out, b_out, ldo, status, wait_ns,
                                                   st, handled)
                    : launch_pack_both_t<uint32_t>(A, B, batch, idx, k_keep, k_pad, a_out, b_out, ldo, status, wait_ns,
                                                   st, handled);
}

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

namespace {

// out[b][t][j] = bf16(Wq[b][idx[b][t]][j] · scale[b][j]) for t < k_keep and
// j < N; zero for k_keep <= t < k_pad and N <= j < ldo. A CTA per kept row
// (grid-stride), 8 weights per thread step (8-byte load, 16-byte store) when
// aligned.
__global__ void __launch_bounds__(kPackThreads)
pack_rows_w8_kernel(const int8_t* __restrict__ Wq, int64_t ldw, int64_t sW, const float* __restrict__ scale,
                    int64_t s_stride, int64_t N, const int32_t* __restrict__ idx, int64_t k_keep, int64_t k_pad,
                    uint16_t* __restrict__ out, int64_t ldo, int vec) {
  pdl_trigger();
  pdl_wait();
  const int64_t b = blockIdx.y;
  const float* sc = scale + b * s_stride;
  for (int64_t t = blockIdx.x; t < k_pad; t += gridDim.x) {
    uint16_t* dst = out + (b * k_pad + t) * ldo;
    if (t >= k_keep) {
      for (int64_t c = threadIdx.x; c < ldo; c += kPackThreads) dst[c] = 0;
      continue;
    }
    const int8_t* src = Wq + b * sW + int64_t(idx[b * k_keep + t]) * ldw;
    int64_t c0 = 0;
    if (vec) {
      const int64_t n8 = N / 8;
      for (int64_t g = threadIdx.x; g < n8; g += kPackThreads) {
        const uint2 q = *reinterpret_cast<const uint2*>(src + 8 * g);
        const float4 s0 = *reinterpret_cast<const float4*>(sc + 8 * g);
        const float4 s1 = *reinterpret_cast<const float4*>(sc + 8 * g + 4);
        float v[8];
        s8x4_to_f32(q.x, v[0], v[1], v[2], v[3]);
        s8x4_to_f32(q.y, v[4], v[5], v[6], v[7]);
        v[0] *= s0.x, v[1] *= s0.y, v[2] *= s0.z, v[3] *= s0.w;
        v[4] *= s1.x, v[5] *= s1.y, v[6] *= s1.z, v[7] *= s1.w;
        *reinterpret_cast<uint4*>(dst + 8 * g) = make_uint4(pack_bf16x2(v[0], v[1]), pack_bf16x2(v[2], v[3]),
                                                            pack_bf16x2(v[4], v[5]), pack_bf16x2(v[6], v[7]));
      }
      c0 = n8 * 8;
    }
    for (int64_t c = c0 + threadIdx.x; c < ldo; c += kPackThreads)
      dst[c] = c < N ? uint16_t(pack_bf16x2(float(src[c]) * sc[c], 0.f) & 0xFFFFu) : uint16_t(0);
  }
}

}  // namespace

cudaError_t launch_pack_rows_w8(const int8_t* Wq, int64_t ldw, int64_t sW, const float* scale, int64_t s_stride,
                                int64_t batch, int64_t N, const int32_t* idx, int64_t k_keep, int64_t k_pad,
                                void* out, int64_t ldo, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  int dev = 0, sms = 148;
  cudaGetDevice(&dev);
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int vec = (reinterpret_cast<uintptr_t>(Wq) % 8 == 0) && ldw % 8 == 0 && (batch == 1 || sW % 8 == 0) &&
                  (reinterpret_cast<uintptr_t>(scale) % 16 == 0) && (batch == 1 || s_stride % 4 == 0) &&
                  (reinterpret_cast<uintptr_t>(out) % 16 == 0) && ldo % 8 == 0;
  const int64_t ctas = std::min<int64_t>(k_pad, std::max<int64_t>(1, 8 * int64_t(sms) / std::max<int64_t>(1, batch)));
  return launch_pdl(pack_rows_w8_kernel, dim3(unsigned(ctas), unsigned(batch)), dim3(kPackThreads), 0, st,
                    dim3(0, 0, 0), Wq, ldw, sW, scale, s_stride, N, idx, k_keep, k_pad, static_cast<uint16_t*>(out),
                    ldo, vec);
}

}  // namespace rmm

// ------------------------------------------------------------------ masked rows
// B with its dropped rows zeroed, for the route that streams A whole: A[:, I]
// · B[I, :] = A · B_M with B_M[r] = B[r] for r in I and 0 otherwise.
namespace rmm {
namespace {

constexpr int kMaskSeg = 64;  // kept indices per CTA

// CTA c owns kept positions [c·64, c·64 + 64) of item b and the rows from its
// first kept index (row 0 for c = 0) up to the next CTA's first kept index
// (K for the last CTA): kept rows are copied, the rows between them zeroed,
// columns N <= j < ldo zeroed. A warp per row, 16-byte vectors when the rows
// of X are 16-byte aligned.
template <typename T>
__global__ void __launch_bounds__(kPackThreads)
mask_rows_kernel(const T* __restrict__ X, int64_t ld, int64_t bstride, int64_t K, int64_t N,
                 const int32_t* __restrict__ idx, int64_t k_keep, T* __restrict__ out, int64_t ldo, int vec) {
  constexpr int V = 16 / sizeof(T);
  __shared__ int32_t seg[kMaskSeg + 1];
  const int64_t b = blockIdx.y;
  const int64_t t0 = int64_t(blockIdx.x) * kMaskSeg;
  const int64_t t1 = min(k_keep, t0 + kMaskSeg);
  const int32_t* ib = idx + b * k_keep;
  pdl_trigger();
  pdl_wait();
  if (threadIdx.x <= t1 - t0) seg[threadIdx.x] = threadIdx.x < t1 - t0 ? ib[t0 + threadIdx.x] : 0;
  __syncthreads();
  const int64_t r_lo = t0 == 0 ? 0 : seg[0];
  const int64_t r_hi = t1 == k_keep ? K : int64_t(ib[t1]);
  const int n = int(t1 - t0);
  const int warp = threadIdx.x >> 5, lane = threadIdx.x & 31;
  const T* Xb = X + b * bstride;
  T* Ob = out + b * K * ldo;
  // kept rows of the segment come in ascending order: walk them with the rows
  int p = 0;  // first segment entry >= r (all warps walk the same rows in the same order)
  for (int64_t r0 = r_lo; r0 < r_hi; r0 += kPackThreads / 32) {
    const int64_t r = r0 + warp;
    // advance p to the first kept index >= r0 (the same for every warp)
    while (p < n && seg[p] < r0) ++p;
    if (r >= r_hi) continue;
    bool kept = false;
    for (int q = p; q < n && seg[q] <= r; ++q) kept |= seg[q] == r;
    T* dst = Ob + r * ldo;
    if (vec) {
      const int64_t nv = ldo / V;  // ldo is a multiple of V when vec
      for (int64_t j = lane; j < nv; j += 32) {
        uint4 v = make_uint4(0u, 0u, 0u, 0u);
        if (kept && (j + 1) * V <= N) v = *reinterpret_cast<const uint4*>(Xb + r * ld + j * V);
        else if (kept) {
          alignas(16) T tmp[V];
#pragma unroll
          for (int e = 0; e < V; ++e) tmp[e] = j * V + e < N ? Xb[r * ld + j * V + e] : T(0);
          v = *reinterpret_cast<const uint4*>(tmp);
        }
        *reinterpret_cast<uint4*>(dst + j * V) = v;
      }
    } else {
      for (int64_t j = lane; j < ldo; j += 32) dst[j] = (kept && j < N) ? Xb[r * ld + j] : T(0);
    }
  }
}

template <typename T>
cudaError_t launch_mask_rows_t(const MatView& X, int64_t batch, const int32_t* idx, int64_t k_keep, void* out,
                               int64_t ldo, cudaStream_t st) {
  constexpr int V = 16 / sizeof(T);
  const int vec = (reinterpret_cast<uintptr_t>(X.ptr) & 15u) == 0 && (X.ld % V) == 0 &&
                  (batch == 1 || X.bstride % V == 0) && (reinterpret_cast<uintptr_t>(out) & 15u) == 0 &&
                  ldo % V == 0;
  const int64_t ctas = (k_keep + kMaskSeg - 1) / kMaskSeg;
  return launch_pdl(mask_rows_kernel<T>, dim3(unsigned(ctas), unsigned(batch)), dim3(kPackThreads), 0, st,
                    dim3(0, 0, 0), static_cast<const T*>(X.ptr), X.ld, X.bstride, X.rows, X.cols, idx, k_keep,
                    static_cast<T*>(out), ldo, vec);
}

}  // namespace

cudaError_t launch_mask_rows(const MatView& X, ElemKind e, int64_t batch, const int32_t* idx, int64_t k_keep,
                             void* out, int64_t ldo, cudaStream_t st) {
  if (batch == 0 || X.rows == 0) return cudaSuccess;
  return e == kBF16 ? launch_mask_rows_t<uint16_t>(X, batch, idx, k_keep, out, ldo, st)
                    : launch_mask_rows_t<uint32_t>(X, batch, idx, k_keep, out, ldo, st);
}

}  // namespace rmm
