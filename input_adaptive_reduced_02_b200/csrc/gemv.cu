// Decode-shaped reduced product ("Mecanismo Central" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference", with the autoregressive setting its
// "Escopo de Aplicação" names): C = A[:, I]·B[I, :] for M <= 16 rows of A,
// read straight from A and B through the kept indices, with no packed copy.
//
// With a handful of rows the product is a matrix-vector product that streams
// the kept rows of B once; skipping a row of B saves its bytes outright, so
// the kernel is built around HBM reads of B:
//  * a CTA owns 128 columns of C (4 per lane: 8-byte loads of bf16, 16-byte
//    of f32) and a share of the kept slices; its 8 warps take the slices in
//    turn, up to 16 rows of B in flight per lane;
//  * the A values it needs, A[m][idx[t]], and the row numbers idx[t] are
//    staged in shared memory 256 slices at a time;
//  * the CTAs of a thread-block cluster (up to 8) split the kept slices; each
//    sums its warps' partial products in warp order, then rank 0 adds the
//    CTAs' partials in rank order through distributed shared memory and
//    writes C. Fixed order throughout: bit-reproducible, no atomics.
// Products and sums in f32 (FFMA); C in f32 or bf16 (round to nearest even).
#include <cooperative_groups.h>

#include <algorithm>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace cg = cooperative_groups;

namespace rmm {
namespace {

constexpr int kGvThreads = 256;
constexpr int kGvWarps = kGvThreads / 32;
constexpr int kGvCols = 128;  // columns of C per CTA
constexpr int kGvSub = 256;   // kept slices staged per pass
constexpr unsigned kGvMaxCluster = 8;

template <int MT>
constexpr size_t gv_smem_bytes() {
  return size_t(kGvWarps) * MT * kGvCols * 4 + size_t(MT) * kGvCols * 4 + size_t(kGvSub) * MT * 4 +
         size_t(kGvSub) * 4;
}

// Four consecutive elements of a row of B starting at column c, as f32 (zero
// past column N). vec: 8-byte (bf16) / 16-byte (f32) loads are aligned.
__device__ __forceinline__ float4 load4(const uint16_t* row, int64_t c, int64_t N, bool vec) {
  if (vec && c + 4 <= N) {
    uint2 u;
    asm volatile("ld.global.nc.L1::no_allocate.v2.u32 {%0, %1}, [%2];" : "=r"(u.x), "=r"(u.y) : "l"(row + c));
    return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                       __uint_as_float(u.y & 0xFFFF0000u));
  }
  float v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = c + j < N ? elem_to_f32(row[c + j]) : 0.f;
  return make_float4(v[0], v[1], v[2], v[3]);
}

__device__ __forceinline__ float4 load4(const uint32_t* row, int64_t c, int64_t N, bool vec) {
  if (vec && c + 4 <= N) {
    uint4 u;
    asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
                 : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                 : "l"(row + c));
    return make_float4(__uint_as_float(u.x), __uint_as_float(u.y), __uint_as_float(u.z), __uint_as_float(u.w));
  }
  float v[4];
#pragma unroll
  for (int j = 0; j < 4; ++j) v[j] = c + j < N ? elem_to_f32(row[c + j]) : 0.f;
  return make_float4(v[0], v[1], v[2], v[3]);
}

template <int MT>
__device__ __forceinline__ void fma_row(float (&acc)[MT][4], const float* xrow, float4 w) {
#pragma unroll
  for (int m = 0; m < MT; ++m) {
    const float xm = xrow[m];
    acc[m][0] = fmaf(xm, w.x, acc[m][0]);
    acc[m][1] = fmaf(xm, w.y, acc[m][1]);
    acc[m][2] = fmaf(xm, w.z, acc[m][2]);
    acc[m][3] = fmaf(xm, w.w, acc[m][3]);
  }
}

// T: uint16_t (bf16 bits) or uint32_t (f32 bits). MT >= M rows of A.
template <typename T, int MT>
__global__ void __launch_bounds__(kGvThreads)
gemv_gather_kernel(const T* __restrict__ A, int64_t lda, int64_t sA, const T* __restrict__ B, int64_t ldb,
                   int64_t sB, int64_t M, int64_t N, const int32_t* __restrict__ idx, int64_t k_keep,
                   void* __restrict__ C, int64_t ldc, int64_t sC, int out_bf16, int b_vec) {
  constexpr int U = MT <= 4 ? 16 : 8;  // rows of B in flight per lane
  extern __shared__ float gv_smem[];
  float* part = gv_smem;                                     // [warp][MT][kGvCols]
  float* cta = part + kGvWarps * MT * kGvCols;               // [MT][kGvCols]
  float* xs = cta + MT * kGvCols;                            // [kGvSub][MT]
  int32_t* rows = reinterpret_cast<int32_t*>(xs + kGvSub * MT);  // [kGvSub]

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();
  const int64_t b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = int64_t(blockIdx.x) * kGvCols;
  const int64_t c = n0 + 4 * lane;
  const T* Ab = A + b * sA;
  const T* Bb = B + b * sB;
  const int32_t* ib = idx + b * k_keep;
  const int64_t per = (k_keep + cs - 1) / cs;
  const int64_t t_begin = min(k_keep, int64_t(crank) * per), t_end = min(k_keep, t_begin + per);

  float acc[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;

  pdl_trigger();
  pdl_wait();
  for (int64_t s0 = t_begin; s0 < t_end; s0 += kGvSub) {
    const int nsub = int(min(int64_t(kGvSub), t_end - s0));
    __syncthreads();  // the previous pass is done with xs and rows
    for (int i = tid; i < nsub; i += kGvThreads) {
      const int32_t r = ib[s0 + i];
      rows[i] = r;
#pragma unroll
      for (int m = 0; m < MT; ++m) xs[i * MT + m] = m < M ? elem_to_f32(Ab[int64_t(m) * lda + r]) : 0.f;
    }
    __syncthreads();
    int i = warp;
    for (; i + kGvWarps * (U - 1) < nsub; i += kGvWarps * U) {
      float4 w[U];
#pragma unroll
      for (int u = 0; u < U; ++u) w[u] = load4(Bb + int64_t(rows[i + kGvWarps * u]) * ldb, c, N, b_vec != 0);
#pragma unroll
      for (int u = 0; u < U; ++u) fma_row<MT>(acc, xs + (i + kGvWarps * u) * MT, w[u]);
    }
    for (; i < nsub; i += kGvWarps) fma_row<MT>(acc, xs + i * MT, load4(Bb + int64_t(rows[i]) * ldb, c, N, b_vec != 0));
  }
  // the CTA's partial: its warps' sums added in warp order
#pragma unroll
  for (int m = 0; m < MT; ++m)
    *reinterpret_cast<float4*>(part + (warp * MT + m) * kGvCols + 4 * lane) =
        make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
  __syncthreads();
  for (int e = tid; e < MT * kGvCols; e += kGvThreads) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < kGvWarps; ++q) t += part[q * MT * kGvCols + e];
    cta[e] = t;
  }
  cluster.sync();  // every CTA's partial is written and visible cluster-wide
  if (crank == 0) {
    for (int e = tid; e < MT * kGvCols; e += kGvThreads) {
      const int m = e / kGvCols;
      const int64_t col = n0 + (e % kGvCols);
      if (m >= M || col >= N) continue;
      float t = 0.f;
      for (unsigned q = 0; q < cs; ++q) t += cluster.map_shared_rank(cta, q)[e];
      const int64_t off = b * sC + int64_t(m) * ldc + col;
      if (out_bf16)
        static_cast<uint16_t*>(C)[off] = uint16_t(pack_bf16x2(t, 0.f) & 0xFFFFu);
      else
        static_cast<float*>(C)[off] = t;
    }
  }
  cluster.sync();  // keep shared memory alive until rank 0 has read it
}

// ---------------------------------------------------------------- async path
// B's rows reach shared memory by cp.async (no registers held while the
// copies are in flight): each lane copies its own 4 columns of each row into a
// private slot and later reads back only that slot, so a lane's own
// cp.async.wait_group is the only synchronisation the data needs. Passes of
// kGvPass kept slices are double-buffered: while pass p is summed, the rows of
// pass p + 1 are in flight and the indices and A values of pass p + 2 are
// staged.
constexpr int kGvPass = 128;

template <typename T>
constexpr int lane_bytes() { return 4 * int(sizeof(T)); }  // 4 columns

template <typename T, int MT>
constexpr size_t gv_async_smem_bytes() {
  return size_t(2) * kGvPass * 32 * lane_bytes<T>()  // ring (the warp partials reuse it afterwards)
         + size_t(2) * kGvPass * MT * 4               // A values
         + size_t(2) * kGvPass * 4                    // row numbers
         + size_t(MT) * kGvCols * 4;                  // the CTA's partial
}

template <int BYTES>
__device__ __forceinline__ void cp_async_zfill(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(smem_dst)), "l"(gsrc),
                 "r"(src_bytes) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_addr(smem_dst)), "l"(gsrc),
                 "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ float4 slot_to_f32(const uint16_t*, const unsigned char* slot) {
  const uint2 u = *reinterpret_cast<const uint2*>(slot);
  return make_float4(__uint_as_float(u.x << 16), __uint_as_float(u.x & 0xFFFF0000u), __uint_as_float(u.y << 16),
                     __uint_as_float(u.y & 0xFFFF0000u));
}
__device__ __forceinline__ float4 slot_to_f32(const uint32_t*, const unsigned char* slot) {
  return *reinterpret_cast<const float4*>(slot);
}

// Requires B's rows (and its base) aligned to lane_bytes<T>().
template <typename T, int MT>
__global__ void __launch_bounds__(kGvThreads)
gemv_gather_async_kernel(const T* __restrict__ A, int64_t lda, int64_t sA, const T* __restrict__ B, int64_t ldb,
                         int64_t sB, int64_t M, int64_t N, const int32_t* __restrict__ idx, int64_t k_keep,
                         void* __restrict__ C, int64_t ldc, int64_t sC, int out_bf16) {
  constexpr int LB = lane_bytes<T>();
  constexpr int RPW = kGvPass / kGvWarps;  // slices per warp per pass
  extern __shared__ __align__(16) unsigned char gva_smem[];
  unsigned char* ring = gva_smem;                                              // [2][kGvPass][32][LB]
  float* xs = reinterpret_cast<float*>(ring + size_t(2) * kGvPass * 32 * LB);  // [2][kGvPass][MT]
  int32_t* rows = reinterpret_cast<int32_t*>(xs + 2 * kGvPass * MT);           // [2][kGvPass]
  float* cta = reinterpret_cast<float*>(rows + 2 * kGvPass);                   // [MT][kGvCols]
  float* part = reinterpret_cast<float*>(ring);                                // [warp][MT][kGvCols], after the loop

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();
  const int64_t b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = int64_t(blockIdx.x) * kGvCols;
  const int64_t c = n0 + 4 * lane;
  const uint32_t src_bytes = c >= N ? 0u : uint32_t(min(int64_t(4), N - c) * int64_t(sizeof(T)));
  const T* Ab = A + b * sA;
  const T* Bb = B + b * sB;
  const int32_t* ib = idx + b * k_keep;
  const int64_t per = (k_keep + cs - 1) / cs;
  const int64_t t_begin = min(k_keep, int64_t(crank) * per), t_end = min(k_keep, t_begin + per);
  const int np = int((t_end - t_begin + kGvPass - 1) / kGvPass);

  auto pass_rows = [&](int p) { return int(min(int64_t(kGvPass), t_end - t_begin - int64_t(p) * kGvPass)); };
  auto stage = [&](int p) {
    const int buf = p & 1, n = pass_rows(p);
    for (int i = tid; i < n; i += kGvThreads) {
      const int32_t r = ib[t_begin + int64_t(p) * kGvPass + i];
      rows[buf * kGvPass + i] = r;
#pragma unroll
      for (int m = 0; m < MT; ++m)
        xs[(buf * kGvPass + i) * MT + m] = m < M ? elem_to_f32(Ab[int64_t(m) * lda + r]) : 0.f;
    }
  };
  auto issue = [&](int p) {
    const int buf = p & 1, n = pass_rows(p);
#pragma unroll
    for (int j = 0; j < RPW; ++j) {
      const int i = warp + kGvWarps * j;
      if (i < n) {
        const T* src = src_bytes ? Bb + int64_t(rows[buf * kGvPass + i]) * ldb + c : Bb;
        cp_async_zfill<LB>(ring + (size_t(buf * kGvPass + i) * 32 + lane) * LB, src, src_bytes);
      }
    }
    cp_async_commit();  // one group per pass in every thread, empty or not
  };

  float acc[MT][4];
#pragma unroll
  for (int m = 0; m < MT; ++m) acc[m][0] = acc[m][1] = acc[m][2] = acc[m][3] = 0.f;

  pdl_trigger();
  pdl_wait();
  if (np > 0) {
    stage(0);
    __syncthreads();
    issue(0);
  }
  if (np > 1) {
    stage(1);
    __syncthreads();
    issue(1);
  }
  for (int p = 0; p < np; ++p) {
    const int buf = p & 1, n = pass_rows(p);
    if (p + 1 < np)
      cp_async_wait<1>();  // this thread's copies of pass p have landed
    else
      cp_async_wait<0>();
#pragma unroll 4
    for (int j = 0; j < RPW; ++j) {
      const int i = warp + kGvWarps * j;
      if (i < n)
        fma_row<MT>(acc, xs + (buf * kGvPass + i) * MT,
                    slot_to_f32(static_cast<const T*>(nullptr), ring + (size_t(buf * kGvPass + i) * 32 + lane) * LB));
    }
    __syncthreads();  // every warp is done with buffer `buf`
    if (p + 2 < np) {
      stage(p + 2);
      __syncthreads();
      issue(p + 2);
    }
  }
  __syncthreads();  // the ring is free: the warp partials take its place
#pragma unroll
  for (int m = 0; m < MT; ++m)
    *reinterpret_cast<float4*>(part + (warp * MT + m) * kGvCols + 4 * lane) =
        make_float4(acc[m][0], acc[m][1], acc[m][2], acc[m][3]);
  __syncthreads();
  for (int e = tid; e < MT * kGvCols; e += kGvThreads) {
    float t = 0.f;
#pragma unroll
    for (int q = 0; q < kGvWarps; ++q) t += part[q * MT * kGvCols + e];
    cta[e] = t;
  }
  cluster.sync();
  if (crank == 0) {
    for (int e = tid; e < MT * kGvCols; e += kGvThreads) {
      const int m = e / kGvCols;
      const int64_t col = n0 + (e % kGvCols);
      if (m >= M || col >= N) continue;
      float t = 0.f;
      for (unsigned q = 0; q < cs; ++q) t += cluster.map_shared_rank(cta, q)[e];
      const int64_t off = b * sC + int64_t(m) * ldc + col;
      if (out_bf16)
        static_cast<uint16_t*>(C)[off] = uint16_t(pack_bf16x2(t, 0.f) & 0xFFFFu);
      else
        static_cast<float*>(C)[off] = t;
    }
  }
  cluster.sync();
}
static_assert(size_t(kGvWarps) * 16 * kGvCols * 4 <= size_t(2) * kGvPass * 32 * 8, "warp partials fit in the ring");

template <typename T, int MT>
cudaError_t launch_mt(const GemvArgs& g, cudaStream_t st) {
  const size_t smem = gv_smem_bytes<MT>();
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_gather_kernel<T, MT>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(smem));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nblk = (g.N + kGvCols - 1) / kGvCols;
  // split the kept slices over a cluster until there are about two CTAs per
  // SM, keeping at least 64 slices per CTA
  unsigned cs = 1;
  while (cs < kGvMaxCluster && nblk * g.batch * cs < 2 * int64_t(sms) && g.k_keep >= int64_t(cs) * 2 * 64) cs *= 2;
  const T* a = static_cast<const T*>(g.a);
  const T* bp = static_cast<const T*>(g.b);
  const int b_vec = (reinterpret_cast<uintptr_t>(g.b) % 16 == 0) && (g.ldb * int64_t(sizeof(T))) % 16 == 0 &&
                    (g.batch == 1 || (g.strideB * int64_t(sizeof(T))) % 16 == 0);
  if (b_vec) {
    const size_t asmem = gv_async_smem_bytes<T, MT>();
    static bool async_attr[64] = {};
    if (dev >= 0 && dev < 64 && !async_attr[dev]) {
      cudaError_t e = cudaFuncSetAttribute(gemv_gather_async_kernel<T, MT>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(asmem));
      if (e != cudaSuccess) return e;
      async_attr[dev] = true;
    }
    return launch_pdl(gemv_gather_async_kernel<T, MT>, dim3(unsigned(nblk), cs, unsigned(g.batch)),
                      dim3(kGvThreads), asmem, st, dim3(1, cs, 1), a, g.lda, g.strideA, bp, g.ldb, g.strideB, g.M,
                      g.N, g.idx, g.k_keep, g.c, g.ldc, g.strideC, int(g.out == kBF16));
  }
  return launch_pdl(gemv_gather_kernel<T, MT>, dim3(unsigned(nblk), cs, unsigned(g.batch)), dim3(kGvThreads), smem,
                    st, dim3(1, cs, 1), a, g.lda, g.strideA, bp, g.ldb, g.strideB, g.M, g.N, g.idx, g.k_keep, g.c,
                    g.ldc, g.strideC, int(g.out == kBF16), b_vec);
}

template <typename T>
cudaError_t launch_t(const GemvArgs& g, cudaStream_t st) {
  if (g.M <= 1) return launch_mt<T, 1>(g, st);
  if (g.M <= 2) return launch_mt<T, 2>(g, st);
  if (g.M <= 4) return launch_mt<T, 4>(g, st);
  if (g.M <= 8) return launch_mt<T, 8>(g, st);
  return launch_mt<T, 16>(g, st);
}

}  // namespace

cudaError_t launch_gemv_gather(const GemvArgs& g, cudaStream_t st) {
  if (g.batch == 0 || g.M == 0 || g.N == 0) return cudaSuccess;
  if (g.M > kGemvMaxRows) return cudaErrorInvalidValue;
  return g.in == kBF16 ? launch_t<uint16_t>(g, st) : launch_t<uint32_t>(g, st);
}

}  // namespace rmm
