// Decode-shaped reduced product ("Mecanismo Central" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference", with the autoregressive setting its
// "Escopo de Aplicação" names): C = A[:, I]·B[I, :] for M <= 16 rows of A,
// read straight from A and B through the kept indices, with no packed copy.
//
// With a handful of rows the product is a matrix-vector product that streams
// the kept rows of B once; skipping a row of B saves its bytes outright, so
// every kernel here is built around HBM reads of B, and in all of them the
// CTAs of a thread-block cluster (up to 8) split the kept slices, and the
// cluster's CTAs then share out the output elements, each adding the CTAs'
// partials in rank order through distributed shared memory (fixed order
// throughout: bit-reproducible, no atomics). By B:
//  * bf16, rows 16-byte aligned: gemv_gather_mma_kernel (tensor-core path,
//    below) — each warp streams its own column strip through a private
//    cp.async ring of 32-slice passes, mma.sync m16n8k16;
//  * INT8 with per-column scales, rows 16-byte aligned:
//    gemv_gather_mma_w8_kernel — mma.sync m16n8k16 too, each warp streaming
//    its own column strip through a private cp.async ring and converting the
//    int8 bytes exactly, straight into the MMA's bf16 B fragments;
//  * f32 with rows 16-byte aligned, or INT8 with rows only 4-byte aligned:
//    gemv_gather_async_kernel (FFMA, cp.async of 4 columns into per-lane
//    slots);
//  * bf16 or f32 rows that are not 16-byte aligned: gemv_gather_kernel (FFMA,
//    plain loads), sketched next —
//    a CTA owns 128 columns of C (4 per lane) and a share of the kept slices;
//    its 8 warps take the slices in turn, up to 16 rows of B in flight per
//    lane; A[m][idx[t]] and idx[t] are staged in shared memory 256 slices at
//    a time; each CTA sums its warps' partials in warp order.
// Sums in f32; C in f32 or bf16 (round to nearest even).
#include <cooperative_groups.h>

#include <algorithm>
#include <atomic>
#include <cmath>

#include "int8_convert.cuh"
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

// C[m][n0 + j] (m < M, j < cols, clipped to N) = the sum of the cluster's
// CTA partials part[m·cols + j], added in rank order from 0 (the same bits
// whichever thread adds them), times scale[n0 + j] when a column scale is
// given. The elements are shared out over all of the cluster's CTAs, and each
// thread keeps the remote loads of four elements in flight.
__device__ __forceinline__ void cluster_sum_store(cg::cluster_group& cluster, float* part, int cols, int64_t M,
                                                  int64_t n0, int64_t N, int64_t b, int64_t sC, int64_t ldc, void* C,
                                                  int out_bf16, const float* scale, int nthreads) {
  const int cs = int(cluster.num_blocks()), crank = int(cluster.block_rank());
  const int total = int(M) * cols;
  const int per = (total + cs - 1) / cs;
  const int e0 = crank * per, e1 = min(total, e0 + per);
  for (int e = e0 + int(threadIdx.x); e < e1; e += 4 * nthreads) {
    float t[4] = {0.f, 0.f, 0.f, 0.f};
    for (int q = 0; q < cs; ++q) {
      const float* src = cluster.map_shared_rank(part, q);
#pragma unroll
      for (int u = 0; u < 4; ++u)
        if (e + u * nthreads < e1) t[u] += src[e + u * nthreads];
    }
#pragma unroll
    for (int u = 0; u < 4; ++u) {
      const int eu = e + u * nthreads;
      if (eu >= e1) break;
      const int m = eu / cols;
      const int64_t col = n0 + (eu - m * cols);
      if (col >= N) continue;
      float v = t[u];
      if (scale) v *= scale[col];
      const int64_t off = b * sC + int64_t(m) * ldc + col;
      if (out_bf16)
        static_cast<uint16_t*>(C)[off] = uint16_t(pack_bf16x2(v, 0.f) & 0xFFFFu);
      else
        static_cast<float*>(C)[off] = v;
    }
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
  cluster_sum_store(cluster, cta, kGvCols, M, n0, N, b, sC, ldc, C, out_bf16, nullptr, kGvThreads);
  cluster.sync();  // keep shared memory alive until every rank has read it
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
  return size_t(2) * kGvPass * 32 * (lane_bytes<T>() < 8 ? 8 : lane_bytes<T>())  // ring (then the warp partials)
         + size_t(2) * kGvPass * MT * 4               // A values
         + size_t(2) * kGvPass * 4                    // row numbers
         + size_t(MT) * kGvCols * 4;                  // the CTA's partial
}

template <int BYTES>
__device__ __forceinline__ void cp_async_zfill(void* smem_dst, const void* gsrc, uint32_t src_bytes) {
  if constexpr (BYTES == 16)
    asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_addr(smem_dst)), "l"(gsrc),
                 "r"(src_bytes) : "memory");
  else if constexpr (BYTES == 8)
    asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_addr(smem_dst)), "l"(gsrc),
                 "r"(src_bytes) : "memory");
  else
    asm volatile("cp.async.ca.shared.global [%0], [%1], 4, %2;" ::"r"(smem_addr(smem_dst)), "l"(gsrc),
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
__device__ __forceinline__ float4 slot_to_f32(const int8_t*, const unsigned char* slot) {
  float4 f;
  s8x4_to_f32(*reinterpret_cast<const uint32_t*>(slot), f.x, f.y, f.z, f.w);
  return f;
}

// Requires B's rows (and its base) aligned to lane_bytes<TB>(). TB is B's
// element type (T's, or int8_t for an INT8 weight whose column j is scaled by
// col_scale[b * s_stride + j] at the end; col_scale null: no scale).
template <typename T, int MT, typename TB = T>
__global__ void __launch_bounds__(kGvThreads)
gemv_gather_async_kernel(const T* __restrict__ A, int64_t lda, int64_t sA, const TB* __restrict__ B, int64_t ldb,
                         int64_t sB, int64_t M, int64_t N, const int32_t* __restrict__ idx, int64_t k_keep,
                         void* __restrict__ C, int64_t ldc, int64_t sC, int out_bf16,
                         const float* __restrict__ col_scale, int64_t s_stride) {
  constexpr int LB = lane_bytes<TB>() < 8 ? 8 : lane_bytes<TB>();  // slot bytes (int8: 4 used of 8)
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
  const uint32_t src_bytes = c >= N ? 0u : uint32_t(min(int64_t(4), N - c) * int64_t(sizeof(TB)));
  const T* Ab = A + b * sA;
  const TB* Bb = B + b * sB;
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
        const TB* src = src_bytes ? Bb + int64_t(rows[buf * kGvPass + i]) * ldb + c : Bb;
        cp_async_zfill<lane_bytes<TB>()>(ring + (size_t(buf * kGvPass + i) * 32 + lane) * LB, src, src_bytes);
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
                    slot_to_f32(static_cast<const TB*>(nullptr), ring + (size_t(buf * kGvPass + i) * 32 + lane) * LB));
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
  cluster_sum_store(cluster, cta, kGvCols, M, n0, N, b, sC, ldc, C, out_bf16,
                    col_scale ? col_scale + b * s_stride : nullptr, kGvThreads);
  cluster.sync();
}
static_assert(size_t(kGvWarps) * 16 * kGvCols * 4 <= size_t(2) * kGvPass * 32 * 8, "warp partials fit in the ring");

// ---------------------------------------------------------------- bf16 tensor-core path
// Same data movement idea as the async path, but the products run on the
// tensor cores as warp-level mma.sync m16n8k16 (bf16 x bf16 -> f32), A being
// x_S padded to 16 rows. A CTA owns 8·WC columns of C, WC per warp, and each
// warp streams its own column strip (2·WC bytes of a row) of the kept rows
// through a private cp.async ring of 32-slice passes, so the main loop
// synchronises only within a warp; the whole block waits only while the
// indices and A's values of the next kMmaChunk slices are staged. WC = 64
// (512 columns per CTA) puts the grid of a large layer in one wave of two CTAs
// per SM; WC = 32 keeps more CTAs busy on a small one.
//  * B's rows stream through MmaCfg<WC>::BUFS passes per warp; BUFS - 1 are
//    in flight while one is summed.
//  * Ring rows and A rows are XOR-swizzled in 16-byte chunks so that
//    ldmatrix reads are free of bank conflicts; slices past the end are zero
//    in both.
constexpr int kMmaPass = 32;    // kept slices per ring buffer
constexpr int kMmaChunk = 256;  // slices whose indices and A values are staged at once

template <int WC>
struct MmaCfg {
  static constexpr int COLS = kGvWarps * WC;       // columns of C per CTA
  static constexpr int ROW = WC * 2;               // bytes of one slice of a warp's strip
  static constexpr int CPR = ROW / 16;             // 16-byte chunks per strip row
  static constexpr int BUFS = WC == 64 ? 3 : 4;    // passes per warp ring
  static constexpr uint32_t STAGE = uint32_t(kMmaPass) * ROW;  // one pass of one warp
  static constexpr int COPIES = kMmaPass * CPR / 32;          // 16-byte copies per lane per pass
  static constexpr size_t SMEM = size_t(kGvWarps) * BUFS * STAGE  // warp rings (then the CTA's partial)
                                 + size_t(16) * kMmaChunk * 2      // A: 16 rows of kMmaChunk bf16
                                 + size_t(kMmaChunk) * 4;          // row numbers
  static_assert(WC == 32 || WC == 64, "four or eight n8 tiles per warp");
  static_assert(size_t(16) * COLS * 4 <= size_t(kGvWarps) * BUFS * STAGE, "the partial fits in the rings");
  static_assert(2 * (SMEM + 1024) <= 228 * 1024, "two CTAs per SM");
};
static_assert(kMmaChunk % kMmaPass == 0 && kMmaPass % 16 == 0, "pass shape");

// 16-byte chunk `chunk` of row `row` of a swizzled array of rows of row_bytes
// (a multiple of 128): chunk ^ (row % 8), so the same chunk of 8 consecutive
// rows falls in 8 different bank groups.
__device__ __forceinline__ uint32_t swz(int row, int row_bytes, int chunk) {
  return uint32_t(row) * uint32_t(row_bytes) + (uint32_t(chunk ^ (row & 7)) << 4);
}
// The same for rows of CPR = 4 or 8 chunks: with 4 chunks (64-byte rows) two
// rows share a 128-byte bank line, so the XOR pattern advances every 2 rows.
template <int CPR>
__device__ __forceinline__ uint32_t swz_strip(int row, int chunk) {
  if constexpr (CPR == 8)
    return uint32_t(row) * 128u + (uint32_t(chunk ^ (row & 7)) << 4);
  else
    return uint32_t(row) * 64u + (uint32_t(chunk ^ ((row >> 1) & 3)) << 4);
}

__device__ __forceinline__ void ldsm_x4(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void ldsm_x4_t(uint32_t addr, uint32_t& r0, uint32_t& r1, uint32_t& r2, uint32_t& r3) {
  asm volatile("ldmatrix.sync.aligned.m8n8.x4.trans.shared.b16 {%0, %1, %2, %3}, [%4];"
               : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
               : "r"(addr));
}
__device__ __forceinline__ void mma_bf16_16816(float (&d)[4], uint32_t a0, uint32_t a1, uint32_t a2, uint32_t a3,
                                               uint32_t b0, uint32_t b1) {
  asm volatile(
      "mma.sync.aligned.m16n8k16.row.col.f32.bf16.bf16.f32 {%0, %1, %2, %3}, {%4, %5, %6, %7}, {%8, %9}, "
      "{%0, %1, %2, %3};"
      : "+f"(d[0]), "+f"(d[1]), "+f"(d[2]), "+f"(d[3])
      : "r"(a0), "r"(a1), "r"(a2), "r"(a3), "r"(b0), "r"(b1));
}
__device__ __forceinline__ void cp_async16_zfill(uint32_t smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_dst), "l"(gsrc), "r"(src_bytes)
               : "memory");
}

// Requires B's rows (and its base) 16-byte aligned.
template <int WC>
__global__ void __launch_bounds__(kGvThreads)
gemv_gather_mma_kernel(const uint16_t* __restrict__ A, int64_t lda, int64_t sA, const uint16_t* __restrict__ B,
                       int64_t ldb, int64_t sB, int64_t M, int64_t N, const int32_t* __restrict__ idx, int64_t k_keep,
                       void* __restrict__ C, int64_t ldc, int64_t sC, int out_bf16) {
  using Cfg = MmaCfg<WC>;
  constexpr int AROW = kMmaChunk * 2;  // bytes per row of A in shared memory
  constexpr int NT = WC / 8;           // n8 tiles per warp
  constexpr int LPR = 32 / Cfg::CPR;   // slice rows one copy step of the warp covers
  extern __shared__ __align__(128) unsigned char gvm_smem[];
  unsigned char* rings = gvm_smem;                                      // [warp][BUFS][kMmaPass][ROW]
  unsigned char* as = rings + size_t(kGvWarps) * Cfg::BUFS * Cfg::STAGE;  // [16][AROW]
  int32_t* rows = reinterpret_cast<int32_t*>(as + 16 * AROW);           // [kMmaChunk]
  float* cta = reinterpret_cast<float*>(rings);                         // [16][COLS], once the rings are drained

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();
  const int64_t b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = int64_t(blockIdx.x) * Cfg::COLS;
  // this lane's copies: slices lane / CPR + LPR·j of a pass, 8 columns at chunk lane % CPR of the warp's strip
  const int cchunk = lane % Cfg::CPR;
  const int64_t c = n0 + int64_t(warp) * WC + 8 * cchunk;
  const uint32_t src_bytes = c >= N ? 0u : uint32_t(min(int64_t(8), N - c) * 2);
  const uint16_t* Ab = A + b * sA;
  const uint16_t* Bc = B + b * sB + (src_bytes ? c : 0);  // this lane's column start in row 0
  const int32_t* ib = idx + b * k_keep;
  const int64_t per = (k_keep + cs - 1) / cs;
  const int64_t t_begin = min(k_keep, int64_t(crank) * per), t_end = min(k_keep, t_begin + per);
  const uint32_t ring_s = smem_addr(rings) + uint32_t(warp) * Cfg::BUFS * Cfg::STAGE, as_s = smem_addr(as);
  // ldmatrix lane roles: A x4 = (m 0-7 | 8-15) x (k 0-7 | 8-15) of a 16-slice step;
  // B x4.trans = (k 0-7 | 8-15) x (two of this warp's NT 8-column tiles)
  const int a_m = (lane & 7) + ((lane >> 3) & 1) * 8, a_kc = lane >> 4;
  const int b_k = (lane & 7) + ((lane >> 3) & 1) * 8, b_nt = lane >> 4;

  // rows m >= M of A stay zero for the whole kernel
  for (int e = tid; e < 16 * AROW / 16; e += kGvThreads)
    reinterpret_cast<uint4*>(as)[e] = make_uint4(0u, 0u, 0u, 0u);

  float d[NT][4];
#pragma unroll
  for (int t = 0; t < NT; ++t) d[t][0] = d[t][1] = d[t][2] = d[t][3] = 0.f;

  pdl_trigger();
  pdl_wait();
#pragma unroll 1
  for (int64_t c0 = t_begin; c0 < t_end; c0 += kMmaChunk) {
    const int nc = int(min(int64_t(kMmaChunk), t_end - c0));
    const int np = (nc + kMmaPass - 1) / kMmaPass;
    __syncthreads();  // every warp is done with the previous chunk's rows and A (and the zero fill is done)
    for (int i = tid; i < np * kMmaPass; i += kGvThreads) rows[i] = i < nc ? ib[c0 + i] : 0;
    __syncthreads();
    // this lane's copies of pass p (zeros past the chunk end); one commit group
    // per call in every lane, so that group counts stay uniform
    auto issue = [&](int p) {
      if (p < np) {
        const uint32_t boff = uint32_t(p % Cfg::BUFS) * Cfg::STAGE;
#pragma unroll
        for (int j = 0; j < Cfg::COPIES; ++j) {
          const int sl = lane / Cfg::CPR + LPR * j;  // slice within the pass
          const int i = p * kMmaPass + sl;
          const bool live = i < nc && src_bytes != 0;
          cp_async16_zfill(ring_s + boff + swz_strip<Cfg::CPR>(sl, cchunk), live ? Bc + int64_t(rows[i]) * ldb : Bc,
                           live ? src_bytes : 0u);
        }
      }
      cp_async_commit();
    };
#pragma unroll 1
    for (int q = 0; q < Cfg::BUFS - 1; ++q) issue(q);
    // A[m][idx] as bf16 bits for m < M (zero past the chunk end), loaded while
    // the first passes of B are in flight; all loads before the stores
    for (int i = tid; i < np * kMmaPass; i += kGvThreads) {
      const int32_t r = rows[i];
      uint16_t v[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) v[m] = (m < M && i < nc) ? __ldg(Ab + int64_t(m) * lda + r) : uint16_t(0);
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (m < M) *reinterpret_cast<uint16_t*>(as + swz(m, AROW, i >> 3) + (i & 7) * 2) = v[m];
    }
    __syncthreads();  // A's values of this chunk are visible to every warp
#pragma unroll 1
    for (int p = 0; p < np; ++p) {
      cp_async_wait<Cfg::BUFS - 2>();  // this lane's copies of pass p have landed
      __syncwarp();                    // and the whole warp's are visible to all its lanes
      const uint32_t rb = ring_s + uint32_t(p % Cfg::BUFS) * Cfg::STAGE;
#pragma unroll
      for (int kc = 0; kc < kMmaPass / 16; ++kc) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(as_s + swz(a_m, AROW, (p * kMmaPass + kc * 16) / 8 + a_kc), a0, a1, a2, a3);
#pragma unroll
        for (int t2 = 0; t2 < NT / 2; ++t2) {
          uint32_t b0, b1, b2, b3;
          ldsm_x4_t(rb + swz_strip<Cfg::CPR>(kc * 16 + b_k, 2 * t2 + b_nt), b0, b1, b2, b3);
          mma_bf16_16816(d[2 * t2], a0, a1, a2, a3, b0, b1);
          mma_bf16_16816(d[2 * t2 + 1], a0, a1, a2, a3, b2, b3);
        }
      }
      __syncwarp();  // every lane is done reading this buffer before it is refilled
      issue(p + Cfg::BUFS - 1);
    }
    cp_async_wait<0>();
  }
  __syncthreads();  // every warp is done with its ring: the partial takes their place
  // accumulator fragment of tile t: rows lane/4 and lane/4 + 8, columns 2·(lane%4) + {0, 1}
#pragma unroll
  for (int t = 0; t < NT; ++t) {
    const int col = warp * WC + t * 8 + (lane & 3) * 2;
    const int m = lane >> 2;
    cta[m * Cfg::COLS + col] = d[t][0];
    cta[m * Cfg::COLS + col + 1] = d[t][1];
    cta[(m + 8) * Cfg::COLS + col] = d[t][2];
    cta[(m + 8) * Cfg::COLS + col + 1] = d[t][3];
  }
  cluster.sync();
  cluster_sum_store(cluster, cta, Cfg::COLS, M, n0, N, b, sC, ldc, C, out_bf16, nullptr, kGvThreads);
  cluster.sync();
}

// cluster size (slices split over 1..8 CTAs): the one whose grid fills whole
// waves of two CTAs per SM best, each CTA keeping >= 64 slices
unsigned mma_cluster(int64_t blocks, int64_t k_keep, int sms) {
  unsigned best_q = 1;
  double best = -1.0;
  for (unsigned q = 1; q <= kGvMaxCluster; ++q) {
    if (q > 1 && k_keep < int64_t(q) * 64) break;
    const double waves = double(blocks * q) / double(2 * sms);
    const double eff = waves / std::max(1.0, std::ceil(waves));
    if (eff > best + 1e-9) {
      best = eff;
      best_q = q;
    }
  }
  return best_q;
}

template <int WC>
cudaError_t launch_mma(const GemvArgs& g, int sms, int dev, cudaStream_t st) {
  using Cfg = MmaCfg<WC>;
  static std::atomic<bool> attr_done[64];  // per device; racing first calls both set the attribute
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_gather_mma_kernel<WC>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(Cfg::SMEM));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  const int64_t mblk = (g.N + Cfg::COLS - 1) / Cfg::COLS;
  const unsigned mcs = mma_cluster(mblk * g.batch, g.k_keep, sms);
  return launch_pdl(gemv_gather_mma_kernel<WC>, dim3(unsigned(mblk), mcs, unsigned(g.batch)), dim3(kGvThreads),
                    Cfg::SMEM, st, dim3(1, mcs, 1), static_cast<const uint16_t*>(g.a), g.lda, g.strideA,
                    static_cast<const uint16_t*>(g.b), g.ldb, g.strideB, g.M, g.N, g.idx, g.k_keep, g.c, g.ldc,
                    g.strideC, int(g.out == kBF16));
}

template <typename T, int MT>
cudaError_t launch_mt(const GemvArgs& g, cudaStream_t st) {
  const size_t smem = gv_smem_bytes<MT>();
  static std::atomic<bool> attr_done[64];  // per device; racing first calls both set the attribute
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
  if (b_vec && sizeof(T) == 2) {
    // 512 columns per CTA when that grid, with clusters of up to 8 CTAs, can
    // fill a wave of two CTAs per SM; 256 otherwise (small layers)
    const int64_t wide = (g.N + MmaCfg<64>::COLS - 1) / MmaCfg<64>::COLS;
    if (wide * g.batch * int64_t(kGvMaxCluster) >= 2 * int64_t(sms))
      return launch_mma<64>(g, sms, dev, st);
    return launch_mma<32>(g, sms, dev, st);
  }
  if (b_vec) {
    const size_t asmem = gv_async_smem_bytes<T, MT>();
    static std::atomic<bool> async_attr[64];  // per device; racing first calls both set the attribute
    if (dev >= 0 && dev < 64 && !async_attr[dev]) {
      cudaError_t e = cudaFuncSetAttribute(gemv_gather_async_kernel<T, MT>,
                                           cudaFuncAttributeMaxDynamicSharedMemorySize, int(asmem));
      if (e != cudaSuccess) return e;
      async_attr[dev] = true;
    }
    return launch_pdl(gemv_gather_async_kernel<T, MT>, dim3(unsigned(nblk), cs, unsigned(g.batch)),
                      dim3(kGvThreads), asmem, st, dim3(1, cs, 1), a, g.lda, g.strideA, bp, g.ldb, g.strideB, g.M,
                      g.N, g.idx, g.k_keep, g.c, g.ldc, g.strideC, int(g.out == kBF16),
                      static_cast<const float*>(nullptr), int64_t(0));
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

// ---------------------------------------------------------------- INT8 weight, tensor cores
// The mma path for an INT8 weight. A CTA owns 512 columns of C, 64 per warp,
// and each warp streams its own 64-byte column strip of the kept rows through
// a private cp.async ring of 32-slice passes, so the main loop synchronises
// only within a warp; the whole block waits only while the indices and A's
// values of the next 512 slices are staged. Each thread converts its own
// bytes straight into the MMA's B fragments — no bf16 staging, no ldmatrix of
// B. A warp's 64 columns are two halves of four n8 tiles; within a half,
// fragment column g of tile j is weight column 4g + j, so one 32-bit shared
// load of a slice row gives a thread its byte for all four tiles. For a
// 16-slice step a thread loads rows 2t, 2t+1, 2t+8 and 2t+9 (t = lane % 4) —
// the rows of its b0/b1 fragment registers — converts them exactly
// (s8x4_to_f32) and packs byte j of rows 2t and 2t+1 (and of 2t+8, 2t+9) into
// tile j's b0 (b1); the 80-byte pitch of a warp's ring puts rows 2t of
// t = 0..3 eight banks apart, so these loads are free of bank conflicts.
// Column j of the sums is scaled by scale[j] at the end.
constexpr int kW8Cols = 512;                      // columns of C per CTA
constexpr int kW8WarpCols = kW8Cols / kGvWarps;   // one warp's column strip
constexpr int kW8Bufs = 4;                        // passes per warp ring (kW8Bufs - 1 in flight)
constexpr int kW8Chunk = 512;                     // slices whose indices and A values are staged at once
constexpr int kW8Pitch = kW8WarpCols + 16;        // bytes per slice row in a warp's ring
constexpr uint32_t kW8Stage = uint32_t(kMmaPass) * kW8Pitch;  // one pass of one warp

constexpr size_t gv_mma_w8_smem_bytes() {
  return size_t(kGvWarps) * kW8Bufs * kW8Stage  // warp rings (then the CTA's partial)
         + size_t(16) * kW8Chunk * 2            // A
         + size_t(kW8Chunk) * 4;                // row numbers
}
static_assert(size_t(16) * kW8Cols * 4 <= size_t(kGvWarps) * kW8Bufs * kW8Stage, "the partial fits in the rings");
static_assert(kW8WarpCols == 64, "two halves of four n8 tiles per warp");
static_assert(kMmaPass * (kW8WarpCols / 16) == 4 * 32, "four 16-byte copies per lane per pass");
static_assert((2 * (kW8Pitch / 4)) % 32 == 8 && kW8Pitch % 16 == 0, "rows 2t of t = 0..3 fall 8 banks apart");
static_assert(kW8Chunk % kMmaPass == 0, "whole passes per chunk");

// Requires Wq's rows (and its base) 16-byte aligned.
__global__ void __launch_bounds__(kGvThreads)
gemv_gather_mma_w8_kernel(const uint16_t* __restrict__ A, int64_t lda, int64_t sA, const int8_t* __restrict__ B,
                          int64_t ldb, int64_t sB, int64_t M, int64_t N, const int32_t* __restrict__ idx,
                          int64_t k_keep, void* __restrict__ C, int64_t ldc, int64_t sC, int out_bf16,
                          const float* __restrict__ scale, int64_t s_stride) {
  constexpr int AROW = kW8Chunk * 2;
  extern __shared__ __align__(128) unsigned char gvw_smem[];
  unsigned char* rings = gvw_smem;                                     // [warp][kW8Bufs][kMmaPass][kW8Pitch]
  unsigned char* as = rings + size_t(kGvWarps) * kW8Bufs * kW8Stage;   // [16][AROW]
  int32_t* rows = reinterpret_cast<int32_t*>(as + 16 * AROW);          // [kW8Chunk]
  float* cta = reinterpret_cast<float*>(rings);                        // [16][kW8Cols], once the rings are drained

  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();
  const int64_t b = blockIdx.z;
  const int tid = threadIdx.x, warp = tid >> 5, lane = tid & 31;
  const int64_t n0 = int64_t(blockIdx.x) * kW8Cols;
  // this lane's copies: slices lane/4 + 8j of a pass, 16 bytes at 16·(lane % 4) of the warp's strip
  const int64_t c = n0 + int64_t(warp) * kW8WarpCols + 16 * (lane & 3);
  const uint32_t src_bytes = c >= N ? 0u : uint32_t(min(int64_t(16), N - c));
  const uint16_t* Ab = A + b * sA;
  const int8_t* Bc = B + b * sB + (src_bytes ? c : 0);
  const int32_t* ib = idx + b * k_keep;
  const int64_t per = (k_keep + cs - 1) / cs;
  const int64_t t_begin = min(k_keep, int64_t(crank) * per), t_end = min(k_keep, t_begin + per);
  const unsigned char* ring = rings + size_t(warp) * kW8Bufs * kW8Stage;
  const uint32_t ring_s = smem_addr(ring), as_s = smem_addr(as);
  const uint32_t cp_off = uint32_t(lane >> 2) * kW8Pitch + uint32_t(lane & 3) * 16u;
  const int a_m = (lane & 7) + ((lane >> 3) & 1) * 8, a_kc = lane >> 4;
  const int g = lane >> 2, t = lane & 3;  // fragment group and thread-in-group
  // this thread's fragment bytes: row 2t of a step, columns 4g .. 4g + 3 of each half
  const uint32_t frag_off = uint32_t(2 * t) * kW8Pitch + uint32_t(4 * g);

  for (int e = tid; e < 16 * AROW / 16; e += kGvThreads) reinterpret_cast<uint4*>(as)[e] = make_uint4(0u, 0u, 0u, 0u);

  float d[8][4];
#pragma unroll
  for (int j = 0; j < 8; ++j) d[j][0] = d[j][1] = d[j][2] = d[j][3] = 0.f;

  pdl_trigger();
  pdl_wait();
#pragma unroll 1
  for (int64_t c0 = t_begin; c0 < t_end; c0 += kW8Chunk) {
    const int nc = int(min(int64_t(kW8Chunk), t_end - c0));
    const int np = (nc + kMmaPass - 1) / kMmaPass;
    __syncthreads();  // every warp is done with the previous chunk's rows and A (and the zero fill is done)
    for (int i = tid; i < np * kMmaPass; i += kGvThreads) rows[i] = i < nc ? ib[c0 + i] : 0;
    __syncthreads();
    // this lane's copies of pass p (zeros past the chunk end); one commit group
    // per call in every lane, so that group counts stay uniform
    auto issue = [&](int p) {
      if (p < np) {
        const uint32_t dst = ring_s + uint32_t(p % kW8Bufs) * kW8Stage + cp_off;
#pragma unroll
        for (int j = 0; j < 4; ++j) {
          const int i = p * kMmaPass + (lane >> 2) + 8 * j;
          const bool live = i < nc && src_bytes != 0;
          cp_async16_zfill(dst + uint32_t(8 * j) * kW8Pitch, live ? Bc + int64_t(rows[i]) * ldb : Bc,
                           live ? src_bytes : 0u);
        }
      }
      cp_async_commit();
    };
#pragma unroll 1
    for (int q = 0; q < kW8Bufs - 1; ++q) issue(q);
    // A's values while the first passes of B are in flight (all loads before the stores)
    for (int i = tid; i < np * kMmaPass; i += kGvThreads) {
      const int32_t r = rows[i];
      uint16_t v[16];
#pragma unroll
      for (int m = 0; m < 16; ++m) v[m] = (m < M && i < nc) ? __ldg(Ab + int64_t(m) * lda + r) : uint16_t(0);
#pragma unroll
      for (int m = 0; m < 16; ++m)
        if (m < M) *reinterpret_cast<uint16_t*>(as + swz(m, AROW, i >> 3) + (i & 7) * 2) = v[m];
    }
    __syncthreads();  // A's values of this chunk are visible to every warp
#pragma unroll 1
    for (int p = 0; p < np; ++p) {
      cp_async_wait<kW8Bufs - 2>();
      __syncwarp();  // the warp's copies of pass p are visible to all its lanes
      const unsigned char* rb = ring + size_t(p % kW8Bufs) * kW8Stage + frag_off;
#pragma unroll
      for (int kc = 0; kc < kMmaPass / 16; ++kc) {
        uint32_t a0, a1, a2, a3;
        ldsm_x4(as_s + swz(a_m, AROW, (p * kMmaPass + kc * 16) / 8 + a_kc), a0, a1, a2, a3);
        const unsigned char* r0 = rb + kc * 16 * kW8Pitch;
#pragma unroll
        for (int h = 0; h < 2; ++h) {
          // rows 2t, 2t+1, 2t+8, 2t+9 of the step; byte j of each is column 4g + j of tile j
          const uint32_t w0 = *reinterpret_cast<const uint32_t*>(r0 + 32 * h);
          const uint32_t w1 = *reinterpret_cast<const uint32_t*>(r0 + kW8Pitch + 32 * h);
          const uint32_t w2 = *reinterpret_cast<const uint32_t*>(r0 + 8 * kW8Pitch + 32 * h);
          const uint32_t w3 = *reinterpret_cast<const uint32_t*>(r0 + 9 * kW8Pitch + 32 * h);
          float f0[4], f1[4], f2[4], f3[4];
          s8x4_to_f32(w0, f0[0], f0[1], f0[2], f0[3]);
          s8x4_to_f32(w1, f1[0], f1[1], f1[2], f1[3]);
          s8x4_to_f32(w2, f2[0], f2[1], f2[2], f2[3]);
          s8x4_to_f32(w3, f3[0], f3[1], f3[2], f3[3]);
#pragma unroll
          for (int j = 0; j < 4; ++j)
            mma_bf16_16816(d[4 * h + j], a0, a1, a2, a3, pack_bf16x2_exact(f0[j], f1[j]),
                           pack_bf16x2_exact(f2[j], f3[j]));
        }
      }
      __syncwarp();  // every lane is done reading buffer p before it is refilled
      issue(p + kW8Bufs - 1);
    }
    cp_async_wait<0>();
  }
  __syncthreads();  // every warp is done with its ring: the partial reuses them
  // accumulator fragment of tile 4h + j: rows g and g + 8, fragment columns 2t and
  // 2t + 1, i.e. strip columns 32h + 4·(2t) + j and 32h + 4·(2t + 1) + j
#pragma unroll
  for (int h = 0; h < 2; ++h) {
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int col0 = warp * kW8WarpCols + 32 * h + 8 * t + j, col1 = col0 + 4;
      cta[g * kW8Cols + col0] = d[4 * h + j][0];
      cta[g * kW8Cols + col1] = d[4 * h + j][1];
      cta[(g + 8) * kW8Cols + col0] = d[4 * h + j][2];
      cta[(g + 8) * kW8Cols + col1] = d[4 * h + j][3];
    }
  }
  cluster.sync();
  cluster_sum_store(cluster, cta, kW8Cols, M, n0, N, b, sC, ldc, C, out_bf16, scale + b * s_stride, kGvThreads);
  cluster.sync();
}

template <int MT>
cudaError_t launch_w8_mt(const GemvArgs& g, const float* scale, int64_t s_stride, cudaStream_t st) {
  const size_t smem = gv_async_smem_bytes<int8_t, MT>();
  static std::atomic<bool> attr_done[64];  // per device; racing first calls both set the attribute
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(gemv_gather_async_kernel<uint16_t, MT, int8_t>,
                                         cudaFuncAttributeMaxDynamicSharedMemorySize, int(smem));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  int sms = 148;
  cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
  const int64_t nblk = (g.N + kGvCols - 1) / kGvCols;
  unsigned cs = 1;
  while (cs < kGvMaxCluster && nblk * g.batch * cs < 2 * int64_t(sms) && g.k_keep >= int64_t(cs) * 2 * 64) cs *= 2;
  return launch_pdl(gemv_gather_async_kernel<uint16_t, MT, int8_t>, dim3(unsigned(nblk), cs, unsigned(g.batch)),
                    dim3(kGvThreads), smem, st, dim3(1, cs, 1), static_cast<const uint16_t*>(g.a), g.lda, g.strideA,
                    static_cast<const int8_t*>(g.b), g.ldb, g.strideB, g.M, g.N, g.idx, g.k_keep, g.c, g.ldc,
                    g.strideC, int(g.out == kBF16), scale, s_stride);
}

}  // namespace

cudaError_t launch_gemv_gather_w8(const GemvArgs& g, const float* scale, int64_t s_stride, cudaStream_t st) {
  if (g.batch == 0 || g.M == 0 || g.N == 0) return cudaSuccess;
  if (g.M > kGemvMaxRows) return cudaErrorInvalidValue;
  if ((reinterpret_cast<uintptr_t>(g.b) % 16 == 0) && g.ldb % 16 == 0 && (g.batch == 1 || g.strideB % 16 == 0)) {
    const size_t smem = gv_mma_w8_smem_bytes();
    static std::atomic<bool> attr_done[64];  // per device; racing first calls both set the attribute
    int dev = 0, sms = 148;
    cudaGetDevice(&dev);
    if (dev >= 0 && dev < 64 && !attr_done[dev]) {
      cudaError_t e = cudaFuncSetAttribute(gemv_gather_mma_w8_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                           int(smem));
      if (e != cudaSuccess) return e;
      attr_done[dev] = true;
    }
    cudaDeviceGetAttribute(&sms, cudaDevAttrMultiProcessorCount, dev);
    const int64_t mblk = (g.N + kW8Cols - 1) / kW8Cols;
    const unsigned mcs = mma_cluster(mblk * g.batch, g.k_keep, sms);
    return launch_pdl(gemv_gather_mma_w8_kernel, dim3(unsigned(mblk), mcs, unsigned(g.batch)), dim3(kGvThreads),
                      smem, st, dim3(1, mcs, 1), static_cast<const uint16_t*>(g.a), g.lda, g.strideA,
                      static_cast<const int8_t*>(g.b), g.ldb, g.strideB, g.M, g.N, g.idx, g.k_keep, g.c, g.ldc,
                      g.strideC, int(g.out == kBF16), scale, s_stride);
  }
  if (g.M <= 1) return launch_w8_mt<1>(g, scale, s_stride, st);
  if (g.M <= 2) return launch_w8_mt<2>(g, scale, s_stride, st);
  if (g.M <= 4) return launch_w8_mt<4>(g, scale, s_stride, st);
  if (g.M <= 8) return launch_w8_mt<8>(g, scale, s_stride, st);
  return launch_w8_mt<16>(g, scale, s_stride, st);
}

cudaError_t launch_gemv_gather(const GemvArgs& g, cudaStream_t st) {
  if (g.batch == 0 || g.M == 0 || g.N == 0) return cudaSuccess;
  if (g.M > kGemvMaxRows) return cudaErrorInvalidValue;
  return g.in == kBF16 ? launch_t<uint16_t>(g, st) : launch_t<uint32_t>(g, st);
}

}  // namespace rmm
