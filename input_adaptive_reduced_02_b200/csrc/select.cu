// Top-k slice selection for RMM ("Estratégia de Seleção" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference": keep the k = ceil(rho·d) highest-scoring
// indices). Ties go to the lower index; the kept indices come out ascending.
//
// One 1024-thread CTA per batch item. Scores become order-preserving 32-bit
// keys in shared memory (up to 32768 of them; larger K re-reads the scores
// from global memory, which stays in L2). A 4-pass MSB-first radix select
// (8-bit digits) finds the exact key T of the k-th largest score and how many
// keys equal to T must be kept; per-warp histograms with match-any
// aggregation avoid hot-bin atomic contention. Two block-wide scans then
// compact the kept indices in index order. Integer work only: the result
// depends on the order of the scores, never on rounding.
#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kSelThreads = 1024;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int64_t kSelSmemKeys = 32768;

// Order-preserving map from f32 to u32 (larger score -> larger key), with
// -0.0 folded onto +0.0 so that the two compare equal.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one value per thread over the block; *total receives the sum.
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  const int lane = threadIdx.x & 31, warp = threadIdx.x >> 5;
  uint32_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) warp_sums[warp] = x;
  __syncthreads();
  if (warp == 0) {
    uint32_t w = warp_sums[lane];
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    warp_sums[lane] = w;
  }
  __syncthreads();
  const uint32_t before = (warp ? warp_sums[warp - 1] : 0u) + x - v;
  *total = warp_sums[kSelWarps - 1];
  __syncthreads();
  return before;
}

__global__ void __launch_bounds__(kSelThreads, 1)
select_kernel(const float* __restrict__ s, int64_t K, int64_t k_keep, int32_t* __restrict__ idx,
              uint32_t* status, int keys_in_smem) {
  extern __shared__ uint32_t keys[];
  __shared__ uint32_t hist[kSelWarps][256];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t sh_digit, sh_above;
  __shared__ int sh_nan;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* sb = s + int64_t(blockIdx.x) * K;
  int32_t* ib = idx + int64_t(blockIdx.x) * k_keep;

  if (tid == 0) sh_nan = 0;
  __syncthreads();
  bool nan_seen = false;
  for (int64_t i = tid; i < K; i += kSelThreads) {
    const float x = sb[i];
    nan_seen |= (x != x);
    if (keys_in_smem) keys[i] = order_key(x);
  }
  if (nan_seen) sh_nan = 1;
  __syncthreads();
  if (tid == 0 && sh_nan) status_or(status, RMM_NONFINITE_BIT);

  if (k_keep >= K) {  // everything is kept
    for (int64_t i = tid; i < K; i += kSelThreads) ib[i] = int32_t(i);
    return;
  }

  uint32_t prefix = 0, mask = 0, remaining = uint32_t(k_keep);
  for (int shift = 24; shift >= 0; shift -= 8) {
    for (int i = tid; i < kSelWarps * 256; i += kSelThreads) (&hist[0][0])[i] = 0u;
    __syncthreads();
    for (int64_t i0 = int64_t(warp) * 32; i0 < K; i0 += kSelThreads) {
      const int64_t i = i0 + lane;
      uint32_t key = 0;
      bool active = false;
      if (i < K) {
        key = keys_in_smem ? keys[i] : order_key(sb[i]);
        active = (key & mask) == prefix;
      }
      const unsigned am = __ballot_sync(0xffffffffu, active);
      if (active) {
        const uint32_t d = (key >> shift) & 0xFFu;
        const unsigned peers = __match_any_sync(am, d);
        if (lane == __ffs(peers) - 1) atomicAdd(&hist[warp][d], uint32_t(__popc(peers)));
      }
    }
    __syncthreads();
    if (tid < 256) {
      uint32_t t = 0;
      for (int w = 0; w < kSelWarps; ++w) t += hist[w][tid];
      hist[0][tid] = t;
    }
    __syncthreads();
    if (warp == 0) {
      // lane l owns digits 255-8l .. 248-8l, scanned from the top digit down
      uint32_t c[8], local = 0;
#pragma unroll
      for (int j = 0; j < 8; ++j) {
        c[j] = hist[0][255 - 8 * lane - j];
        local += c[j];
      }
      uint32_t incl = local;
#pragma unroll
      for (int o = 1; o < 32; o <<= 1) {
        const uint32_t y = __shfl_up_sync(0xffffffffu, incl, o);
        if (lane >= o) incl += y;
      }
      const uint32_t excl = incl - local;
      if (excl < remaining && remaining <= incl) {
        uint32_t run = excl;
#pragma unroll
        for (int j = 0; j < 8; ++j) {
          if (run + c[j] >= remaining) {
            sh_digit = uint32_t(255 - 8 * lane - j);
            sh_above = run;
            break;
          }
          run += c[j];
        }
      }
    }
    __syncthreads();
    prefix |= sh_digit << shift;
    mask |= 0xFFu << shift;
    remaining -= sh_above;
  }
  // prefix is now the exact key T of the k-th largest score; `remaining` keys
  // equal to T are kept (the lowest-indexed ones), plus every key above T.
  const uint32_t T = prefix, need_eq = remaining;
  const int64_t per = (K + kSelThreads - 1) / kSelThreads;
  const int64_t lo = min(K, int64_t(tid) * per), hi = min(K, lo + per);
  uint32_t n_gt = 0, n_eq = 0;
  for (int64_t i = lo; i < hi; ++i) {
    const uint32_t k = keys_in_smem ? keys[i] : order_key(sb[i]);
    n_gt += (k > T);
    n_eq += (k == T);
  }
  uint32_t total;
  const uint32_t eq_before = block_exclusive_scan(n_eq, warp_sums, &total);
  const uint32_t eq_take = eq_before >= need_eq ? 0u : min(n_eq, need_eq - eq_before);
  uint32_t pos = block_exclusive_scan(n_gt + eq_take, warp_sums, &total);
  uint32_t taken_eq = 0;
  for (int64_t i = lo; i < hi; ++i) {
    const uint32_t k = keys_in_smem ? keys[i] : order_key(sb[i]);
    if (k > T) {
      ib[pos++] = int32_t(i);
    } else if (k == T && taken_eq < eq_take) {
      ib[pos++] = int32_t(i);
      ++taken_eq;
    }
  }
}

}  // namespace

cudaError_t launch_select(const float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx,
                          uint32_t* status, cudaStream_t st) {
  if (batch == 0) return cudaSuccess;
  const int keys_in_smem = K <= kSelSmemKeys;
  const size_t smem = keys_in_smem ? size_t(K) * 4 : 0;
  static bool attr_done[64] = {};
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSelSmemKeys * 4));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  count_launch();
  select_kernel<<<unsigned(batch), kSelThreads, smem, st>>>(s, K, k_keep, idx, status, keys_in_smem);
  return cudaGetLastError();
}

}  // namespace rmm
