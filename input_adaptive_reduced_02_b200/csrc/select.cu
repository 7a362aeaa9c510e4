// Top-k slice selection for RMM ("Estratégia de Seleção" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference": keep the k = ceil(rho·d) highest-scoring
// indices). Ties go to the lower index; the kept indices come out ascending.
//
// One 1024-thread CTA per batch item. Scores become order-preserving 32-bit
// keys in shared memory (up to 32768 of them; larger K re-reads the scores
// from global memory, which stays in L2). The block's smallest and largest
// keys share every bit above the highest bit where they differ, so an
// MSB-first radix select starts there: 11-bit digits counted into one shared
// histogram with shared-memory atomics, a block scan to find the bin of the
// k-th largest key, and an early stop as soon as that bin is kept whole. Two
// block-wide scans then compact the kept indices in index order (ties: the
// lowest indices among keys equal to the threshold). Integer work only: the
// result depends on the order of the scores, never on rounding.
//
// Spare blocks of the same launch (in the fused call) zero the f32 C tiles
// that the GEMM's split-K round reduce-adds into, while one SM per batch item
// selects.
#include <algorithm>
#include <atomic>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int64_t kSelSmemKeys = 32768;

// Order-preserving map from f32 to u32 (larger score -> larger key), with
// -0.0 folded onto +0.0 so that the two compare equal.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

// Exclusive scan of one value per thread over the block; *total receives the sum.
template <int THREADS>
__device__ __forceinline__ uint32_t block_exclusive_scan(uint32_t v, uint32_t* warp_sums, uint32_t* total) {
  constexpr int kWarps = THREADS / 32;
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
    uint32_t w = lane < kWarps ? warp_sums[lane] : 0u;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, w, o);
      if (lane >= o) w += y;
    }
    if (lane < kWarps) warp_sums[lane] = w;
  }
  __syncthreads();
  const uint32_t before = (warp ? warp_sums[warp - 1] : 0u) + x - v;
  *total = warp_sums[kWarps - 1];
  __syncthreads();
  return before;
}

constexpr int kSelThreads = 1024;
constexpr int kDigitBits = 11;
constexpr int kBins = 1 << kDigitBits;

template <int THREADS>
__global__ void __launch_bounds__(THREADS, 1)
select_kernel(const float* __restrict__ s, int64_t K64, int64_t k_keep, int32_t* __restrict__ idx,
              uint32_t* status, int keys_in_smem, int64_t items, const SplitZero zero, int late_launch) {
  constexpr int kWarps = THREADS / 32;
  const int K = int(K64);  // K <= 2^21 (checked on the host)
  extern __shared__ uint32_t keys[];  // K keys when keys_in_smem
  __shared__ uint32_t hist[kBins];
  __shared__ uint32_t warp_sums[32];
  __shared__ uint32_t warp_min[kWarps], warp_max[kWarps];
  __shared__ uint32_t sh_digit, sh_above, sh_count;
  __shared__ int sh_nan;

  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const float* sb = s + int64_t(blockIdx.x) * K;
  int32_t* ib = idx + int64_t(blockIdx.x) * k_keep;

  // late_launch: the next kernel (a gather-GEMV in clusters of CTAs with
  // large shared memory) is released only once the previous kernel has
  // completed (pdl_wait returns after that); released before, it would be
  // placed around the previous kernel's CTAs and part of it would run as a
  // second wave
  if (!late_launch) pdl_trigger();
  pdl_wait();
  if (late_launch) pdl_trigger();
  if (blockIdx.x >= items) {  // helper block: zero C tiles for the GEMM later on the stream
    zero_split_tiles(zero, blockIdx.x - items, gridDim.x - items, tid, THREADS);
    return;
  }
  if (tid == 0) sh_nan = 0;
  __syncthreads();
  bool nan_seen = false;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  if (keys_in_smem && (K & 3) == 0 && (reinterpret_cast<uintptr_t>(sb) & 15u) == 0) {
    const float4* s4 = reinterpret_cast<const float4*>(sb);
    for (int i = tid; i < K / 4; i += THREADS) {
      const float4 x = s4[i];
      nan_seen |= !isfinite(x.x) | !isfinite(x.y) | !isfinite(x.z) | !isfinite(x.w);
      const uint4 k4 = make_uint4(order_key(x.x), order_key(x.y), order_key(x.z), order_key(x.w));
      kmin = min(min(kmin, min(k4.x, k4.y)), min(k4.z, k4.w));
      kmax = max(max(kmax, max(k4.x, k4.y)), max(k4.z, k4.w));
      reinterpret_cast<uint4*>(keys)[i] = k4;
    }
  } else {
    for (int i = tid; i < K; i += THREADS) {
      const float x = sb[i];
      nan_seen |= !isfinite(x);
      const uint32_t k = order_key(x);
      kmin = min(kmin, k);
      kmax = max(kmax, k);
      if (keys_in_smem) keys[i] = k;
    }
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (lane == 0) {
    warp_min[warp] = kmin;
    warp_max[warp] = kmax;
  }
  if (nan_seen) sh_nan = 1;
  __syncthreads();
  if (tid == 0 && sh_nan) status_or(status, RMM_NONFINITE_BIT);
  kmin = warp_min[0];
  kmax = warp_max[0];
  for (int w = 1; w < kWarps; ++w) {
    kmin = min(kmin, warp_min[w]);
    kmax = max(kmax, warp_max[w]);
  }

  if (k_keep >= K) {  // everything is kept
    for (int i = tid; i < K; i += THREADS) ib[i] = i;
    return;
  }

  // MSB-first radix select over the bits in which the keys differ: every key
  // shares the bits of kmin above the highest bit where kmin and kmax differ,
  // so the first histogram already spreads the keys over many bins. After
  // each pass, `prefix` (under `mask`) is the digit string of the k-th largest
  // key so far and `remaining` the number of keys still to take among those
  // matching it.
  const uint32_t diff = kmin ^ kmax;
  int hi = diff ? 31 - __clz(diff) : -1;  // highest unresolved bit
  uint32_t mask = hi >= 0 ? uint32_t(~((uint64_t(2) << hi) - 1)) : 0xFFFFFFFFu;
  uint32_t prefix = kmin & mask, remaining = uint32_t(k_keep), bin_count = uint32_t(K);
  while (hi >= 0) {
    const int width = min(kDigitBits, hi + 1);
    const int shift = hi - width + 1;
    const uint32_t dmask = (1u << width) - 1u;
    for (int b = tid; b < kBins; b += THREADS) hist[b] = 0u;
    __syncthreads();
    for (int i = tid; i < K; i += THREADS) {
      const uint32_t key = keys_in_smem ? keys[i] : order_key(sb[i]);
      if ((key & mask) == prefix) atomicAdd(&hist[(key >> shift) & dmask], 1u);
    }
    __syncthreads();
    // descending scan to find the bin of the k-th key: thread t owns bins
    // kBins-1-2t and kBins-2-2t
    uint32_t c0 = 0, c1 = 0;
    if (tid < kBins / 2) {
      c0 = hist[kBins - 1 - 2 * tid];
      c1 = hist[kBins - 2 - 2 * tid];
    }
    uint32_t all;
    const uint32_t excl = block_exclusive_scan<THREADS>(c0 + c1, warp_sums, &all);
    if (tid < kBins / 2 && excl < remaining && remaining <= excl + c0 + c1) {
      if (excl + c0 >= remaining) {
        sh_digit = uint32_t(kBins - 1 - 2 * tid);
        sh_above = excl;
        sh_count = c0;
      } else {
        sh_digit = uint32_t(kBins - 2 - 2 * tid);
        sh_above = excl + c0;
        sh_count = c1;
      }
    }
    __syncthreads();
    prefix |= sh_digit << shift;
    mask |= dmask << shift;
    remaining -= sh_above;
    bin_count = sh_count;
    // every key in the chosen bin is kept: no finer threshold is needed
    if (remaining == bin_count) break;
    hi = shift - 1;
  }
  // Kept: keys whose masked bits exceed `prefix`, plus the `remaining`
  // lowest-indexed keys whose masked bits equal it (all of them when the bin
  // is taken whole). Larger K: warp w compacts the contiguous chunk w of the
  // keys, 32 consecutive keys per step (conflict-free shared-memory reads; a
  // contiguous run per thread would read 32 runs in one bank), in two sweeps:
  // counts, then writes at offsets from a scan over the warps' counts.
  const uint32_t T = prefix, need_eq = remaining;
  const bool take_all_eq = remaining == bin_count;
  if (K <= 4 * THREADS) {
    // up to 4 keys per thread: a contiguous run each and two block scans
    // (measured faster than the warp sweeps below at this size)
    const int per = (K + THREADS - 1) / THREADS;
    const int lo = min(K, tid * per), hi_i = min(K, lo + per);
    uint32_t c_gt = 0, c_eq = 0;
    for (int i = lo; i < hi_i; ++i) {
      const uint32_t k = (keys_in_smem ? keys[i] : order_key(sb[i])) & mask;
      c_gt += (k > T);
      c_eq += (k == T);
    }
    uint32_t total, eq_take = c_eq;
    if (!take_all_eq) {
      const uint32_t eq_before = block_exclusive_scan<THREADS>(c_eq, warp_sums, &total);
      eq_take = eq_before >= need_eq ? 0u : min(c_eq, need_eq - eq_before);
    }
    uint32_t pos = block_exclusive_scan<THREADS>(c_gt + eq_take, warp_sums, &total);
    uint32_t taken_eq = 0;
    for (int i = lo; i < hi_i; ++i) {
      const uint32_t k = (keys_in_smem ? keys[i] : order_key(sb[i])) & mask;
      if (k > T) {
        ib[pos++] = i;
      } else if (k == T && taken_eq < eq_take) {
        ib[pos++] = i;
        ++taken_eq;
      }
    }
    return;
  }
  const int chunk = (K + kWarps - 1) / kWarps;
  const int w_lo = min(K, warp * chunk), w_hi = min(K, w_lo + chunk);
  const uint32_t lt_mask = (1u << lane) - 1u;
  uint32_t n_gt = 0, n_eq = 0;
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const bool valid = i < w_hi;
    const uint32_t k = valid ? ((keys_in_smem ? keys[i] : order_key(sb[i])) & mask) : 0u;
    n_gt += __popc(__ballot_sync(0xffffffffu, valid && k > T));
    n_eq += __popc(__ballot_sync(0xffffffffu, valid && k == T));
  }
  // exclusive scans over the warps (in warp order) of the equal counts and of
  // the kept counts; warp_min/warp_max are free again (the barrier covers the
  // case without radix passes, where they were last read for kmin/kmax)
  __syncthreads();
  if (lane == 0) {
    warp_min[warp] = n_eq;
    warp_max[warp] = n_gt;
  }
  __syncthreads();
  if (warp == 0) {
    const uint32_t e = lane < kWarps ? warp_min[lane] : 0u, g = lane < kWarps ? warp_max[lane] : 0u;
    uint32_t e_incl = e;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, e_incl, o);
      if (lane >= o) e_incl += y;
    }
    const uint32_t e_before = e_incl - e;
    const uint32_t take = take_all_eq ? e : (e_before >= need_eq ? 0u : min(e, need_eq - e_before));
    uint32_t k_incl = g + take;
#pragma unroll
    for (int o = 1; o < 32; o <<= 1) {
      const uint32_t y = __shfl_up_sync(0xffffffffu, k_incl, o);
      if (lane >= o) k_incl += y;
    }
    if (lane < kWarps) {
      warp_min[lane] = take;                  // equal keys this warp keeps
      warp_max[lane] = k_incl - (g + take);   // first output slot of this warp
    }
  }
  __syncthreads();
  const uint32_t eq_take = warp_min[warp];
  uint32_t pos = warp_max[warp], eq_seen = 0;
  for (int base = w_lo; base < w_hi; base += 32) {
    const int i = base + lane;
    const bool valid = i < w_hi;
    const uint32_t k = valid ? ((keys_in_smem ? keys[i] : order_key(sb[i])) & mask) : 0u;
    const bool gt = valid && k > T, eq = valid && k == T;
    const uint32_t eq_mask = __ballot_sync(0xffffffffu, eq);
    const bool take = gt || (eq && eq_seen + __popc(eq_mask & lt_mask) < eq_take);
    const uint32_t t_mask = __ballot_sync(0xffffffffu, take);
    if (take) ib[pos + __popc(t_mask & lt_mask)] = i;
    pos += __popc(t_mask);
    eq_seen += __popc(eq_mask);
  }
}

}  // namespace

cudaError_t launch_select(const float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx,
                          uint32_t* status, cudaStream_t st, const SplitZero* zero, bool late_launch) {
  if (batch == 0) return cudaSuccess;
  SplitZero z = {};
  int64_t helpers = 0;
  if (zero && zero->count > 0) {
    z = *zero;
    const int64_t vecs = z.count * z.tile_rows * (z.tile_cols / 4);
    helpers = std::min<int64_t>(147, (vecs + 8 * kSelThreads - 1) / (8 * kSelThreads));
  }
  const int keys_in_smem = K <= kSelSmemKeys;
  const size_t smem = keys_in_smem ? size_t(K) * 4 : 0;
  static std::atomic<bool> attr_done[64];  // per device; racing first calls both set the attribute
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(select_kernel<kSelThreads>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kSelSmemKeys * 4));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  return launch_pdl(select_kernel<kSelThreads>, dim3(unsigned(batch + helpers)), dim3(kSelThreads), smem, st,
                    dim3(0, 0, 0), s, K, k_keep, idx, status, keys_in_smem, batch, z, int(late_launch));
}

}  // namespace rmm
