// Top-k slice selection for RMM ("Estratégia de Seleção" on the gist.science
// summary of "Reduced Matrix Multiplication: Input-Adaptive Matrix-Product
// Reduction for LLM Inference": keep the k = ceil(rho·d) highest-scoring
// indices). Ties go to the lower index; the kept indices come out ascending.
//
// One 512-thread CTA per batch item. Thread t holds the run of keys
// [t·KPT, (t+1)·KPT) as order-preserving 32-bit keys in registers (K <= 32768,
// loaded 16 bytes at a time; larger K re-reads the scores from global memory,
// which stays in L2). The block's smallest and largest keys share every bit
// above the highest bit where they differ, so an MSB-first radix select
// starts there, 12 bits per pass:
//  * histogram: each candidate key adds one to its digit's bin with a shared
//    atomic (measured: warp-level merging of equal digits before the atomic,
//    by match.any or by ballots, costs more in vote latency than it saves);
//  * the bin of the k-th largest key: each thread sums 8 bins (top first), a
//    warp scan plus a scan of the 16 warp totals locates the crossing thread;
//  * the two histograms alternate, so clearing the next one needs no barrier
//    of its own; three barriers per pass, and the passes stop as soon as the
//    threshold bin is taken whole.
// Compaction in index order: every thread counts, in its own run, the keys
// above the threshold and those equal to it; one block scan of the two counts
// packed in 64 bits gives each thread its first output slot and how many of
// its equal keys are still kept (equal keys are kept lowest index first), and
// the thread writes its kept indices in order. Integer work only: the result
// depends on the order of the scores, never on rounding.
//
// Spare blocks of the same launch (in the fused call) zero the f32 C tiles
// that the GEMM's split-K round reduce-adds into, while one SM per batch item
// selects.
#include <algorithm>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int kSelThreads = 512;
constexpr int kSelWarps = kSelThreads / 32;
constexpr int kMaxKeysPerThread = 64;  // keys held in registers: K <= 32768
static_assert(int64_t(kSelThreads) * kMaxKeysPerThread == kSelectRegisterK, "register-key limit");
constexpr int kRowScoreKeys = 16;  // keys per thread up to which the selection can score A's rows
static_assert(int64_t(kSelThreads) * kRowScoreKeys == kRowScoreMaxK, "row-score limit");
constexpr int kDigitBits = 12;
constexpr int kBins = 1 << kDigitBits;
constexpr int kBinsPerThread = kBins / kSelThreads;
static_assert(kBinsPerThread == 8, "the bin scan reads 8 bins per thread as two vectors");
static_assert(kSelWarps <= 32, "warp totals are scanned by one warp");

// Order-preserving map from f32 to u32 (larger score -> larger key), with
// -0.0 folded onto +0.0 so that the two compare equal.
__device__ __forceinline__ uint32_t order_key(float x) {
  uint32_t u = __float_as_uint(x);
  if ((u & 0x7FFFFFFFu) == 0) u = 0;
  return (u & 0x80000000u) ? ~u : (u | 0x80000000u);
}

__device__ __forceinline__ uint32_t warp_incl_scan(uint32_t x, int lane) {
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint32_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  return x;
}

// Exclusive scan over the block of one 64-bit value per thread (used for two
// packed 32-bit counts); `wtot` holds kSelWarps entries and is free on entry.
__device__ __forceinline__ uint64_t block_excl_scan64(uint64_t v, uint64_t* wtot, int lane, int warp) {
  uint64_t x = v;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, x, o);
    if (lane >= o) x += y;
  }
  if (lane == 31) wtot[warp] = x;
  __syncthreads();
  uint64_t w = lane < kSelWarps ? wtot[lane] : 0ull;
#pragma unroll
  for (int o = 1; o < 32; o <<= 1) {
    const uint64_t y = __shfl_up_sync(0xffffffffu, w, o);
    if (lane >= o) w += y;
  }
  const uint64_t wprev = __shfl_sync(0xffffffffu, w, (warp + 31) & 31);  // warps before this one
  return (warp ? wprev : 0ull) + x - v;
}

// KPT > 0: thread t holds keys [t·KPT, (t+1)·KPT) in registers (K <= 512·KPT);
// KPT == 0: thread t owns [t·kpt, (t+1)·kpt), re-read from global memory in
// every sweep (any K up to 2^21).
template <int KPT>
__device__ __forceinline__ void select_item(float* __restrict__ sb, int K, int64_t k_keep,
                                            int32_t* __restrict__ ib, uint32_t* status, uint32_t (*hist)[kBins],
                                            uint32_t* wsum_a, uint32_t* wsum_b, uint64_t* wtot, uint32_t* sh,
                                            const RowScore& rs, int64_t item) {
  constexpr int R = KPT ? KPT : 1;  // register slots
  const int tid = threadIdx.x, lane = tid & 31, warp = tid >> 5;
  const int kpt = KPT ? KPT : (K + kSelThreads - 1) / kSelThreads;  // keys per thread
  const int base = tid * kpt;  // this thread's first key
  uint32_t key[R] = {};
  // key j of this thread (meaningful only when base + j < K)
  auto key_of = [&](int j) -> uint32_t {
    if constexpr (KPT > 0) {
      return key[j];
    } else {
      return order_key(sb[base + j]);
    }
  };

  // ---- keys, their min and max, non-finite check; hist[0] cleared meanwhile
  {
    uint4* h4 = reinterpret_cast<uint4*>(hist[0]);
    for (int v = tid; v < kBins / 4; v += kSelThreads) h4[v] = make_uint4(0u, 0u, 0u, 0u);
  }
  bool bad = false;
  uint32_t kmin = 0xFFFFFFFFu, kmax = 0u;
  auto take_key = [&](int j, float x) {
    bad |= !isfinite(x);
    const uint32_t k = order_key(x);
    if constexpr (KPT > 0) key[j] = k;
    kmin = min(kmin, k);
    kmax = max(kmax, k);
  };
  bool taken = false;  // keys computed from A's rows
  if constexpr (KPT > 0 && KPT <= kRowScoreKeys) {
    if (rs.A) {
      // Scores of this thread's run from A's rows (and B's row norms): per
      // key the rounded squares added in row order from 0, as the score
      // kernel's single CTA per strip adds its row lanes (one row each for
      // these M); then sqrt, then the product with ||B[k,:]||. Every operation
      // rounds on its own (no fused multiply-add), so the bits match. All
      // loads of a pair of rows (and the norms) are issued before any use:
      // one memory round trip per pair of rows.
      const bool full = base + KPT <= K;
      const float* bnb = rs.bn ? rs.bn + item * rs.bn_stride : nullptr;
      float nb[KPT];
      if (bnb) {
        if (KPT % 4 == 0 && full && (reinterpret_cast<uintptr_t>(bnb + base) & 15u) == 0) {
#pragma unroll
          for (int q = 0; q < KPT / 4; ++q) {
            const float4 v = reinterpret_cast<const float4*>(bnb + base)[q];
            nb[4 * q] = v.x;
            nb[4 * q + 1] = v.y;
            nb[4 * q + 2] = v.z;
            nb[4 * q + 3] = v.w;
          }
        } else {
#pragma unroll
          for (int q = 0; q < KPT; ++q) nb[q] = base + q < K ? bnb[base + q] : 0.f;
        }
      }
      float ss[KPT];
#pragma unroll
      for (int q = 0; q < KPT; ++q) ss[q] = 0.f;
      const int64_t e = rs.bf16 ? 2 : 4;
      const bool avec = rs.a_vec && full && (KPT * e) % 16 == 0;
      const unsigned char* a_run = static_cast<const unsigned char*>(rs.A) + (item * rs.sA + base) * e;
      for (int m0 = 0; m0 < rs.M; m0 += 2) {
        float x[2][KPT];
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          const int m = m0 + r;
#pragma unroll
          for (int q = 0; q < KPT; ++q) x[r][q] = 0.f;
          if (m >= rs.M) continue;
          const unsigned char* row = a_run + int64_t(m) * rs.lda * e;
          if (rs.bf16) {
            if (avec) {
#pragma unroll
              for (int q = 0; q < KPT / 8; ++q) {
                const uint4 u = reinterpret_cast<const uint4*>(row)[q];
                const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
                for (int h = 0; h < 4; ++h) {
                  x[r][8 * q + 2 * h] = __uint_as_float(w[h] << 16);
                  x[r][8 * q + 2 * h + 1] = __uint_as_float(w[h] & 0xFFFF0000u);
                }
              }
            } else {
#pragma unroll
              for (int q = 0; q < KPT; ++q)
                if (base + q < K) x[r][q] = bf16_to_f32(reinterpret_cast<const uint16_t*>(row)[q]);
            }
          } else {
            if (avec) {
#pragma unroll
              for (int q = 0; q < KPT / 4; ++q) {
                const float4 v = reinterpret_cast<const float4*>(row)[q];
                x[r][4 * q] = v.x;
                x[r][4 * q + 1] = v.y;
                x[r][4 * q + 2] = v.z;
                x[r][4 * q + 3] = v.w;
              }
            } else {
#pragma unroll
              for (int q = 0; q < KPT; ++q)
                if (base + q < K) x[r][q] = reinterpret_cast<const float*>(row)[q];
            }
          }
        }
#pragma unroll
        for (int r = 0; r < 2; ++r) {
          if (m0 + r >= rs.M) break;
#pragma unroll
          for (int q = 0; q < KPT; ++q) ss[q] = __fadd_rn(ss[q], __fmul_rn(x[r][q], x[r][q]));
        }
      }
      float sc[KPT];
#pragma unroll
      for (int q = 0; q < KPT; ++q) {
        sc[q] = sqrtf(ss[q]);
        if (bnb) sc[q] = __fmul_rn(sc[q], nb[q]);
        if (base + q < K) take_key(q, sc[q]);
      }
      // the scores, for the caller's workspace
      if (KPT % 4 == 0 && full && (reinterpret_cast<uintptr_t>(sb + base) & 15u) == 0) {
#pragma unroll
        for (int q = 0; q < KPT / 4; ++q)
          reinterpret_cast<float4*>(sb + base)[q] = make_float4(sc[4 * q], sc[4 * q + 1], sc[4 * q + 2], sc[4 * q + 3]);
      } else {
#pragma unroll
        for (int q = 0; q < KPT; ++q)
          if (base + q < K) sb[base + q] = sc[q];
      }
      taken = true;
    }
  }
  bool vec = false;
  if constexpr (KPT > 0 && KPT % 4 == 0) {
    // a whole run in range: 16-byte loads (a warp reads 128·KPT contiguous bytes)
    vec = !taken && base + KPT <= K && (reinterpret_cast<uintptr_t>(sb) & 15u) == 0;
    if (vec) {
#pragma unroll
      for (int j = 0; j < KPT; j += 4) {
        const float4 x = *reinterpret_cast<const float4*>(sb + base + j);
        take_key(j, x.x);
        take_key(j + 1, x.y);
        take_key(j + 2, x.z);
        take_key(j + 3, x.w);
      }
    }
  }
  if (!vec && !taken) {
#pragma unroll
    for (int j = 0; j < kpt; ++j)
      if (base + j < K) take_key(j, sb[base + j]);
  }
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  const bool bad_warp = __any_sync(0xffffffffu, bad);
  if (lane == 0) {
    wsum_a[warp] = kmin;
    wsum_b[warp] = kmax;
    if (bad_warp) status_or(status, RMM_NONFINITE_BIT);
  }
  __syncthreads();
  kmin = lane < kSelWarps ? wsum_a[lane] : 0xFFFFFFFFu;
  kmax = lane < kSelWarps ? wsum_b[lane] : 0u;
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) {
    kmin = min(kmin, __shfl_xor_sync(0xffffffffu, kmin, o));
    kmax = max(kmax, __shfl_xor_sync(0xffffffffu, kmax, o));
  }
  if (k_keep >= K) {  // everything is kept
    for (int i = tid; i < K; i += kSelThreads) ib[i] = i;
    return;
  }

  // ---- MSB-first radix select over the bits in which the keys differ. After
  // each pass, `prefix` (under `mask`) is the digit string of the k-th largest
  // key so far and `remaining` the number of keys still to take among those
  // matching it.
  const uint32_t diff = kmin ^ kmax;
  int hi = diff ? 31 - __clz(diff) : -1;  // highest unresolved bit
  uint32_t mask = hi >= 0 ? uint32_t(~((uint64_t(2) << hi) - 1)) : 0xFFFFFFFFu;
  uint32_t prefix = kmin & mask, remaining = uint32_t(k_keep), bin_count = uint32_t(K);
  int buf = 0;
  while (hi >= 0) {
    const int width = min(kDigitBits, hi + 1);
    const int shift = hi - width + 1;
    const uint32_t dmask = (1u << width) - 1u;
    uint32_t* h = hist[buf];
    {  // the other histogram was last read before the previous pass's final barrier
      uint4* h4 = reinterpret_cast<uint4*>(hist[buf ^ 1]);
      for (int v = tid; v < kBins / 4; v += kSelThreads) h4[v] = make_uint4(0u, 0u, 0u, 0u);
    }
#pragma unroll
    for (int j = 0; j < kpt; ++j) {
      if (base + j < K) {
        const uint32_t k = key_of(j);
        if ((k & mask) == prefix) atomicAdd(&h[(k >> shift) & dmask], 1u);
      }
    }
    __syncthreads();
    // thread t holds bins kBins-1-8t .. kBins-8-8t (top first)
    const uint4 hi4 = reinterpret_cast<const uint4*>(h)[kBins / 4 - 1 - 2 * tid];
    const uint4 lo4 = reinterpret_cast<const uint4*>(h)[kBins / 4 - 2 - 2 * tid];
    const uint32_t cnt[8] = {hi4.w, hi4.z, hi4.y, hi4.x, lo4.w, lo4.z, lo4.y, lo4.x};
    uint32_t c = 0;
#pragma unroll
    for (int q = 0; q < 8; ++q) c += cnt[q];
    const uint32_t incl = warp_incl_scan(c, lane);
    if (lane == 31) wsum_a[warp] = incl;
    __syncthreads();
    uint32_t wv = lane < kSelWarps ? wsum_a[lane] : 0u;
    wv = warp_incl_scan(wv, lane);
    const uint32_t wprev = __shfl_sync(0xffffffffu, wv, (warp + 31) & 31);  // warps before this one
    uint32_t acc = (warp ? wprev : 0u) + incl - c;
    if (acc < remaining && remaining <= acc + c) {
#pragma unroll
      for (int q = 0; q < 8; ++q) {
        if (acc + cnt[q] >= remaining) {
          sh[0] = uint32_t(kBins - 1 - 8 * tid - q);
          sh[1] = acc;
          sh[2] = cnt[q];
          break;
        }
        acc += cnt[q];
      }
    }
    __syncthreads();
    prefix |= sh[0] << shift;
    mask |= dmask << shift;
    remaining -= sh[1];
    bin_count = sh[2];
    buf ^= 1;
    // every key in the chosen bin is kept: no finer threshold is needed
    if (remaining == bin_count) break;
    hi = shift - 1;
  }

  // ---- compaction in index order. Kept: keys whose masked bits exceed
  // `prefix`, plus the `remaining` lowest-indexed keys whose masked bits equal
  // it (all of them when the bin is taken whole). Each thread counts both
  // kinds in its run; one block scan of the packed counts (equal keys in the
  // upper half) gives every thread its output slot and its share of equal keys.
  const uint32_t T = prefix, need_eq = remaining;
  const bool take_all_eq = remaining == bin_count;
  uint32_t n_gt = 0, n_eq = 0;
#pragma unroll
  for (int j = 0; j < kpt; ++j) {
    if (base + j < K) {
      const uint32_t k = key_of(j) & mask;
      n_gt += k > T;
      n_eq += k == T;
    }
  }
  // wtot is only ever used here (after the passes' barriers, or the first barrier)
  const uint64_t before = block_excl_scan64((uint64_t(n_eq) << 32) | n_gt, wtot, lane, warp);
  const uint32_t eq_before = uint32_t(before >> 32), gt_before = uint32_t(before);
  uint32_t eq_left = take_all_eq ? n_eq : (eq_before >= need_eq ? 0u : min(n_eq, need_eq - eq_before));
  uint32_t pos = gt_before + (take_all_eq ? eq_before : min(eq_before, need_eq));
#pragma unroll
  for (int j = 0; j < kpt; ++j) {
    if (base + j < K) {
      const uint32_t k = key_of(j) & mask;
      const bool tk = k > T || (k == T && eq_left > 0);
      if (k == T && eq_left > 0) --eq_left;
      if (tk) ib[pos++] = base + j;
    }
  }
}

template <int KPT>
__global__ void __launch_bounds__(kSelThreads, 1)
select_kernel(float* __restrict__ s, int64_t K64, int64_t k_keep, int32_t* __restrict__ idx,
              uint32_t* status, int64_t items, const SplitZero zero, int late_launch, const RowScore rs,
              int clear_status) {
  const int K = int(K64);  // K <= 2^21 (checked on the host)
  __shared__ __align__(16) uint32_t hist[2][kBins];
  __shared__ uint32_t wsum_a[kSelWarps], wsum_b[kSelWarps];
  __shared__ uint64_t wtot[kSelWarps];
  __shared__ uint32_t sh[3];

  // late_launch: the next kernel (a gather-GEMV in clusters of CTAs with
  // large shared memory) is released only once the previous kernel has
  // completed (pdl_wait returns after that); released before, it would be
  // placed around the previous kernel's CTAs and part of it would run as a
  // second wave
  if (!late_launch) pdl_trigger();
  pdl_wait();
  if (late_launch) pdl_trigger();
  if (clear_status) {  // a launch of one block, the call's first kernel
    if (threadIdx.x == 0) *status = 0u;
    __syncthreads();
  }
  if (blockIdx.x >= items) {  // helper block: zero C tiles for the GEMM later on the stream
    zero_split_tiles(zero, blockIdx.x - items, gridDim.x - items, threadIdx.x, kSelThreads);
    return;
  }
  select_item<KPT>(s + int64_t(blockIdx.x) * K, K, k_keep, idx + int64_t(blockIdx.x) * k_keep, status, hist,
                   wsum_a, wsum_b, wtot, sh, rs, int64_t(blockIdx.x));
}

}  // namespace

cudaError_t launch_select(float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx,
                          uint32_t* status, cudaStream_t st, const SplitZero* zero, bool late_launch,
                          const RowScore* rows, bool clear_status) {
  if (batch == 0) return cudaSuccess;
  SplitZero z = {};
  int64_t helpers = 0;
  if (zero && zero->count > 0) {
    z = *zero;
    const int64_t vecs = z.count * z.tile_rows * (z.tile_cols / 4);
    helpers = std::min<int64_t>(147, (vecs + 4 * kSelThreads - 1) / (4 * kSelThreads));
  }
  RowScore rs = {};
  if (rows) {
    if (K > kRowScoreMaxK || rows->M > kRowScoreMaxM) return cudaErrorInvalidValue;
    rs = *rows;
  }
  if (clear_status && batch + helpers != 1) return cudaErrorInvalidValue;
  const dim3 grid(unsigned(batch + helpers)), block(kSelThreads), none(0, 0, 0);
  const int ll = int(late_launch), cl = int(clear_status);
  const int64_t kpt = (K + kSelThreads - 1) / kSelThreads;
#define RMM_SELECT(KPT_) \
  launch_pdl(select_kernel<KPT_>, grid, block, 0, st, none, s, K, k_keep, idx, status, batch, z, ll, rs, cl)
  if (kpt <= 1) return RMM_SELECT(1);
  if (kpt <= 2) return RMM_SELECT(2);
  if (kpt <= 4) return RMM_SELECT(4);
  if (kpt <= 8) return RMM_SELECT(8);
  if (kpt <= 16) return RMM_SELECT(16);
  if (kpt <= 32) return RMM_SELECT(32);
  if (kpt <= kMaxKeysPerThread) return RMM_SELECT(kMaxKeysPerThread);
  return RMM_SELECT(0);
#undef RMM_SELECT
}

}  // namespace rmm
