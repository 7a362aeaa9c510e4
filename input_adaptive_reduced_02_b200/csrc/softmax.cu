// The attention matrix P of P·V produced from its logits, with the slice
// score of the reduced product P·V accumulated while P is written ("Escopo de
// Aplicação" on the gist.science summary of "Reduced Matrix Multiplication:
// Input-Adaptive Matrix-Product Reduction for LLM Inference": P·V reduced over
// the keys; "Estratégia de Seleção": score each key by a norm). The key score
// s_k = ||P[:, k]||_2 · ||V[k, :]||_2 needs the column sums of squares of P,
// which a producer that writes P column strip by column strip has in hand, so
// P is never read back to score it.
//
// Two launches per call:
//  * softmax_stats_kernel: one warp per query row streams the row's visible
//    logits once (16-byte loads, several in flight) and keeps a running
//    maximum and rescaled sum of exp2: stats[q] = (max of x, 1 / sum exp2(x -
//    max)) with x = scale·log2(e)·L, the row's normalisation.
//  * softmax_score_kernel: a cluster of up to 8 CTAs per (128-key strip, head)
//    splits the strip's query rows: p = exp2(x - max)·(1/sum) for visible
//    keys, 0 for masked ones, rounded to bf16 (nearest even) and stored
//    (16-byte stores), and the squares of the stored values summed per key
//    column in a fixed order (each thread in row order, the 32 row lanes in
//    order, then the cluster's CTAs in rank order through distributed shared
//    memory). Rows whose keys in the strip are all masked are written as
//    zeros without reading their logits. The strip's ||V[k, :]||^2 come from a
//    warp per key; the kernel writes s_k (or P alone when no score is asked
//    for). Splitting the rows keeps the strips near the first key (which
//    every query sees) from running far longer than the others.
// With the causal mask query q sees key k when k <= q + S_k - S_q (the last
// query sees every key), so about half of the logits are never read.
#include <algorithm>
#include <atomic>
#include <cooperative_groups.h>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace cg = cooperative_groups;

namespace rmm {
namespace {

constexpr int kSmThreads = 256;
constexpr unsigned kSmMaxCluster = 8;  // CTAs splitting one strip's rows
constexpr int kStrip = 128;     // keys per CTA of the score kernel (256-byte row segments for bf16)
constexpr int kRowUnroll = 8;   // rows per ring stage per thread
constexpr int kRing = 3;        // ring stages (two in flight while one is used)
// ring of 16-byte logits slots per thread, then the rows' statistics (float2
// per row lane; 32 row lanes at most)
constexpr size_t kScoreSmem = size_t(kRing) * kRowUnroll * kSmThreads * 16 + size_t(kRing) * kRowUnroll * 32 * 8;
constexpr float kLog2e = 1.4426950408889634f;

__device__ __forceinline__ uint4 ld_nc16(const void* p) {
  uint4 v;
  asm volatile("ld.global.nc.L1::no_allocate.v4.u32 {%0, %1, %2, %3}, [%4];"
               : "=r"(v.x), "=r"(v.y), "=r"(v.z), "=r"(v.w)
               : "l"(p));
  return v;
}

// Elements of one 16-byte vector as f32.
__device__ __forceinline__ void unpack16(uint4 u, float (&x)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int j = 0; j < 4; ++j) {
    x[2 * j] = __uint_as_float(w[j] << 16);
    x[2 * j + 1] = __uint_as_float(w[j] & 0xFFFF0000u);
  }
}
__device__ __forceinline__ void unpack16(uint4 u, float (&x)[4]) {
  x[0] = __uint_as_float(u.x);
  x[1] = __uint_as_float(u.y);
  x[2] = __uint_as_float(u.z);
  x[3] = __uint_as_float(u.w);
}

// 2^x by the SFU instruction (PTX ex2.approx.ftz.f32: relative error below
// 2^-22, subnormal results flushed to zero, 2^-inf = 0).
__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ void cp_async_zfill16(uint32_t smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.cg.shared.global [%0], [%1], 16, %2;" ::"r"(smem_dst), "l"(gsrc), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_zfill8(uint32_t smem_dst, const void* gsrc, uint32_t src_bytes) {
  asm volatile("cp.async.ca.shared.global [%0], [%1], 8, %2;" ::"r"(smem_dst), "l"(gsrc), "r"(src_bytes) : "memory");
}
__device__ __forceinline__ void cp_async_commit_group() { asm volatile("cp.async.commit_group;" ::: "memory"); }
template <int N>
__device__ __forceinline__ void cp_async_wait_group() { asm volatile("cp.async.wait_group %0;" ::"n"(N) : "memory"); }

__device__ __forceinline__ int64_t visible_keys(int64_t q, int64_t S_q, int64_t S_k, int causal) {
  return causal ? min(S_k, q + 1 + (S_k - S_q)) : S_k;
}

// Fold x into a running (max m, sum of exp2(. - m)) pair.
__device__ __forceinline__ void online_add(float& m, float& s, float x) {
  if (x > m) {
    s = s * ex2(m - x) + 1.f;
    m = x;
  } else {
    s += ex2(x - m);
  }
}

// Merge two running pairs.
__device__ __forceinline__ void online_merge(float& m, float& s, float m2, float s2) {
  if (m2 > m) {
    s = s * ex2(m - m2) + s2;
    m = m2;
  } else if (m2 > -INFINITY) {
    s += s2 * ex2(m2 - m);
  }
}

// T: logits element (uint16_t = bf16 bits, uint32_t = f32 bits).
template <typename T>
__global__ void __launch_bounds__(kSmThreads)
softmax_stats_kernel(const T* __restrict__ L, int64_t bh, int64_t S_q, int64_t S_k, float xscale, int causal,
                     int vec, float2* __restrict__ stats, uint32_t* status, int clear_status) {
  constexpr int V = 16 / sizeof(T);
  constexpr int U = 4;  // vectors in flight per lane
  pdl_trigger();
  pdl_wait();
  if (clear_status && blockIdx.x == 0 && threadIdx.x == 0 && status) *status = 0u;
  const int lane = threadIdx.x & 31;
  const int64_t rows = bh * S_q;
  const int64_t warps = int64_t(gridDim.x) * (kSmThreads / 32);
  for (int64_t row = int64_t(blockIdx.x) * (kSmThreads / 32) + (threadIdx.x >> 5); row < rows; row += warps) {
    const int64_t q = row % S_q;
    const T* lr = L + row * S_k;
    const int64_t n = visible_keys(q, S_q, S_k, causal);
    float m = -INFINITY, s = 0.f;
    int64_t tail = 0;
    if (vec) {
      const int64_t nv = n / V;
      int64_t j = lane;
      for (; j + 32 * (U - 1) < nv; j += 32 * U) {
        uint4 u[U];
#pragma unroll
        for (int t = 0; t < U; ++t) u[t] = ld_nc16(lr + (j + 32 * t) * V);
#pragma unroll
        for (int t = 0; t < U; ++t) {
          float x[V];
          unpack16(u[t], x);
          float mv = x[0] * xscale;
#pragma unroll
          for (int e = 1; e < V; ++e) mv = fmaxf(mv, x[e] * xscale);
          if (mv > m) {
            s *= ex2(m - mv);
            m = mv;
          }
#pragma unroll
          for (int e = 0; e < V; ++e) s += ex2(x[e] * xscale - m);
        }
      }
      for (; j < nv; j += 32) {
        float x[V];
        unpack16(ld_nc16(lr + j * V), x);
#pragma unroll
        for (int e = 0; e < V; ++e) online_add(m, s, x[e] * xscale);
      }
      tail = nv * V;
    }
    for (int64_t c = tail + lane; c < n; c += 32) online_add(m, s, elem_to_f32(lr[c]) * xscale);
#pragma unroll
    for (int o = 16; o > 0; o >>= 1) {
      const float m2 = __shfl_xor_sync(0xffffffffu, m, o);
      const float s2 = __shfl_xor_sync(0xffffffffu, s, o);
      online_merge(m, s, m2, s2);
    }
    if (lane == 0) {
      stats[row] = make_float2(m, 1.f / s);
      if (!isfinite(m) || !(s > 0.f) || !isfinite(s)) status_or(status, RMM_NONFINITE_BIT);
    }
  }
}

// P for one 16-byte group of logits (VT elements) starting at key c: stored
// bf16 values, zero where masked, and their squares added to acc.
template <int VT>
__device__ __forceinline__ void p_group(const float (&x)[VT], int64_t c, int64_t n, float xscale, float m, float rz,
                                        float (&acc)[VT], uint32_t (&pk)[VT / 2]) {
  float p[VT];
#pragma unroll
  for (int e = 0; e < VT; ++e) p[e] = c + e < n ? ex2(fmaf(x[e], xscale, -m)) * rz : 0.f;
#pragma unroll
  for (int e = 0; e < VT / 2; ++e) {
    pk[e] = pack_bf16x2(p[2 * e], p[2 * e + 1]);
    const float lo = __uint_as_float(pk[e] << 16), hi = __uint_as_float(pk[e] & 0xFFFF0000u);
    acc[2 * e] = fmaf(lo, lo, acc[2 * e]);
    acc[2 * e + 1] = fmaf(hi, hi, acc[2 * e + 1]);
  }
}

// T: logits element. Threads: CL column lanes of VT keys (kStrip keys = one strip)
// x RL row lanes; the CTAs of a cluster split the strip's rows, and with
// s_out their partial column sums are added in rank order through
// distributed shared memory. P is bf16 [bh][S_q][S_k]; s_out[b][k] (nullable:
// P only).
template <typename T>
__global__ void __launch_bounds__(kSmThreads, 2)
softmax_score_kernel(const T* __restrict__ L, int64_t S_q, int64_t S_k, float xscale, int causal, int vec,
                     const float2* __restrict__ stats, uint16_t* __restrict__ P, const uint16_t* __restrict__ Vm,
                     int64_t d, int v_vec, float* __restrict__ s_out, uint32_t* status) {
  constexpr int VT = 16 / sizeof(T);       // logits per 16-byte load
  constexpr int CL = kStrip / VT;          // column lanes
  constexpr int RL = kSmThreads / CL;      // row lanes
  __shared__ float red[RL][kStrip + 1];
  __shared__ float part[kStrip];
  __shared__ float vsq[kStrip];
  cg::cluster_group cluster = cg::this_cluster();
  const unsigned cs = cluster.num_blocks();
  const unsigned crank = cluster.block_rank();
  const int64_t b = blockIdx.z;
  const int64_t k0 = int64_t(blockIdx.x) * kStrip;
  const int tid = threadIdx.x, rl = tid / CL, cl = tid % CL;
  const int64_t c0 = k0 + int64_t(cl) * VT;  // this thread's first key
  pdl_trigger();
  pdl_wait();
  const int64_t off = S_k - S_q;
  // rows before q_first see none of this strip's keys
  const int64_t q_first = causal ? min(S_q, k0 - off > 0 ? k0 - off : int64_t(0)) : 0;
  const T* Lb = L + b * S_q * S_k;
  uint16_t* Pb = P + b * S_q * S_k;
  const float2* st = stats + b * S_q;
  const bool full16 = vec && c0 + VT <= S_k;  // whole 16-byte logits group inside the row
  // The ring path (with its warp barriers) only when every thread of the CTA
  // has a whole 16-byte group: the choice must be the same for all lanes of a
  // warp. A partial last strip takes the scalar path in every thread.
  const bool ring_path = vec && k0 + kStrip <= S_k;

  // ||V[k, :]||^2 of the strip's keys: CTA r of the cluster takes keys r, r + cs,
  // ..., a warp per key, before its main loop so that the loads overlap it
  const int warp = tid >> 5, lane = tid & 31;
  if (s_out && Vm) {
    for (int j = int(crank) + warp * int(cs); j < kStrip; j += int(cs) * (kSmThreads / 32)) {
      const int64_t k = k0 + j;
      float a = 0.f;
      if (k < S_k) {
        const uint16_t* vr = Vm + (b * S_k + k) * d;
        if (v_vec) {
          for (int64_t c = lane; c < d / 8; c += 32) {
            float x[8];
            unpack16(ld_nc16(vr + c * 8), x);
#pragma unroll
            for (int e = 0; e < 8; ++e) a = fmaf(x[e], x[e], a);
          }
        } else {
          for (int64_t c = lane; c < d; c += 32) {
            const float x = bf16_to_f32(vr[c]);
            a = fmaf(x, x, a);
          }
        }
      }
#pragma unroll
      for (int o = 16; o > 0; o >>= 1) a += __shfl_xor_sync(0xffffffffu, a, o);
      if (lane == 0) vsq[j] = a;
    }
  }

  // zero rows: P = 0 without reading logits (this CTA's share)
  {
    const int64_t zper = (q_first + cs - 1) / cs;
    const int64_t z0 = min(q_first, int64_t(crank) * zper), z1 = min(q_first, z0 + zper);
    for (int64_t q = z0 + rl; q < z1; q += RL) {
      uint16_t* pr = Pb + q * S_k;
      if (full16) {
        if constexpr (VT == 8) {
          *reinterpret_cast<uint4*>(pr + c0) = make_uint4(0u, 0u, 0u, 0u);
        } else {
          *reinterpret_cast<uint2*>(pr + c0) = make_uint2(0u, 0u);
        }
      } else {
        for (int e = 0; e < VT; ++e)
          if (c0 + e < S_k) pr[c0 + e] = 0;
      }
    }
  }

  // computed rows: this CTA's share of [q_first, S_q), in row order per thread
  const int64_t per = (S_q - q_first + cs - 1) / cs;
  const int64_t r0 = min(S_q, q_first + int64_t(crank) * per), r1 = min(S_q, r0 + per);
  float acc[VT];
#pragma unroll
  for (int e = 0; e < VT; ++e) acc[e] = 0.f;
  if (ring_path) {
    // The logits of this thread's rows reach shared memory by cp.async into
    // its own ring slots (kRing stages of kRowUnroll rows, two stages in
    // flight): no registers are held while the loads are in flight. The
    // first column lane of each row also copies the row's statistics into a
    // slot the row's CL lanes (all in one warp) read after a warp barrier.
    extern __shared__ __align__(16) unsigned char sm_ring[];
    const uint32_t ring = smem_addr(sm_ring);
    const uint32_t srow = ring + uint32_t(kRing * kRowUnroll * kSmThreads * 16);  // [kRing][kRowUnroll][RL] float2
    const int64_t nrows = r1 - r0 > rl ? (r1 - r0 - rl + RL - 1) / RL : 0;  // rows of this thread
    const int64_t nbat_cta = ((r1 - r0 + RL - 1) / RL + kRowUnroll - 1) / kRowUnroll;  // the same in every thread
    const T* Lt = Lb + c0;
    uint16_t* Pt = Pb + c0;
    auto issue = [&](int64_t j) {
      if (j < nbat_cta) {
        const uint32_t st0 = uint32_t(j % kRing) * kRowUnroll;
#pragma unroll
        for (int t = 0; t < kRowUnroll; ++t) {
          const int64_t i = j * kRowUnroll + t;
          const int64_t qq = r0 + rl + int64_t(RL) * i;
          const bool live = i < nrows;
          cp_async_zfill16(ring + ((st0 + t) * kSmThreads + tid) * 16, live ? Lt + qq * S_k : Lt, live ? 16u : 0u);
          if (cl == 0)
            cp_async_zfill8(srow + ((st0 + t) * RL + rl) * 8, live ? st + qq : st, live ? 8u : 0u);
        }
      }
      cp_async_commit_group();  // one group per stage in every thread, empty or not
    };
    issue(0);
    issue(1);
    for (int64_t j = 0; j < nbat_cta; ++j) {
      issue(j + 2);
      cp_async_wait_group<2>();  // this thread's copies of stage j have landed
      __syncwarp();              // and the statistics its row's first lane copied
      const uint32_t st0 = uint32_t(j % kRing) * kRowUnroll;
#pragma unroll
      for (int t = 0; t < kRowUnroll; ++t) {
        const int64_t i = j * kRowUnroll + t;
        if (i < nrows) {
          const int64_t qq = r0 + rl + int64_t(RL) * i;
          uint4 u;
          float2 sv;
          asm volatile("ld.shared.v4.u32 {%0, %1, %2, %3}, [%4];"
                       : "=r"(u.x), "=r"(u.y), "=r"(u.z), "=r"(u.w)
                       : "r"(ring + ((st0 + t) * kSmThreads + tid) * 16));
          asm volatile("ld.shared.v2.f32 {%0, %1}, [%2];" : "=f"(sv.x), "=f"(sv.y) : "r"(srow + ((st0 + t) * RL + rl) * 8));
          float x[VT];
          unpack16(u, x);
          uint32_t pk[VT / 2];
          p_group<VT>(x, c0, visible_keys(qq, S_q, S_k, causal), xscale, sv.x, sv.y, acc, pk);
          if constexpr (VT == 8) {
            *reinterpret_cast<uint4*>(Pt + qq * S_k) = make_uint4(pk[0], pk[1], pk[2], pk[3]);
          } else {
            *reinterpret_cast<uint2*>(Pt + qq * S_k) = make_uint2(pk[0], pk[1]);
          }
        }
      }
      __syncwarp();  // the stage's slots are read before the next issue overwrites them
    }
    cp_async_wait_group<0>();
  } else {
    for (int64_t q = r0 + rl; q < r1; q += RL) {
      const float2 sv = st[q];
      const int64_t n = visible_keys(q, S_q, S_k, causal);
      float x[VT];
#pragma unroll
      for (int e = 0; e < VT; ++e) x[e] = c0 + e < S_k ? elem_to_f32(Lb[q * S_k + c0 + e]) : 0.f;
      uint32_t pk[VT / 2];
      p_group<VT>(x, c0, n, xscale, sv.x, sv.y, acc, pk);
      for (int e = 0; e < VT; ++e)
        if (c0 + e < S_k) Pb[q * S_k + c0 + e] = uint16_t(pk[e >> 1] >> ((e & 1) * 16));
    }
  }
  if (!s_out) return;  // (the same in every CTA of the cluster)

  // this CTA's column sums of squares: row lanes in order
#pragma unroll
  for (int e = 0; e < VT; ++e) red[rl][cl * VT + e] = acc[e];
  __syncthreads();
  if (tid < kStrip) {
    float t = 0.f;
    for (int r = 0; r < RL; ++r) t += red[r][tid];
    part[tid] = t;
  }
  cluster.sync();  // every CTA's partial sums are written and visible cluster-wide
  if (crank == 0 && tid < kStrip && k0 + tid < S_k) {
    float t = 0.f;
    for (unsigned r = 0; r < cs; ++r) t += cluster.map_shared_rank(part, r)[tid];
    float sc = sqrtf(t);
    if (Vm) sc *= sqrtf(cluster.map_shared_rank(vsq, tid % cs)[tid]);
    s_out[b * S_k + k0 + tid] = sc;
  }
  cluster.sync();  // keep shared memory alive until rank 0 has read it
}

template <typename T>
cudaError_t launch_softmax_t(const void* L, int64_t bh, int64_t S_q, int64_t S_k, float scale, int causal,
                             float2* stats, uint16_t* P, const uint16_t* V, int64_t d, float* s_out, uint32_t* status,
                             int stage, int clear_status, cudaStream_t st) {
  constexpr int VT = 16 / sizeof(T);
  const float xscale = scale * kLog2e;
  const int vec = (reinterpret_cast<uintptr_t>(L) & 15u) == 0 && (S_k % VT) == 0 &&
                  (reinterpret_cast<uintptr_t>(P) & 15u) == 0;
  if (stage == 0) {
    const int64_t rows = bh * S_q;
    const int64_t ctas = std::max<int64_t>(1, std::min<int64_t>((rows + 7) / 8, 148 * 16));
    return launch_pdl(softmax_stats_kernel<T>, dim3(unsigned(ctas)), dim3(kSmThreads), 0, st, dim3(0, 0, 0),
                      static_cast<const T*>(L), bh, S_q, S_k, xscale, causal, vec, stats, status, clear_status);
  }
  const int v_vec = V && (reinterpret_cast<uintptr_t>(V) & 15u) == 0 && d % 8 == 0;
  // CTAs per strip: split the rows until a CTA has about 512 of them
  unsigned cs = 1;
  while (cs < kSmMaxCluster && S_q >= int64_t(cs) * 2 * 512) cs *= 2;
  static std::atomic<bool> attr_done[64];  // per device; racing first calls both set the attribute
  int dev = 0;
  cudaGetDevice(&dev);
  if (dev >= 0 && dev < 64 && !attr_done[dev]) {
    cudaError_t e = cudaFuncSetAttribute(softmax_score_kernel<T>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                                         int(kScoreSmem));
    if (e != cudaSuccess) return e;
    attr_done[dev] = true;
  }
  return launch_pdl(softmax_score_kernel<T>, dim3(unsigned((S_k + kStrip - 1) / kStrip), cs, unsigned(bh)),
                    dim3(kSmThreads), kScoreSmem, st, dim3(1, cs, 1), static_cast<const T*>(L), S_q, S_k, xscale, causal, vec,
                    static_cast<const float2*>(stats), P, V, d, v_vec, s_out, status);
}

}  // namespace

cudaError_t launch_softmax_stats(const void* L, ElemKind e, int64_t bh, int64_t S_q, int64_t S_k, float scale,
                                 int causal, float* stats, uint32_t* status, int clear_status, cudaStream_t st) {
  if (bh == 0 || S_q == 0) return cudaSuccess;
  float2* s2 = reinterpret_cast<float2*>(stats);
  return e == kBF16 ? launch_softmax_t<uint16_t>(L, bh, S_q, S_k, scale, causal, s2, nullptr, nullptr, 0, nullptr,
                                                 status, 0, clear_status, st)
                    : launch_softmax_t<uint32_t>(L, bh, S_q, S_k, scale, causal, s2, nullptr, nullptr, 0, nullptr,
                                                 status, 0, clear_status, st);
}

cudaError_t launch_softmax_score(const void* L, ElemKind e, int64_t bh, int64_t S_q, int64_t S_k, float scale,
                                 int causal, const float* stats, void* P, const void* V, int64_t d, float* s_out,
                                 uint32_t* status, cudaStream_t st) {
  if (bh == 0 || S_k == 0) return cudaSuccess;
  float2* s2 = reinterpret_cast<float2*>(const_cast<float*>(stats));
  uint16_t* p = static_cast<uint16_t*>(P);
  const uint16_t* v = static_cast<const uint16_t*>(V);
  return e == kBF16 ? launch_softmax_t<uint16_t>(L, bh, S_q, S_k, scale, causal, s2, p, v, d, s_out, status, 1, 0, st)
                    : launch_softmax_t<uint32_t>(L, bh, S_q, S_k, scale, causal, s2, p, v, d, s_out, status, 1, 0, st);
}

}  // namespace rmm
