// Reduced product on the B200 tensor cores ("Mecanismo Central" on the
// gist.science summary of "Reduced Matrix Multiplication: Input-Adaptive
// Matrix-Product Reduction for LLM Inference": C = A[:, I]·B[I, :], here on
// the packed operands: A_S [M][k_pad] K-major; B either K-major B_St [N][k_pad]
// (Q·Kᵀ, where B is given as Kmat) or N-major B_S [k_pad][N], the kept rows
// of B as they are).
//
// Persistent, warp-specialised tcgen05 kernel; by default CTA pairs run 2-SM
// MMAs (cta_group::2): a pair owns a 256 x BN output tile, each CTA holds 128
// rows of A and BN/2 columns of B in shared memory and 128 x BN accumulators in
// its tensor memory, and the even (leader) CTA issues the MMAs for both.
// Per CTA:
//   warp 0      TMA producer: 128x64 A tile + (BN/CG)x64 B tile per stage into
//               a shared-memory ring (128-byte swizzle, no multicast); both
//               CTAs' loads complete on the leader's stage barrier
//   warp 1      allocates tensor memory; in the leader one lane issues
//               tcgen05.mma (kind::f16, bf16 x bf16 -> f32, K = 16) into one of
//               two TMEM accumulators and commits ring stages back to both CTAs
//   warps 2..    epilogue (4 warps, one per TMEM lane quadrant; or 8, two per
//               quadrant each taking half the columns, when a tile has at most
//               two k-blocks and the product is bound by writing C):
//               tcgen05.ld 32 lanes x 32 columns, optional bf16
//               rounding, swizzled staging in shared memory, TMA tile store
// Two accumulators let the epilogue of tile i overlap the mainloop of tile
// i+1. Tiles are visited m-fastest so a column block of B is shared through
// L2 by the pairs working on it at the same time. When the tile count leaves
// the last round less than half full, those tiles are split in two along K
// and both halves reduce-add (f32) into C, whose tiles are zeroed beforehand
// (by a small kernel, or within the fused call by spare blocks of the select
// launch, which leaves all but one SM per batch item idle).
//
// Every mbarrier wait is bounded (rmm_set_wait_limit_ns). A role whose wait
// runs out records RMM_STATUS_BIT_TIMEOUT, raises its CTA's abort flag, and
// winds down: the producer waits for its own TMA loads still in flight, the
// MMA lane waits for its issued MMAs, the epilogue waits for its TMA stores,
// and warp 1 frees tensor memory after a final CTA (and cluster) barrier. No
// thread leaves before that barrier.
#include <cudaTypedefs.h>

#include <algorithm>
#include <mutex>

#include "rmm_device.cuh"
#include "rmm_internal.h"

namespace rmm {
namespace {

constexpr int BM = 128;  // rows of A per CTA
constexpr int BK = 64;   // 64 bf16 = one 128-byte swizzle row
constexpr int kUmmaK = 16;
// Epilogue warps EW: 4, one per TMEM lane quadrant; or 8 (two per quadrant,
// each taking half of the tile's columns) for write-bound products with few
// k-blocks per tile, at the cost of one ring stage.
template <int BN, int CG, int EW = 4>
struct TcCfg {
  static constexpr int THREADS = 64 + 32 * EW;
  static constexpr int BN_CTA = BN / CG;  // columns of B held by one CTA
  static constexpr uint32_t A_BYTES = BM * BK * 2;
  static constexpr uint32_t B_BYTES = BN_CTA * BK * 2;
  static constexpr uint32_t STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES = int(((EW == 8 ? 160u : 192u) * 1024u) / STAGE_BYTES);
  static constexpr uint32_t EPI_BUF = 32 * 128;  // 32 rows x 128 bytes
  static constexpr uint32_t EPI_BYTES = EW * 2 * EPI_BUF;
  static constexpr uint32_t TMEM_COLS = 2 * BN;
  static constexpr uint32_t BAR_BYTES = 256;
  static constexpr size_t SMEM = 1024 + size_t(STAGES) * STAGE_BYTES + EPI_BYTES + BAR_BYTES;
};
static_assert(TcCfg<256, 1>::SMEM <= 232448 && TcCfg<128, 1>::SMEM <= 232448, "shared memory budget");
static_assert(TcCfg<256, 2>::SMEM <= 232448 && TcCfg<128, 2>::SMEM <= 232448, "shared memory budget");
static_assert(TcCfg<256, 2, 8>::SMEM <= 232448 && TcCfg<128, 2, 8>::SMEM <= 232448, "shared memory budget");
static_assert(TcCfg<128, 2>::STAGES * 2 + 6 <= 32, "barrier area");

struct TcParams {
  int32_t M, N, num_kb, tiles_m, tiles_n;
  int64_t total_tiles;
  // Work units: units [0, full_units) are whole tiles; when the last round
  // would leave pairs idle, its tiles are split at k-block kb_mid into two
  // units each (same tile, two halves of K) that add into a zeroed C.
  int64_t full_units, total_units;
  int32_t kb_mid;
  int64_t causal_off;  // >= 0: A[i][k] = 0 for k > i + causal_off; -1: dense
  int32_t cg2;         // 1: 2-SM tiles (BM·2 rows)
  uint32_t* status;
  uint64_t wait_limit_ns;
  int stall_producer;
  int tma_store;  // 1: TMA tile stores; 0: bounds-checked direct stores
  int out_bf16;
  void* c;
  int64_t ldc, strideC;
};

// Tile t -> (batch item, m block of BM*CG rows, n block of BN columns), m fastest.
__device__ __forceinline__ void decode_tile(int64_t t, const TcParams& p, int32_t& b, int32_t& mb, int32_t& nb) {
  const int64_t per = int64_t(p.tiles_m) * p.tiles_n;
  b = int32_t(t / per);
  const int64_t r = t - int64_t(b) * per;
  nb = int32_t(r / p.tiles_m);
  mb = int32_t(r - int64_t(nb) * p.tiles_m);
}

struct Unit {
  int64_t tile;
  int32_t kb0, kb1;
  bool split;
};

__device__ __forceinline__ Unit unit_info(int64_t u, const TcParams& p) {
  Unit w;
  if (u < p.full_units) {
    w.tile = u;
    w.kb0 = 0;
    w.kb1 = p.num_kb;
    w.split = false;
    if (p.causal_off >= 0) {  // the tile's last row sees keys up to that row + causal_off
      int32_t b, mb, nb;
      decode_tile(u, p, b, mb, nb);
      const int64_t last_row = min(int64_t(p.M), int64_t(mb + 1) * BM * (p.cg2 ? 2 : 1)) - 1;
      const int64_t kb_end = (last_row + p.causal_off) / BK + 1;
      if (kb_end < w.kb1) w.kb1 = int32_t(kb_end);
    }
  } else {
    const int64_t j = u - p.full_units;
    w.tile = p.full_units + (j >> 1);
    const bool second = (j & 1) != 0;
    w.kb0 = second ? p.kb_mid : 0;
    w.kb1 = second ? p.num_kb : p.kb_mid;
    w.split = true;
  }
  return w;
}

__device__ __forceinline__ void raise_abort(volatile int* abort_flag, uint32_t* status) {
  *abort_flag = 1;
  status_or(status, RMM_TIMEOUT_BIT);
}

template <int BN, bool BMN, int CG, int EW>
__global__ void __launch_bounds__(TcCfg<BN, CG, EW>::THREADS, 1)
gemm_tc_kernel(const __grid_constant__ CUtensorMap tmA, const __grid_constant__ CUtensorMap tmB,
               const __grid_constant__ CUtensorMap tmC, const TcParams p) {
  using Cfg = TcCfg<BN, CG, EW>;
  constexpr int STAGES = Cfg::STAGES;
  constexpr int BN_CTA = Cfg::BN_CTA;
  extern __shared__ uint8_t tc_smem_raw[];
  uint8_t* smem = reinterpret_cast<uint8_t*>((reinterpret_cast<uintptr_t>(tc_smem_raw) + 1023) & ~uintptr_t(1023));
  uint8_t* sA = smem;
  uint8_t* sB = sA + STAGES * Cfg::A_BYTES;
  uint8_t* sEpi = sB + STAGES * Cfg::B_BYTES;
  uint64_t* full = reinterpret_cast<uint64_t*>(sEpi + Cfg::EPI_BYTES);
  uint64_t* empty = full + STAGES;
  uint64_t* tfull = empty + STAGES;   // [2] accumulator ready for the epilogue
  uint64_t* tempty = tfull + 2;       // [2] accumulator drained by the epilogue(s)
  uint64_t* drain = tempty + 2;       // MMA completion at wind-down
  uint32_t* tmem_base_sh = reinterpret_cast<uint32_t*>(drain + 1);
  int* abort_sh = reinterpret_cast<int*>(tmem_base_sh + 1);
  int* never_sh = abort_sh + 1;       // stays 0: waits that must not be cut short

  const int warp = threadIdx.x >> 5;
  const int lane = threadIdx.x & 31;
  const uint32_t rank = CG == 2 ? cluster_ctarank() : 0u;  // 0 = leader
  const int64_t pair = blockIdx.x / CG;
  const int64_t npairs = gridDim.x / CG;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(&full[s], 1);
      mbar_init(&empty[s], 1);
    }
    for (int a = 0; a < 2; ++a) {
      mbar_init(&tfull[a], 1);
      mbar_init(&tempty[a], EW * CG);
    }
    mbar_init(drain, 1);
    *abort_sh = 0;
    *never_sh = 0;
    fence_mbar_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_desc(&tmA);
    tma_prefetch_desc(&tmB);
    if (p.tma_store) tma_prefetch_desc(&tmC);
  }
  if (warp == 1) {
    tmem_alloc<CG>(tmem_base_sh, Cfg::TMEM_COLS);
    tmem_relinquish<CG>();
  }
  pdl_trigger();
  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();  // the peer's barriers exist before anyone signals them
  tc_fence_after();
  const uint32_t tmem_base = *tmem_base_sh;
  pdl_wait();  // set-up above overlaps the previous kernel's tail
  volatile int* abort_v = abort_sh;
  const volatile int* never_v = never_sh;
  const uint64_t limit = p.wait_limit_ns;
  const uint32_t peer = rank ^ 1u;

  if (warp == 0) {
    // ------------------------------------------------------------ TMA producer (one lane)
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      uint32_t issued = 0;      // bit s: this CTA loaded stage s
      uint32_t issued_par = 0;  // bit s: parity of that stage's last phase
      bool ok = true;
      for (int64_t u = pair; ok && u < p.total_units; u += npairs) {
        const Unit w = unit_info(u, p);
        int32_t b, mb, nb;
        decode_tile(w.tile, p, b, mb, nb);
        const int32_t m_row = mb * BM * CG + int32_t(rank) * BM;
        const int32_t n_col = nb * BN + int32_t(rank) * BN_CTA;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait_bounded(&empty[stage], phase ^ 1u, limit, abort_v)) {
            ok = false;
            break;
          }
          if (!p.stall_producer) {
            uint8_t* a_dst = sA + stage * Cfg::A_BYTES;
            uint8_t* b_dst = sB + stage * Cfg::B_BYTES;
            if constexpr (CG == 1) {
              mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES);
              tma_load_3d(a_dst, &tmA, &full[stage], kb * BK, m_row, b);
              if constexpr (BMN) {
#pragma unroll
                for (int j = 0; j < BN_CTA / 64; ++j)
                  tma_load_3d(b_dst + j * 8192, &tmB, &full[stage], n_col + j * 64, kb * BK, b);
              } else {
                tma_load_3d(b_dst, &tmB, &full[stage], kb * BK, n_col, b);
              }
            } else {
              // both CTAs' bytes complete on the leader's barrier; the leader arms it
              if (rank == 0) mbar_arrive_expect_tx(&full[stage], Cfg::STAGE_BYTES * CG);
              const uint32_t bar = mapa_shared(smem_addr(&full[stage]), 0);
              tma_load_3d_pair(a_dst, &tmA, bar, kb * BK, m_row, b);
              if constexpr (BMN) {
#pragma unroll
                for (int j = 0; j < BN_CTA / 64; ++j)
                  tma_load_3d_pair(b_dst + j * 8192, &tmB, bar, n_col + j * 64, kb * BK, b);
              } else {
                tma_load_3d_pair(b_dst, &tmB, bar, kb * BK, n_col, b);
              }
            }
            issued |= 1u << stage;
            issued_par = (issued_par & ~(1u << stage)) | (phase << stage);
          }
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      if (!ok) raise_abort(abort_v, p.status);
      // Loads complete on their own; make sure none is still writing shared
      // memory when the CTA exits. The leader waits on its stage barriers
      // (which also count the peer's bytes); the peer's loads land on the
      // leader's barriers, so on an abort it gives them time to land.
      if (CG == 1 || rank == 0) {
        for (int s = 0; s < STAGES; ++s)
          if (issued & (1u << s)) mbar_wait_bounded(&full[s], (issued_par >> s) & 1u, limit, never_v);
      } else if (!ok && issued) {
        const uint64_t t0 = globaltimer_ns();
        while (globaltimer_ns() - t0 < 200000ull) __nanosleep(1000);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    // ------------------------------------------------------------ MMA issuer (one lane of the leader)
    if (rank == 0 && lane == 0) {
      constexpr uint32_t idesc = umma_idesc_bf16_f32(BM * CG, BN, BMN);
      uint32_t stage = 0, phase = 0;
      uint32_t acc = 0, acc_phase = 0;
      bool ok = true;
      for (int64_t u = pair; ok && u < p.total_units; u += npairs) {
        const Unit w = unit_info(u, p);
        if (!mbar_wait_bounded(&tempty[acc], acc_phase ^ 1u, limit, abort_v)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + acc * BN;
        for (int kb = w.kb0; kb < w.kb1; ++kb) {
          if (!mbar_wait_bounded(&full[stage], phase, limit, abort_v)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t a0 = smem_addr(sA + stage * Cfg::A_BYTES);
          const uint32_t b0 = smem_addr(sB + stage * Cfg::B_BYTES);
#pragma unroll
          for (int kk = 0; kk < BK / kUmmaK; ++kk) {
            // K-major: 16 elements = 32 bytes along the swizzled row;
            // N-major: 16 K-rows of 128 bytes
            const uint64_t bdesc = BMN ? umma_desc_mn_sw128(b0 + kk * 2048, 8192) : umma_desc_k_sw128(b0 + kk * 32);
            umma_bf16<CG>(d_tmem, umma_desc_k_sw128(a0 + kk * 32), bdesc, idesc, (kb > w.kb0) || kk != 0);
          }
          // this stage's smem is free in both CTAs once these MMAs are done
          umma_commit<CG>(smem_addr(&empty[stage]));
          if constexpr (CG == 2) umma_commit<CG>(mapa_shared(smem_addr(&empty[stage]), peer));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        umma_commit<CG>(smem_addr(&tfull[acc]));
        if constexpr (CG == 2) umma_commit<CG>(mapa_shared(smem_addr(&tfull[acc]), peer));
        acc ^= 1u;
        if (acc == 0) acc_phase ^= 1u;
      }
      if (!ok) raise_abort(abort_v, p.status);
      // Wait for every MMA this lane issued before tensor memory is freed.
      umma_commit<CG>(smem_addr(drain));
      mbar_wait_bounded(drain, 0, limit, never_v);
    }
    __syncwarp();
  } else {
    // ------------------------------------------------------------ epilogue
    const int q = warp & 3;  // TMEM lane quadrant this warp may access
    uint8_t* bufs = sEpi + (warp - 2) * 2 * Cfg::EPI_BUF;
    uint32_t acc = 0, acc_phase = 0, nbuf = 0;
    bool ok = true;
    const int cols_per_chunk = p.out_bf16 ? 64 : 32;
    const int chunks = BN / cols_per_chunk;
    // this warp's chunks: all of them, or one half with two warps per quadrant
    const int c_begin = EW == 8 ? ((warp - 2) >> 2) * (chunks / 2) : 0;
    const int c_end = EW == 8 ? c_begin + chunks / 2 : chunks;
    for (int64_t u = pair; ok && u < p.total_units; u += npairs) {
      const Unit unit = unit_info(u, p);
      int32_t b, mb, nb;
      decode_tile(unit.tile, p, b, mb, nb);
      int w = 1;
      if (lane == 0) w = mbar_wait_bounded(&tfull[acc], acc_phase, limit, abort_v);
      w = __shfl_sync(0xffffffffu, w, 0);
      if (!w) {
        ok = false;
        break;
      }
      tc_fence_after();
      const uint32_t t_row = tmem_base + (uint32_t(q * 32) << 16) + acc * BN;
      const int32_t row0 = mb * BM * CG + int32_t(rank) * BM + q * 32;
      // Store chunk c (32 rows x cols_per_chunk columns, `packed` holding its 32
      // words per lane) through the staging buffers, or directly.
      auto store_chunk = [&](int c, const uint32_t (&packed)[32]) {
        const int32_t col0 = nb * BN + c * cols_per_chunk;
        if (p.tma_store) {
          uint8_t* buf = bufs + nbuf * Cfg::EPI_BUF;
          if (lane == 0) tma_store_wait_read<1>();  // the store that last read `buf` is done
          __syncwarp();
          // row `lane` of the 32x128-byte box, 16-byte chunks in 128-byte swizzle order
#pragma unroll
          for (int j = 0; j < 8; ++j) {
            *reinterpret_cast<uint4*>(buf + lane * 128 + ((j ^ (lane & 7)) << 4)) =
                make_uint4(packed[4 * j], packed[4 * j + 1], packed[4 * j + 2], packed[4 * j + 3]);
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            if (unit.split)
              tma_reduce_add_3d(&tmC, buf, col0, row0, b);  // the tile's other K half adds too
            else
              tma_store_3d(&tmC, buf, col0, row0, b);
            tma_store_commit();
          }
          __syncwarp();
          nbuf ^= 1u;
        } else {
          const int64_t row = int64_t(row0) + lane;
          if (row < p.M) {
            if (p.out_bf16) {
              uint16_t* cp = static_cast<uint16_t*>(p.c) + int64_t(b) * p.strideC + row * p.ldc;
              for (int j = 0; j < 64; ++j) {
                const int64_t col = int64_t(col0) + j;
                if (col < p.N) cp[col] = uint16_t(packed[j >> 1] >> ((j & 1) * 16));
              }
            } else {
              float* cp = static_cast<float*>(p.c) + int64_t(b) * p.strideC + row * p.ldc;
              for (int j = 0; j < 32; ++j) {
                const int64_t col = int64_t(col0) + j;
                if (col < p.N) cp[col] = __uint_as_float(packed[j]);
              }
            }
          }
        }
      };
      if constexpr (EW == 8) {
        // This warp's whole share of the tile (BN / 2 columns) is read from
        // TMEM at once, and the accumulator is handed back before any store:
        // one TMEM round trip per tile instead of one per chunk.
        constexpr int NLD = BN / 64;  // 32-column loads
        uint32_t r[NLD][32];
        const uint32_t col_base = uint32_t(c_begin * cols_per_chunk);
#pragma unroll
        for (int l = 0; l < NLD; ++l) tmem_ld_32x32b_x32(t_row + col_base + 32 * l, r[l]);
        tmem_ld_wait();
        tc_fence_before();
        __syncwarp();
        if (lane == 0) {
          if (CG == 1 || rank == 0)
            mbar_arrive(&tempty[acc]);
          else
            mbar_arrive_cluster(mapa_shared(smem_addr(&tempty[acc]), 0));
        }
        if (p.out_bf16) {
#pragma unroll
          for (int i = 0; i < NLD / 2; ++i) {
            uint32_t packed[32];
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              packed[j] = pack_bf16x2(__uint_as_float(r[2 * i][2 * j]), __uint_as_float(r[2 * i][2 * j + 1]));
              packed[16 + j] =
                  pack_bf16x2(__uint_as_float(r[2 * i + 1][2 * j]), __uint_as_float(r[2 * i + 1][2 * j + 1]));
            }
            store_chunk(c_begin + i, packed);
          }
        } else {
#pragma unroll
          for (int i = 0; i < NLD; ++i) store_chunk(c_begin + i, r[i]);
        }
      } else {
        for (int c = c_begin; c < c_end; ++c) {
          uint32_t packed[32];
          if (p.out_bf16) {
            uint32_t r0[32], r1[32];
            tmem_ld_32x32b_x32(t_row + c * 64, r0);
            tmem_ld_32x32b_x32(t_row + c * 64 + 32, r1);
            tmem_ld_wait();
#pragma unroll
            for (int j = 0; j < 16; ++j) {
              packed[j] = pack_bf16x2(__uint_as_float(r0[2 * j]), __uint_as_float(r0[2 * j + 1]));
              packed[16 + j] = pack_bf16x2(__uint_as_float(r1[2 * j]), __uint_as_float(r1[2 * j + 1]));
            }
          } else {
            tmem_ld_32x32b_x32(t_row + c * 32, packed);
            tmem_ld_wait();
          }
          if (c == c_end - 1) {
            // this warp's part of the accumulator read: hand it back to the leader's MMA lane
            tc_fence_before();
            __syncwarp();
            if (lane == 0) {
              if (CG == 1 || rank == 0)
                mbar_arrive(&tempty[acc]);
              else
                mbar_arrive_cluster(mapa_shared(smem_addr(&tempty[acc]), 0));
            }
          }
          store_chunk(c, packed);
        }
      }
      acc ^= 1u;
      if (acc == 0) acc_phase ^= 1u;
    }
    if (!ok && lane == 0) raise_abort(abort_v, p.status);
    if (lane == 0) tma_store_wait_all();
    __syncwarp();
  }

  tc_fence_before();
  __syncthreads();
  if constexpr (CG == 2) cluster_sync_all();  // the pair is done with each other's barriers and TMEM
  tc_fence_after();
  if (warp == 1) tmem_dealloc<CG>(tmem_base, Cfg::TMEM_COLS);
}

// Zero the f32 C tiles that the split-K round reduce-adds into. Waits for its
// predecessor first: C may still be written by earlier work on the stream, and
// the GEMM launched after this kernel relies on it having waited.
__global__ void __launch_bounds__(256) zero_split_tiles_kernel(const SplitZero z) {
  pdl_trigger();
  pdl_wait();
  zero_split_tiles(z, blockIdx.x, gridDim.x, threadIdx.x, 256);
}

// ------------------------------------------------------------------ host side
PFN_cuTensorMapEncodeTiled_v12000 tensor_map_encoder() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(f);
  });
  return fn;
}

bool encode_3d(CUtensorMap* m, CUtensorMapDataType dt, const void* base, uint64_t d0, uint64_t d1, uint64_t d2,
               uint64_t stride1_bytes, uint64_t stride2_bytes, uint32_t box0, uint32_t box1) {
  auto enc = tensor_map_encoder();
  if (!enc) return false;
  cuuint64_t dims[3] = {d0, d1, d2};
  cuuint64_t strides[2] = {stride1_bytes, stride2_bytes};
  cuuint32_t box[3] = {box0, box1, 1};
  cuuint32_t estr[3] = {1, 1, 1};
  CUresult r = enc(m, dt, 3, const_cast<void*>(base), dims, strides, box, estr, CU_TENSOR_MAP_INTERLEAVE_NONE,
                   CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B, CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  return r == CUDA_SUCCESS;
}

struct DevInfo {
  int sms = 0;
  int cc_major = 0, cc_minor = 0;
  bool attr_done = false;
};

template <int BN, bool BMN, int CG, int EW = 4>
void set_attr() {
  cudaFuncSetAttribute(gemm_tc_kernel<BN, BMN, CG, EW>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                       int(TcCfg<BN, CG, EW>::SMEM));
}

DevInfo& dev_info(int dev) {
  static DevInfo info[64];
  static std::mutex mu;
  std::lock_guard<std::mutex> lock(mu);
  DevInfo& d = info[dev & 63];
  if (!d.attr_done) {
    cudaDeviceGetAttribute(&d.sms, cudaDevAttrMultiProcessorCount, dev);
    cudaDeviceGetAttribute(&d.cc_major, cudaDevAttrComputeCapabilityMajor, dev);
    cudaDeviceGetAttribute(&d.cc_minor, cudaDevAttrComputeCapabilityMinor, dev);
    if (d.cc_major == 10 && d.cc_minor == 0) {
      set_attr<256, false, 1>();
      set_attr<128, false, 1>();
      set_attr<256, true, 1>();
      set_attr<128, true, 1>();
      set_attr<256, false, 2>();
      set_attr<128, false, 2>();
      set_attr<256, true, 2>();
      set_attr<128, true, 2>();
      set_attr<256, false, 2, 8>();
      set_attr<128, false, 2, 8>();
      set_attr<256, true, 2, 8>();
      set_attr<128, true, 2, 8>();
    }
    d.attr_done = true;
  }
  return d;
}

// C through TMA tile stores: rows 16-byte aligned and a tensor map that encodes.
bool encode_c(const GemmArgs& g, CUtensorMap* tmC) {
  const uint64_t eb = g.out == kBF16 ? 2 : 4;
  const bool c_ok = (reinterpret_cast<uintptr_t>(g.c) & 15u) == 0 && (uint64_t(g.ldc) * eb) % 16 == 0 &&
                    (g.batch == 1 || (uint64_t(g.strideC) * eb) % 16 == 0);
  if (!c_ok) return false;
  const uint64_t s2 = g.batch == 1 ? uint64_t(g.ldc) * eb * uint64_t(g.M) : uint64_t(g.strideC) * eb;
  return encode_3d(tmC, g.out == kBF16 ? CU_TENSOR_MAP_DATA_TYPE_BFLOAT16 : CU_TENSOR_MAP_DATA_TYPE_FLOAT32, g.c,
                   uint64_t(g.N), uint64_t(g.M), uint64_t(g.batch), uint64_t(g.ldc) * eb, s2 == 0 ? 16 : s2,
                   uint32_t(128 / eb), 32);
}

// Tile grid and K split of one launch. Tiles are visited m-fastest; the pairs
// (units) take them round-robin. When the last round would leave more than
// half the pairs idle, its tiles are split along K into two halves that
// reduce-add (f32, TMA) into C zeroed beforehand; with C zero, a + b == b + a
// keeps the result independent of which half lands first.
struct Plan {
  int32_t tiles_m, tiles_n, num_kb, bn, bm;
  int64_t total_tiles, units, rem;
  bool split;
};

Plan make_plan(const GemmArgs& g, int sms, bool c_tma) {
  Plan q;
  const int cg = g.cta_group == 1 ? 1 : 2;
  q.bn = g.N <= 128 ? 128 : 256;
  q.bm = BM * cg;
  q.tiles_m = int32_t((g.M + q.bm - 1) / q.bm);
  q.tiles_n = int32_t((g.N + q.bn - 1) / q.bn);
  q.num_kb = int32_t((g.k_pad + BK - 1) / BK);
  q.total_tiles = int64_t(q.tiles_m) * q.tiles_n * g.batch;
  q.units = std::max<int64_t>(1, (sms > 0 ? sms : 148) / cg);
  q.rem = q.total_tiles % q.units;
  q.split = g.out == kF32 && c_tma && q.num_kb >= 2 && q.rem > 0 && 2 * q.rem <= q.units && g.causal_off < 0;
  return q;
}

SplitZero split_zero(const GemmArgs& g, const Plan& q) {
  SplitZero z;
  z.c = static_cast<float*>(g.c);
  z.ldc = g.ldc;
  z.strideC = g.batch == 1 ? 0 : g.strideC;
  z.M = g.M;
  z.N = g.N;
  z.first_tile = q.total_tiles - q.rem;
  z.count = q.split ? q.rem : 0;
  z.tiles_m = q.tiles_m;
  z.tiles_n = q.tiles_n;
  z.tile_rows = q.bm;
  z.tile_cols = q.bn;
  return z;
}

template <int BN, bool BMN, int CG, int EW>
cudaError_t launch_cfg(const GemmArgs& g, const DevInfo& di, cudaStream_t st, const char** why) {
  using Cfg = TcCfg<BN, CG, EW>;
  const uint64_t kp = uint64_t(g.k_pad);
  CUtensorMap tmA, tmB, tmC;
  // a batch of one takes any batch stride (TMA needs a nonzero multiple of 16 bytes)
  const uint64_t sA = g.batch == 1 ? uint64_t(g.lda) * 2 * uint64_t(g.M) : uint64_t(g.strideA) * 2;
  bool ok = encode_3d(&tmA, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.a, kp, uint64_t(g.M), uint64_t(g.batch),
                      uint64_t(g.lda) * 2, sA == 0 ? 16 : sA, BK, BM);
  if (BMN) {
    const uint64_t ldb = uint64_t(g.ldb);
    ok = ok && encode_3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.b, uint64_t(g.N), kp, uint64_t(g.batch), ldb * 2,
                         ldb * 2 * kp, 64, BK);
  } else {
    ok = ok && encode_3d(&tmB, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, g.b, kp, uint64_t(g.N), uint64_t(g.batch), kp * 2,
                         kp * 2 * uint64_t(g.N), BK, Cfg::BN_CTA);
  }
  if (!ok) {
    *why = "cuTensorMapEncodeTiled failed for a packed operand";
    return cudaErrorInvalidValue;
  }
  const int tma_store = encode_c(g, &tmC) ? 1 : 0;
  if (!tma_store) tmC = tmA;  // never dereferenced when tma_store == 0
  const Plan q = make_plan(g, di.sms, tma_store != 0);
  if (q.bn != BN || q.bm != BM * CG) {
    *why = "internal: tile plan does not match the launched configuration";
    return cudaErrorInvalidValue;
  }

  TcParams p;
  p.M = int32_t(g.M);
  p.N = int32_t(g.N);
  p.num_kb = q.num_kb;
  p.tiles_m = q.tiles_m;
  p.tiles_n = q.tiles_n;
  p.total_tiles = q.total_tiles;
  p.status = g.status;
  p.wait_limit_ns = g.wait_limit_ns;
  p.stall_producer = g.stall_producer;
  p.tma_store = tma_store;
  p.out_bf16 = g.out == kBF16;
  p.c = g.c;
  p.ldc = g.ldc;
  p.strideC = g.strideC;
  const int64_t units = q.units;
  p.full_units = q.split ? p.total_tiles - q.rem : p.total_tiles;
  p.total_units = q.split ? p.full_units + 2 * q.rem : p.total_tiles;
  p.kb_mid = p.num_kb / 2;
  p.causal_off = g.causal_off;
  p.cg2 = CG == 2 ? 1 : 0;
  if (q.split && !g.c_zeroed) {
    const SplitZero z = split_zero(g, q);
    cudaError_t e = launch_pdl(zero_split_tiles_kernel, dim3(unsigned(std::min<int64_t>(z.count * 8, 1184))),
                               dim3(256), 0, st, dim3(0, 0, 0), z);
    if (e != cudaSuccess) return e;
  }
  const int64_t grid = CG * std::min<int64_t>(p.total_units, units);
  if (g.ev_start) {
    cudaError_t e = cudaEventRecord(g.ev_start, st);
    if (e != cudaSuccess) return e;
  }
  cudaError_t e = launch_pdl(gemm_tc_kernel<BN, BMN, CG, EW>, dim3(unsigned(grid)), dim3(Cfg::THREADS), Cfg::SMEM, st,
                             CG == 2 ? dim3(2, 1, 1) : dim3(0, 0, 0), tmA, tmB, tmC, p);
  if (e == cudaSuccess && g.ev_stop) e = cudaEventRecord(g.ev_stop, st);
  return e;
}

template <int CG, int EW>
cudaError_t launch_cg_ew(const GemmArgs& g, const DevInfo& di, cudaStream_t st, const char** why) {
  if (g.b_kmajor)
    return g.N <= 128 ? launch_cfg<128, false, CG, EW>(g, di, st, why) : launch_cfg<256, false, CG, EW>(g, di, st, why);
  return g.N <= 128 ? launch_cfg<128, true, CG, EW>(g, di, st, why) : launch_cfg<256, true, CG, EW>(g, di, st, why);
}

// With at most two k-blocks per tile the product is bound by writing C: the
// 2-SM kernels then run 8 epilogue warps.
template <int CG>
cudaError_t launch_cg(const GemmArgs& g, const DevInfo& di, cudaStream_t st, const char** why) {
  if constexpr (CG == 2) {
    if (g.k_pad <= 2 * BK) return launch_cg_ew<2, 8>(g, di, st, why);
  }
  return launch_cg_ew<CG, 4>(g, di, st, why);
}

}  // namespace

bool gemm_tc_split_zero(const GemmArgs& g, SplitZero* z) {
  if (g.batch == 0 || g.M == 0 || g.N == 0) return false;
  int dev = 0;
  if (cudaGetDevice(&dev) != cudaSuccess) return false;
  const DevInfo& di = dev_info(dev);
  CUtensorMap tmC;
  const Plan q = make_plan(g, di.sms, encode_c(g, &tmC));
  if (!q.split) return false;
  *z = split_zero(g, q);
  return true;
}

cudaError_t launch_gemm_tc(const GemmArgs& g, cudaStream_t st, const char** why) {
  if (g.batch == 0 || g.M == 0 || g.N == 0) return cudaSuccess;
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return e;
  const DevInfo& di = dev_info(dev);
  if (!(di.cc_major == 10 && di.cc_minor == 0)) {
    *why = "the tensor-core GEMM is built for sm_100a (B200) only";
    return cudaErrorNoKernelImageForDevice;
  }
  if ((reinterpret_cast<uintptr_t>(g.a) & 15u) || (reinterpret_cast<uintptr_t>(g.b) & 15u)) {
    *why = "the operands must be 16-byte aligned";
    return cudaErrorInvalidValue;
  }
  if ((uint64_t(g.lda) * 2) % 16 != 0 || (g.batch > 1 && (uint64_t(g.strideA) * 2) % 16 != 0)) {
    *why = "A's row pitch and batch stride must be multiples of 8 elements";
    return cudaErrorInvalidValue;
  }
  if (g.M > INT32_MAX || g.N > INT32_MAX || g.k_pad > INT32_MAX || g.batch > INT32_MAX) {
    *why = "a dimension exceeds 2^31-1";
    return cudaErrorInvalidValue;
  }
  if (!g.b_kmajor && (uint64_t(g.ldb) * 2) % 16 != 0) {
    *why = "the packed N-major B operand needs a row pitch that is a multiple of 8 elements";
    return cudaErrorInvalidValue;
  }
  return g.cta_group == 1 ? launch_cg<1>(g, di, st, why) : launch_cg<2>(g, di, st, why);
}

}  // namespace rmm
