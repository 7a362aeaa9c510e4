// rmm_matmul_reduced_noalloc: the fused reduced product for callers that may
// not allocate device memory at all, e.g. code running inside another
// framework's memory pool or allocator hooks, plugins handed only input and
// output buffers, or a process whose device heap is fully reserved up front.
//
// Its scratch space (status word, scores, kept indices, packed operands) lives
// in one file-scope device array of fixed size instead of a caller-supplied
// workspace. The caller still passes A, B, C (and optionally idx_out and a
// status word); this file calls no cudaMalloc, cudaFree or any allocating
// routine.
#include <atomic>
#include <cstdio>
#include <mutex>

#include "../../include/rmm.h"
#include "rmm_internal.h"

namespace {

// Largest workspace (rmm_workspace_size) a call may need.
constexpr size_t kScratchBytes = size_t(32) << 20;

// The fused pipeline wants a 1 KiB-aligned workspace; the extra KiB lets the
// aligned window of kScratchBytes always fit.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kScratchBytes + 1024];

constexpr int kMaxDevices = 64;
// Device address of g_noalloc_scratch per device, once a lookup succeeded.
// A failed lookup is not cached: the next call on that device tries again.
std::atomic<void*> g_scratch_base[kMaxDevices];
std::mutex g_scratch_mu;

// The scratch array's device address on the current device `dev`.
cudaError_t scratch_base(int dev, void** base) {
  void* p = g_scratch_base[dev].load(std::memory_order_acquire);
  if (p == nullptr) {
    std::lock_guard<std::mutex> lock(g_scratch_mu);
    p = g_scratch_base[dev].load(std::memory_order_relaxed);
    if (p == nullptr) {
      const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
      if (e != cudaSuccess || p == nullptr) return e != cudaSuccess ? e : cudaErrorInvalidSymbol;
      g_scratch_base[dev].store(p, std::memory_order_release);
    }
  }
  *base = p;
  return cudaSuccess;
}

}  // namespace

extern "C" rmm_status rmm_matmul_reduced_noalloc(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t M,
                                                 int64_t K, int64_t N, double rho, rmm_dtype in, rmm_score_mode mode,
                                                 void* C, int64_t ldc, rmm_dtype out, int32_t* idx_out,
                                                 uint32_t* status_word, cudaStream_t stream) {
  char msg[256];
  const int64_t k = rmm_keep_count(rho, K);
  if (k >= 1) {
    const size_t need = rmm_workspace_size_for(1, M, K, N, k, in, 0);
    if (need > kScratchBytes) {
      snprintf(msg, sizeof(msg),
               "rmm_matmul_reduced_noalloc: this product needs %zu bytes of scratch, the static scratch holds "
               "%zu; call rmm_matmul_reduced with a workspace instead",
               need, kScratchBytes);
      rmm::set_last_error(msg);
      return RMM_ERR_INVALID;
    }
  }
  // Look up this device's scratch address with the stream's device current;
  // the caller's current device is restored when the call returns.
  rmm::DeviceGuard guard;
  cudaError_t e = guard.bind(stream);
  int dev = -1;
  if (e == cudaSuccess) e = cudaGetDevice(&dev);
  if (e == cudaSuccess && (dev < 0 || dev >= kMaxDevices)) e = cudaErrorInvalidDevice;
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "rmm_matmul_reduced_noalloc: selecting the stream's device: %s",
             cudaGetErrorString(e));
    rmm::set_last_error(msg);
    return RMM_ERR_CUDA;
  }
  void* base = nullptr;
  e = scratch_base(dev, &base);
  if (e != cudaSuccess) {
    snprintf(msg, sizeof(msg), "rmm_matmul_reduced_noalloc: cudaGetSymbolAddress: %s", cudaGetErrorString(e));
    rmm::set_last_error(msg);
    return RMM_ERR_CUDA;
  }
  void* ws = reinterpret_cast<void*>((reinterpret_cast<uintptr_t>(base) + 1023) & ~uintptr_t(1023));
  // The fused call clears the status word at the head of the scratch, then
  // validates every argument before it launches anything.
  rmm_status st = rmm_matmul_reduced(A, lda, B, ldb, M, K, N, rho, in, mode, C, ldc, out, idx_out, ws,
                                     kScratchBytes, stream);
  if (st == RMM_OK && status_word != nullptr) {
    e = cudaMemcpyAsync(status_word, ws, sizeof(uint32_t), cudaMemcpyDeviceToDevice, stream);
    if (e != cudaSuccess) {
      snprintf(msg, sizeof(msg), "rmm_matmul_reduced_noalloc: copying the status word: %s", cudaGetErrorString(e));
      rmm::set_last_error(msg);
      return RMM_ERR_CUDA;
    }
  }
  return st;
}
