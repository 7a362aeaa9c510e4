// The librmm C ABI: argument validation, workspace layout and the
// score -> select -> pack -> gemm pipeline of Reduced Matrix Multiplication
// (gist.science summary of "Reduced Matrix Multiplication: Input-Adaptive
// Matrix-Product Reduction for LLM Inference", Resumo Técnico › Metodologia).
// Everything is enqueued on the caller's stream; nothing here allocates or
// synchronises, except rmm_check.
#include <algorithm>
#include <atomic>
#include <cmath>
#include <cstdlib>
#include <cstdarg>
#include <cstdio>
#include <cstring>

#include <nvtx3/nvToolsExt.h>

#include "../../include/rmm.h"
#include "rmm_internal.h"

namespace rmm {

// A named NVTX range around one stage of a call, so that a profiler's
// timeline (or an ncu --nvtx filter) shows score, select, pack and the product
// by name; header-only NVTX costs a branch when no tool is attached.
struct StageRange {
  explicit StageRange(const char* name) { nvtxRangePushA(name); }
  ~StageRange() { nvtxRangePop(); }
  StageRange(const StageRange&) = delete;
  StageRange& operator=(const StageRange&) = delete;
};

static std::atomic<uint64_t> g_launches{0};
static std::atomic<uint64_t> g_wait_limit_ns{0};
static std::atomic<int> g_stall_producer{0};
static std::atomic<int> g_cta_group{2};
static std::atomic<cudaEvent_t> g_ev_start{nullptr}, g_ev_stop{nullptr};
constexpr uint64_t kDefaultWaitLimitNs = 2000000000ull;

void count_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

static thread_local char g_err[512] = "";

static rmm_status fail(rmm_status s, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_err, sizeof(g_err), fmt, ap);
  va_end(ap);
  return s;
}

void set_last_error(const char* msg) { snprintf(g_err, sizeof(g_err), "%s", msg); }

static rmm_status cuda_fail(cudaError_t e, const char* what, const char* why = nullptr) {
  return fail(RMM_ERR_CUDA, "%s: %s%s%s", what, cudaGetErrorString(e), why ? " — " : "", why ? why : "");
}

// ---------------------------------------------------------------- debug checks
// Off by default. On (rmm_set_debug(1), or RMM_DEBUG set to anything but "0"
// in the environment when the first call is made), the stage calls that take
// a caller's index list validate it on the device before anything reads
// through it, and the fused calls wait for their kernels and report the
// device status word; both synchronise the stream.
static std::atomic<int> g_debug{-1};  // -1: not yet read from the environment

static bool debug_on() {
  int d = g_debug.load();
  if (d < 0) {
    const char* e = std::getenv("RMM_DEBUG");
    int want = (e && *e && std::strcmp(e, "0") != 0) ? 1 : 0;
    g_debug.compare_exchange_strong(d, want);
    d = g_debug.load();
  }
  return d == 1;
}

// [0]: number of indices outside [0, K); [1]: the first such position.
__device__ uint32_t g_idx_check[2];

__global__ void check_indices_kernel(const int32_t* __restrict__ idx, int64_t n, int64_t K, uint32_t* out) {
  for (int64_t i = int64_t(blockIdx.x) * blockDim.x + threadIdx.x; i < n; i += int64_t(gridDim.x) * blockDim.x) {
    const int32_t v = idx[i];
    if (v < 0 || int64_t(v) >= K) {
      atomicAdd(&out[0], 1u);
      atomicMin(&out[1], uint32_t(i < 0xFFFFFFFFll ? i : 0xFFFFFFFFll));
    }
  }
}

// idx [batch][k_keep]: every entry must lie in [0, K). Synchronises `st`.
static rmm_status debug_check_indices(const int32_t* idx, int64_t batch, int64_t k_keep, int64_t K, const char* who,
                                      cudaStream_t st) {
  uint32_t* out = nullptr;
  cudaError_t e = cudaGetSymbolAddress(reinterpret_cast<void**>(&out), g_idx_check);
  const uint32_t init[2] = {0u, 0xFFFFFFFFu};
  if (e == cudaSuccess) e = cudaMemcpyAsync(out, init, sizeof(init), cudaMemcpyHostToDevice, st);
  const int64_t n = batch * k_keep;
  if (e == cudaSuccess) {
    const unsigned blocks = unsigned(std::min<int64_t>((n + 255) / 256, 148 * 4));
    count_launch();
    check_indices_kernel<<<blocks, 256, 0, st>>>(idx, n, K, out);
    e = cudaGetLastError();
  }
  uint32_t got[2] = {0u, 0u};
  if (e == cudaSuccess) e = cudaMemcpyAsync(got, out, sizeof(got), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "index check (debug)");
  if (got[0] == 0) return RMM_OK;
  int32_t v = 0;
  e = cudaMemcpy(&v, idx + got[1], sizeof(v), cudaMemcpyDeviceToHost);
  if (e != cudaSuccess) return cuda_fail(e, "index check (debug)");
  return fail(RMM_ERR_INVALID, "%s: %u kept indices outside [0, %lld); first idx[%lld][%lld] = %d", who, got[0],
              (long long)K, (long long)(got[1] / k_keep), (long long)(got[1] % k_keep), v);
}

// Debug mode, after a fused call: wait for it and return its device status.
static rmm_status debug_call_status(uint32_t* status, cudaStream_t st) {
  uint32_t w = 0;
  cudaError_t e = cudaMemcpyAsync(&w, status, sizeof(w), cudaMemcpyDeviceToHost, st);
  if (e == cudaSuccess) e = cudaStreamSynchronize(st);
  if (e != cudaSuccess) return cuda_fail(e, "reading the status word (debug)");
  if (w & RMM_STATUS_BIT_TIMEOUT) return fail(RMM_ERR_TIMEOUT, "a pipeline wait in the GEMM ran out");
  if (w & RMM_STATUS_BIT_NONFINITE) return fail(RMM_ERR_NONFINITE, "a slice score was NaN or Inf");
  return RMM_OK;
}

// Make the stream's device current for the rest of the call (the caller's
// framework may have made another device current); `g` puts the caller's
// device back when the entry point returns.
static rmm_status bind_device(cudaStream_t st, DeviceGuard& g) {
  const cudaError_t e = g.bind(st);
  if (e != cudaSuccess) return cuda_fail(e, "selecting the stream's device");
  return RMM_OK;
}

static inline int64_t round_up(int64_t x, int64_t m) { return (x + m - 1) / m * m; }

// Row pitch (elements) of the packed N-major B operand.
static inline int64_t packed_b_ld(int64_t N) { return round_up(N, 8); }

static uint64_t wait_limit() {
  const uint64_t lim = g_wait_limit_ns.load();
  return lim ? lim : kDefaultWaitLimitNs;
}

static bool dtype_ok(rmm_dtype d) { return d == RMM_BF16 || d == RMM_F32; }
static ElemKind kind(rmm_dtype d) { return d == RMM_BF16 ? kBF16 : kF32; }

// A batch of row-major matrices (rows x cols, leading dimension ld, batch
// stride bstride) must fit its own declared layout.
// Batch items must not overlap, except that a read-only input may repeat one
// matrix for every item (bstride == 0, e.g. one weight for a batch).
static bool layout_ok(int64_t batch, int64_t rows, int64_t cols, int64_t ld, int64_t bstride,
                      bool broadcast_ok = false) {
  if (rows < 0 || cols < 0 || ld < 0 || bstride < 0) return false;
  if (rows > 1 && ld < cols) return false;
  if (batch > 1 && rows > 0 && !(broadcast_ok && bstride == 0) && bstride < (rows - 1) * ld + cols) return false;
  return true;
}

constexpr int64_t kMaxGridBatch = 65535;
// Slices per selection: the select kernel indexes keys with 32-bit integers
// and re-reads them from global memory beyond 32768; 2^21 bounds its work.
constexpr int64_t kMaxSelectK = int64_t(1) << 21;

struct Workspace {
  uint32_t* status;
  float* s;
  int32_t* idx;
  void* a_s;             // pack route: A_S, then B_S
  void* b_st;
  void* b_m;             // stream route: B with its dropped rows zeroed [batch][K][packed_b_ld(N)]
  size_t bytes;          // every route
  size_t bytes_pack;     // the pack route: status, scores, indices, A_S, B_S
  size_t bytes_stream;   // the stream route: status, scores, indices, B_M
  size_t bytes_no_pack;  // the decode route (no packed operands): status, scores, indices
};

// How a fused call computes the product over the kept slices.
enum Route {
  kRoutePack = 0,    // pack A's kept columns and B's kept rows, tensor-core GEMM over k slices
  kRouteStream = 1,  // zero B's dropped rows, tensor-core GEMM over all K slices of A as given
  kRouteGemv = 2,    // a few rows of A: gather-GEMV straight from A and B
};

// The fused calls stream B's kept rows straight into the gather-GEMV, with no
// packed operands, for a few rows of A and a row-major B.
static bool decode_route(int64_t M, int b_kmajor) { return M <= kGemvMaxRows && !b_kmajor; }

// Narrow products (N <= 128: one column tile of the GEMM) are bound by reading
// A, and A's kept columns reach into nearly every 32-byte sector of A, so
// packing A (read A, write and re-read A_S: (1 + 2·rho)·|A| bytes) costs more
// than streaming A whole through the GEMM with B's dropped rows zeroed
// (|A| bytes; the extra multiply-adds by zero stay below the tensor-core
// time of reading A). The GEMM reads A by TMA, so A must be 16-byte aligned
// with a row pitch and batch stride that are multiples of 8 elements.
static bool stream_shape(int64_t M, int64_t N, int b_kmajor, rmm_dtype in) {
  return in == RMM_BF16 && !b_kmajor && N <= 128 && M > kGemvMaxRows;
}
static bool stream_layout_ok(const void* A, int64_t lda, int64_t strideA, int64_t batch) {
  return (reinterpret_cast<uintptr_t>(A) & 15u) == 0 && lda % 8 == 0 &&
         (batch == 1 || (strideA % 8 == 0 && strideA != 0));
}
static Route choose_route(int64_t batch, int64_t M, int64_t N, int b_kmajor, rmm_dtype in, const void* A,
                          int64_t lda, int64_t strideA) {
  if (decode_route(M, b_kmajor)) return kRouteGemv;
  if (stream_shape(M, N, b_kmajor, in) && stream_layout_ok(A, lda, strideA, batch)) return kRouteStream;
  return kRoutePack;
}

static Workspace carve(void* base, int64_t batch, int64_t M, int64_t K, int64_t N, int64_t k_keep, rmm_dtype in) {
  const int64_t kp = round_up(k_keep, 64);
  const int64_t eb = in == RMM_BF16 ? 2 : 4;
  auto al = [](int64_t x) { return round_up(x, 1024); };
  int64_t off = 0;
  Workspace w;
  const uintptr_t p = reinterpret_cast<uintptr_t>(base);
  w.status = reinterpret_cast<uint32_t*>(p + off);
  off += al(4);
  w.s = reinterpret_cast<float*>(p + off);
  off += al(batch * K * 4);
  w.idx = reinterpret_cast<int32_t*>(p + off);
  off += al(batch * k_keep * 4);
  w.bytes_no_pack = size_t(off);
  const int64_t ops = off;
  w.a_s = reinterpret_cast<void*>(p + off);
  off += al(batch * M * kp * eb);
  w.b_st = reinterpret_cast<void*>(p + off);
  off += al(batch * packed_b_ld(N) * kp * eb);
  w.bytes_pack = size_t(off);
  w.b_m = reinterpret_cast<void*>(p + ops);
  w.bytes_stream = size_t(ops + al(batch * K * packed_b_ld(N) * eb));
  // every route these sizes can take (the stream route needs bf16, N <= 128, M > 16)
  w.bytes = in == RMM_BF16 && N <= 128 && M > kGemvMaxRows ? std::max(w.bytes_pack, w.bytes_stream) : w.bytes_pack;
  return w;
}

// ---------------------------------------------------------------- stage bodies
// bn non-null: product scores with B's norms given (B is not read).
static rmm_status do_score(const void* A, int64_t lda, int64_t sA, const void* B, int64_t ldb, int64_t sB,
                           int b_kmajor, int64_t batch, int64_t M, int64_t K, int64_t N, rmm_dtype in,
                           rmm_score_mode mode, float* s, uint32_t* status, cudaStream_t st,
                           const float* bn = nullptr, int64_t bn_stride = 0, int clear_status = 0) {
  StageRange range("rmm score");
  const MatView a{A, lda, sA, M, K};
  const int bmode = bn ? 3 : (mode == RMM_SCORE_A_ONLY ? 0 : (b_kmajor ? 2 : 1));
  const MatView b = b_kmajor ? MatView{B, ldb, sB, N, K} : MatView{B, ldb, sB, K, N};
  const cudaError_t ce = launch_score(a, b, bmode, kind(in), batch, s, status, st, bn, bn_stride, clear_status);
  if (ce != cudaSuccess) return cuda_fail(ce, "score kernel");
  return RMM_OK;
}

static rmm_status do_pack(const void* A, int64_t lda, int64_t sA, const void* B, int64_t ldb, int64_t sB, int b_kmajor,
                          int64_t batch, int64_t M, int64_t K, int64_t N, const int32_t* idx, int64_t k_keep,
                          rmm_dtype in, void* A_S, void* B_S, uint32_t* status, cudaStream_t st) {
  StageRange range("rmm pack");
  const ElemKind e = kind(in);
  const int64_t kp = round_up(k_keep, 64);
  const uint64_t lim = wait_limit();
  if (!b_kmajor) {
    bool handled = false;
    const cudaError_t be = launch_pack_both(MatView{A, lda, sA, M, K}, MatView{B, ldb, sB, K, N}, e, batch, idx, k_keep,
                                            kp, A_S, B_S, packed_b_ld(N), status, lim, st, &handled);
    if (be != cudaSuccess) return cuda_fail(be, "pack kernel (A and B)");
    if (handled) return RMM_OK;
  }
  cudaError_t ce = launch_pack_cols(MatView{A, lda, sA, M, K}, e, batch, idx, k_keep, kp, A_S, status, lim, st);
  if (ce != cudaSuccess) return cuda_fail(ce, "pack kernel (A)");
  if (b_kmajor)
    ce = launch_pack_cols(MatView{B, ldb, sB, N, K}, e, batch, idx, k_keep, kp, B_S, status, lim, st);
  else
    ce = launch_pack_rows(MatView{B, ldb, sB, K, N}, e, batch, idx, k_keep, kp, B_S, packed_b_ld(N), status, lim, st);
  if (ce != cudaSuccess) return cuda_fail(ce, "pack kernel (B)");
  return RMM_OK;
}

// B_M = B with the rows outside idx zeroed, [batch][K][packed_b_ld(N)].
static rmm_status do_mask(const void* B, int64_t ldb, int64_t sB, int64_t batch, int64_t K, int64_t N,
                          const int32_t* idx, int64_t k_keep, rmm_dtype in, void* B_M, cudaStream_t st) {
  StageRange range("rmm mask");
  const cudaError_t ce = launch_mask_rows(MatView{B, ldb, sB, K, N}, kind(in), batch, idx, k_keep, B_M, packed_b_ld(N),
                                          st);
  if (ce != cudaSuccess) return cuda_fail(ce, "mask kernel");
  return RMM_OK;
}

static GemmArgs gemm_args(const void* A_S, const void* B_S, int b_kmajor, int64_t batch, int64_t M, int64_t N,
                          int64_t k_keep, void* C, int64_t ldc, int64_t sC, rmm_dtype out, uint32_t* status) {
  GemmArgs g;
  g.a = A_S;
  g.b = B_S;
  g.b_kmajor = b_kmajor ? 1 : 0;
  g.ldb = packed_b_ld(N);
  g.c = C;
  g.batch = batch;
  g.M = M;
  g.N = N;
  g.k_pad = round_up(k_keep, 64);
  g.lda = g.k_pad;
  g.strideA = g.k_pad * M;
  g.causal_off = -1;
  g.ldc = ldc;
  g.strideC = sC;
  g.out = kind(out);
  g.status = status;
  g.wait_limit_ns = wait_limit();
  g.stall_producer = g_stall_producer.load();
  g.cta_group = g_cta_group.load();
  g.c_zeroed = 0;
  g.ev_start = g_ev_start.load();
  g.ev_stop = g_ev_stop.load();
  return g;
}

static rmm_status do_gemv(const void* A, int64_t lda, int64_t sA, const void* B, int64_t ldb, int64_t sB,
                          int64_t batch, int64_t M, int64_t N, const int32_t* idx, int64_t k_keep, rmm_dtype in,
                          void* C, int64_t ldc, int64_t sC, rmm_dtype out, cudaStream_t st) {
  StageRange range("rmm gather-gemv");
  GemvArgs g;
  g.a = A;
  g.b = B;
  g.lda = lda;
  g.strideA = sA;
  g.ldb = ldb;
  g.strideB = sB;
  g.idx = idx;
  g.k_keep = k_keep;
  g.c = C;
  g.ldc = ldc;
  g.strideC = sC;
  g.batch = batch;
  g.M = M;
  g.N = N;
  g.in = kind(in);
  g.out = kind(out);
  const cudaError_t ce = launch_gemv_gather(g, st);
  if (ce != cudaSuccess) return cuda_fail(ce, "gemv kernel");
  return RMM_OK;
}

static rmm_status do_gemm(const GemmArgs& g, rmm_dtype in, cudaStream_t st) {
  StageRange range("rmm gemm");
  cudaError_t ce;
  const char* why = nullptr;
  if (in == RMM_BF16)
    ce = launch_gemm_tc(g, st, &why);
  else
    ce = launch_gemm_simt(g, st);
  if (ce == cudaErrorNoKernelImageForDevice) return fail(RMM_ERR_UNSUPPORTED, "%s", why ? why : "unsupported device");
  if (ce != cudaSuccess) return cuda_fail(ce, "gemm kernel", why);
  return RMM_OK;
}

static rmm_status check_common(int64_t batch, int64_t M, int64_t K, int64_t N, rmm_dtype in) {
  if (!dtype_ok(in)) return fail(RMM_ERR_INVALID, "unknown input dtype %d", int(in));
  if (batch < 0 || M < 0 || N < 0) return fail(RMM_ERR_INVALID, "negative size");
  if (K < 1) return fail(RMM_ERR_INVALID, "K must be >= 1 (got %lld)", (long long)K);
  if (K > kMaxSelectK) return fail(RMM_ERR_UNSUPPORTED, "K > %lld slices per selection", (long long)kMaxSelectK);
  if (batch > kMaxGridBatch) return fail(RMM_ERR_UNSUPPORTED, "batch > %lld", (long long)kMaxGridBatch);
  return RMM_OK;
}

static rmm_status check_ab(const void* A, int64_t lda, int64_t sA, const void* B, int64_t ldb, int64_t sB,
                           int b_kmajor, int64_t batch, int64_t M, int64_t K, int64_t N, bool need_b) {
  if (batch > 0 && M > 0 && !A) return fail(RMM_ERR_INVALID, "A is NULL");
  if (!layout_ok(batch, M, K, lda, sA, true)) return fail(RMM_ERR_INVALID, "A layout (lda/strideA) is too small");
  if (need_b) {
    if (batch > 0 && N > 0 && !B) return fail(RMM_ERR_INVALID, "B is NULL");
    const bool ok = b_kmajor ? layout_ok(batch, N, K, ldb, sB, true) : layout_ok(batch, K, N, ldb, sB, true);
    if (!ok) return fail(RMM_ERR_INVALID, "B layout (ldb/strideB) is too small");
  }
  return RMM_OK;
}

}  // namespace rmm

using namespace rmm;

extern "C" {

int64_t rmm_keep_count(double rho, int64_t K) {
  if (!(rho > 0.0 && rho <= 1.0) || K < 1) return -1;
  const double k = std::ceil(rho * double(K));
  if (k < 1.0) return 1;
  if (k > double(K)) return K;
  return int64_t(k);
}

int64_t rmm_padded_keep(int64_t k_keep) { return k_keep <= 0 ? 0 : round_up(k_keep, 64); }

size_t rmm_workspace_size(int64_t batch, int64_t M, int64_t K, int64_t N, int64_t k_keep, rmm_dtype in) {
  if (batch < 0 || M < 0 || K < 0 || N < 0 || k_keep < 0 || !dtype_ok(in)) return 0;
  return carve(nullptr, batch, M, K, N, k_keep, in).bytes;
}

size_t rmm_workspace_size_for(int64_t batch, int64_t M, int64_t K, int64_t N, int64_t k_keep, rmm_dtype in,
                              int b_kmajor) {
  if (batch < 0 || M < 0 || K < 0 || N < 0 || k_keep < 0 || !dtype_ok(in)) return 0;
  const Workspace w = carve(nullptr, batch, M, K, N, k_keep, in);
  if (decode_route(M, b_kmajor)) return w.bytes_no_pack;
  return stream_shape(M, N, b_kmajor, in) ? w.bytes_stream : w.bytes_pack;
}

int rmm_fused_route(int64_t batch, int64_t M, int64_t N, int b_kmajor, rmm_dtype in, const void* A, int64_t lda,
                    int64_t strideA) {
  if (batch < 0 || M < 0 || N < 0 || !dtype_ok(in)) return -1;
  return int(choose_route(batch, M, N, b_kmajor, in, A, lda, strideA));
}

rmm_status rmm_score(const void* A, int64_t lda, int64_t strideA, const void* B, int64_t ldb, int64_t strideB,
                     int b_kmajor, int64_t batch, int64_t M, int64_t K, int64_t N, rmm_dtype in, rmm_score_mode mode,
                     float* s, uint32_t* status_word, cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, in);
  if (r) return r;
  if (mode != RMM_SCORE_PRODUCT && mode != RMM_SCORE_A_ONLY) return fail(RMM_ERR_INVALID, "unknown score mode");
  r = check_ab(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, mode == RMM_SCORE_PRODUCT);
  if (r) return r;
  if (batch > 0 && !s) return fail(RMM_ERR_INVALID, "s is NULL");
  if (batch == 0) return RMM_OK;
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  return do_score(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, in, mode, s, status_word, stream);
}

rmm_status rmm_select(const float* s, int64_t batch, int64_t K, int64_t k_keep, int32_t* idx, uint32_t* status_word,
                      cudaStream_t stream) {
  if (batch < 0 || K < 1) return fail(RMM_ERR_INVALID, "need batch >= 0 and K >= 1");
  if (k_keep < 1 || k_keep > K) return fail(RMM_ERR_INVALID, "k_keep must be in [1, K]");
  if (K > kMaxSelectK) return fail(RMM_ERR_UNSUPPORTED, "K > %lld slices per selection", (long long)kMaxSelectK);
  if (batch > kMaxGridBatch) return fail(RMM_ERR_UNSUPPORTED, "batch > %lld", (long long)kMaxGridBatch);
  if (batch == 0) return RMM_OK;
  if (!s || !idx) return fail(RMM_ERR_INVALID, "s or idx is NULL");
  DeviceGuard dg;
  rmm_status r = bind_device(stream, dg);
  if (r) return r;
  StageRange range("rmm select");
  cudaError_t ce = launch_select(const_cast<float*>(s), batch, K, k_keep, idx, status_word, stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "select kernel");
  return RMM_OK;
}

int64_t rmm_packed_b_ld(int64_t N) { return N < 0 ? 0 : packed_b_ld(N); }

rmm_status rmm_pack(const void* A, int64_t lda, int64_t strideA, const void* B, int64_t ldb, int64_t strideB,
                    int b_kmajor, int64_t batch, int64_t M, int64_t K, int64_t N, const int32_t* idx, int64_t k_keep,
                    rmm_dtype in, void* A_S, void* B_S, uint32_t* status_word, cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, in);
  if (r) return r;
  if (k_keep < 1 || k_keep > K) return fail(RMM_ERR_INVALID, "k_keep must be in [1, K]");
  r = check_ab(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, true);
  if (r) return r;
  if (batch == 0) return RMM_OK;
  if (!idx) return fail(RMM_ERR_INVALID, "idx is NULL");
  if ((M > 0 && !A_S) || !B_S) return fail(RMM_ERR_INVALID, "A_S or B_S is NULL");
  if ((reinterpret_cast<uintptr_t>(A_S) | reinterpret_cast<uintptr_t>(B_S)) & 15u)
    return fail(RMM_ERR_INVALID, "A_S and B_S must be 16-byte aligned");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  if (debug_on() && (r = debug_check_indices(idx, batch, k_keep, K, "rmm_pack", stream))) return r;
  return do_pack(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, idx, k_keep, in, A_S, B_S, status_word,
                 stream);
}

rmm_status rmm_gemm(const void* A_S, const void* B_S, int b_kmajor, int64_t batch, int64_t M, int64_t N,
                    int64_t k_keep, rmm_dtype in, void* C, int64_t ldc, int64_t strideC, rmm_dtype out,
                    uint32_t* status_word, cudaStream_t stream) {
  if (!dtype_ok(in) || !dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown dtype");
  if (batch < 0 || M < 0 || N < 0) return fail(RMM_ERR_INVALID, "negative size");
  if (k_keep < 1) return fail(RMM_ERR_INVALID, "k_keep must be >= 1");
  if (batch > kMaxGridBatch) return fail(RMM_ERR_UNSUPPORTED, "batch > %lld", (long long)kMaxGridBatch);
  if (!layout_ok(batch, M, N, ldc, strideC)) return fail(RMM_ERR_INVALID, "C layout (ldc/strideC) is too small");
  if (batch == 0 || M == 0 || N == 0) return RMM_OK;
  if (!A_S || !B_S || !C) return fail(RMM_ERR_INVALID, "A_S, B_S or C is NULL");
  DeviceGuard dg;
  rmm_status r = bind_device(stream, dg);
  if (r) return r;
  return do_gemm(gemm_args(A_S, B_S, b_kmajor, batch, M, N, k_keep, C, ldc, strideC, out, status_word), in, stream);
}

rmm_status rmm_mask_rows(const void* B, int64_t ldb, int64_t strideB, int64_t batch, int64_t K, int64_t N,
                         const int32_t* idx, int64_t k_keep, rmm_dtype in, void* B_M, cudaStream_t stream) {
  rmm_status r = check_common(batch, 1, K, N, in);
  if (r) return r;
  if (k_keep < 1 || k_keep > K) return fail(RMM_ERR_INVALID, "k_keep must be in [1, K]");
  if (batch > 0 && N > 0 && !B) return fail(RMM_ERR_INVALID, "B is NULL");
  if (!layout_ok(batch, K, N, ldb, strideB, true)) return fail(RMM_ERR_INVALID, "B layout (ldb/strideB) is too small");
  if (batch == 0) return RMM_OK;
  if (!idx || !B_M) return fail(RMM_ERR_INVALID, "idx or B_M is NULL");
  if (reinterpret_cast<uintptr_t>(B_M) & 15u) return fail(RMM_ERR_INVALID, "B_M must be 16-byte aligned");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  if (debug_on() && (r = debug_check_indices(idx, batch, k_keep, K, "rmm_mask_rows", stream))) return r;
  return do_mask(B, ldb, strideB, batch, K, N, idx, k_keep, in, B_M, stream);
}

rmm_status rmm_gemm_full(const void* A, int64_t lda, int64_t strideA, const void* B_M, int64_t batch, int64_t M,
                         int64_t K, int64_t N, int64_t causal_off, rmm_dtype in, void* C, int64_t ldc, int64_t strideC,
                         rmm_dtype out, uint32_t* status_word, cudaStream_t stream) {
  if (!dtype_ok(in) || !dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown dtype");
  if (in != RMM_BF16) return fail(RMM_ERR_UNSUPPORTED, "rmm_gemm_full runs on the bf16 tensor cores only");
  if (batch < 0 || M < 0 || N < 0 || K < 1) return fail(RMM_ERR_INVALID, "need batch, M, N >= 0 and K >= 1");
  if (batch > kMaxGridBatch) return fail(RMM_ERR_UNSUPPORTED, "batch > %lld", (long long)kMaxGridBatch);
  if (!layout_ok(batch, M, K, lda, strideA)) return fail(RMM_ERR_INVALID, "A layout (lda/strideA) is too small");
  if (!layout_ok(batch, M, N, ldc, strideC)) return fail(RMM_ERR_INVALID, "C layout (ldc/strideC) is too small");
  if (batch == 0 || M == 0 || N == 0) return RMM_OK;
  if (!A || !B_M || !C) return fail(RMM_ERR_INVALID, "A, B_M or C is NULL");
  if (!stream_layout_ok(A, lda, strideA, batch))
    return fail(RMM_ERR_INVALID, "A must be 16-byte aligned with a row pitch and batch stride that are multiples of 8");
  DeviceGuard dg;
  rmm_status r = bind_device(stream, dg);
  if (r) return r;
  if (causal_off < -1) return fail(RMM_ERR_INVALID, "causal_off must be -1 (dense A) or >= 0");
  GemmArgs g = gemm_args(A, B_M, 0, batch, M, N, K, C, ldc, strideC, out, status_word);
  g.lda = lda;
  g.strideA = strideA;
  g.k_pad = K;
  g.causal_off = causal_off;
  return do_gemm(g, in, stream);
}

// On the decode route a score that needs only A (B's row norms given, or the
// A-only score) is computed by the selection kernel itself when A has at
// most kRowScoreMaxM rows and K <= kRowScoreMaxK: the call then launches the
// selection and the gather-GEMV only. The selection's only block
// clears the status word when there is one batch item; with several, a memset
// does it first.
static bool select_scores(bool gemv, const float* bn, rmm_score_mode mode, int64_t M, int64_t K) {
  return gemv && (bn || mode == RMM_SCORE_A_ONLY) && M <= kRowScoreMaxM && K <= kRowScoreMaxK;
}

static RowScore row_score(const void* A, int64_t lda, int64_t strideA, int64_t batch, int64_t M, rmm_dtype in,
                          const float* bn, int64_t bn_stride) {
  const int64_t e = in == RMM_BF16 ? 2 : 4;
  RowScore rs;
  rs.A = A;
  rs.lda = lda;
  rs.sA = strideA;
  rs.M = int32_t(M);
  rs.bf16 = in == RMM_BF16 ? 1 : 0;
  rs.a_vec = (reinterpret_cast<uintptr_t>(A) & 15u) == 0 && (lda * e) % 16 == 0 && (batch == 1 || (strideA * e) % 16 == 0) ? 1 : 0;
  rs.bn = bn;
  rs.bn_stride = bn_stride;
  return rs;
}

static cudaError_t select_with_scores(const RowScore& rs, float* s, int64_t batch, int64_t K, int64_t k_keep,
                                      int32_t* idx, uint32_t* status, cudaStream_t stream) {
  StageRange range("rmm score + select");
  if (batch > 1) {
    const cudaError_t ce = cudaMemsetAsync(status, 0, 4, stream);
    if (ce != cudaSuccess) return ce;
  }
  return launch_select(s, batch, K, k_keep, idx, status, stream, nullptr, true, &rs, batch == 1);
}

static rmm_status fused_call(const void* A, int64_t lda, int64_t strideA, const void* B, int64_t ldb,
                             int64_t strideB, int b_kmajor, const float* bn, int64_t bn_stride, int64_t batch,
                             int64_t M, int64_t K, int64_t N, double rho, rmm_dtype in, rmm_score_mode mode, void* C,
                             int64_t ldc, int64_t strideC, rmm_dtype out, int32_t* idx_out, void* workspace,
                             size_t workspace_bytes, cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, in);
  if (r) return r;
  if (!dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown output dtype");
  if (mode != RMM_SCORE_PRODUCT && mode != RMM_SCORE_A_ONLY) return fail(RMM_ERR_INVALID, "unknown score mode");
  const int64_t k_keep = rmm_keep_count(rho, K);
  if (k_keep < 1) return fail(RMM_ERR_INVALID, "rho must lie in (0, 1] (got %g)", rho);
  r = check_ab(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, true);
  if (r) return r;
  if (!layout_ok(batch, M, N, ldc, strideC)) return fail(RMM_ERR_INVALID, "C layout (ldc/strideC) is too small");
  if (batch > 0 && M > 0 && N > 0 && !C) return fail(RMM_ERR_INVALID, "C is NULL");
  if (!workspace) return fail(RMM_ERR_INVALID, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) & 1023u) return fail(RMM_ERR_INVALID, "workspace must be 1 KiB aligned");
  const Workspace w = carve(workspace, batch, M, K, N, k_keep, in);
  const Route route = choose_route(batch, M, N, b_kmajor, in, A, lda, strideA);
  const size_t need = route == kRouteGemv ? w.bytes_no_pack : route == kRouteStream ? w.bytes_stream : w.bytes_pack;
  if (workspace_bytes < need)
    return fail(RMM_ERR_INVALID, "workspace too small: %zu < %zu bytes%s", workspace_bytes, need,
                route == kRoutePack && stream_shape(M, N, b_kmajor, in)
                    ? " (A's layout does not allow streaming it: 16-byte aligned base, row pitch and batch stride "
                      "multiples of 8 elements)"
                    : "");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  cudaError_t ce = cudaSuccess;
  if (batch == 0) {  // no kernel runs: clear the status word here
    ce = cudaMemsetAsync(w.status, 0, 4, stream);
    return ce == cudaSuccess ? RMM_OK : cuda_fail(ce, "cudaMemsetAsync(status)");
  }
  int32_t* idx = idx_out ? idx_out : w.idx;
  const bool gemv = route == kRouteGemv;
  const bool fold = select_scores(gemv, bn, mode, M, K);
  // the score kernel clears the status word (it is the call's first kernel)
  if (!fold && (r = do_score(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, in, mode, w.s, w.status,
                             stream, bn, bn_stride, 1)))
    return r;
  // The select runs on one SM per batch item; the C tiles that the GEMM's
  // split-K round adds into are zeroed meanwhile by helper blocks of the same
  // launch instead of by a launch of their own.
  GemmArgs g = gemm_args(w.a_s, w.b_st, b_kmajor, batch, M, N, k_keep, C, ldc, strideC, out, w.status);
  if (route == kRouteStream) {  // the GEMM contracts over all of A with B's dropped rows zeroed
    g.a = A;
    g.lda = lda;
    g.strideA = strideA;
    g.k_pad = K;
    g.b = w.b_m;
  }
  // A few rows of A (decode): the product streams B's kept rows straight
  // through idx, with no packed copy.
  SplitZero z;
  const bool zero = !gemv && in == RMM_BF16 && gemm_tc_split_zero(g, &z);
  if (fold) {
    ce = select_with_scores(row_score(A, lda, strideA, batch, M, in, bn, bn_stride), w.s, batch, K, k_keep, idx,
                            w.status, stream);
  } else {
    StageRange range("rmm select");
    ce = launch_select(w.s, batch, K, k_keep, idx, w.status, stream, zero ? &z : nullptr, gemv);
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "select kernel");
  g.c_zeroed = zero ? 1 : 0;
  if (M == 0 || N == 0) return debug_on() ? debug_call_status(w.status, stream) : RMM_OK;
  if (gemv) {
    if ((r = do_gemv(A, lda, strideA, B, ldb, strideB, batch, M, N, idx, k_keep, in, C, ldc, strideC, out, stream)))
      return r;
    return debug_on() ? debug_call_status(w.status, stream) : RMM_OK;
  }
  if (route == kRouteStream) {
    if ((r = do_mask(B, ldb, strideB, batch, K, N, idx, k_keep, in, w.b_m, stream))) return r;
  } else if ((r = do_pack(A, lda, strideA, B, ldb, strideB, b_kmajor, batch, M, K, N, idx, k_keep, in, w.a_s,
                          w.b_st, w.status, stream))) {
    return r;
  }
  if ((r = do_gemm(g, in, stream))) return r;
  return debug_on() ? debug_call_status(w.status, stream) : RMM_OK;
}

// ---------------------------------------------------------------- P·V with its softmax producer
struct SoftmaxWorkspace {
  uint32_t* status;
  float* stats;  // [bh][S_q][2]
  float* s;      // [bh][S_k]
  int32_t* idx;  // [bh][k_keep]
  void* v_m;     // [bh][S_k][packed_b_ld(d)] bf16
  size_t bytes;
};

static SoftmaxWorkspace carve_softmax(void* base, int64_t bh, int64_t S_q, int64_t S_k, int64_t d, int64_t k_keep) {
  auto al = [](int64_t x) { return round_up(x, 1024); };
  const uintptr_t p = reinterpret_cast<uintptr_t>(base);
  int64_t off = 0;
  SoftmaxWorkspace w;
  w.status = reinterpret_cast<uint32_t*>(p + off);
  off += al(4);
  w.stats = reinterpret_cast<float*>(p + off);
  off += al(bh * S_q * 8);
  w.s = reinterpret_cast<float*>(p + off);
  off += al(bh * S_k * 4);
  w.idx = reinterpret_cast<int32_t*>(p + off);
  off += al(bh * k_keep * 4);
  w.v_m = reinterpret_cast<void*>(p + off);
  off += al(bh * S_k * packed_b_ld(d) * 2);
  w.bytes = size_t(off);
  return w;
}

static rmm_status check_softmax(const void* L, rmm_dtype ldt, int causal, int64_t bh, int64_t S_q, int64_t S_k) {
  if (!dtype_ok(ldt)) return fail(RMM_ERR_INVALID, "unknown logits dtype");
  if (bh < 0 || S_q < 0 || S_k < 1) return fail(RMM_ERR_INVALID, "need bh, S_q >= 0 and S_k >= 1");
  if (causal && S_q > S_k) return fail(RMM_ERR_INVALID, "the causal mask needs S_q <= S_k (every query sees a key)");
  if (bh > kMaxGridBatch) return fail(RMM_ERR_UNSUPPORTED, "bh > %lld", (long long)kMaxGridBatch);
  if (S_k > kMaxSelectK) return fail(RMM_ERR_UNSUPPORTED, "S_k > %lld keys per selection", (long long)kMaxSelectK);
  if (bh > 0 && S_q > 0 && !L) return fail(RMM_ERR_INVALID, "logits are NULL");
  return RMM_OK;
}

static rmm_status fused_softmax_call(const void* L, rmm_dtype ldt, float scale, int causal, const void* V,
                                     int64_t bh, int64_t S_q, int64_t S_k, int64_t d, double rho,
                                     rmm_score_mode mode, void* P, void* O, rmm_dtype out, int32_t* idx_out,
                                     void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  rmm_status r = check_softmax(L, ldt, causal, bh, S_q, S_k);
  if (r) return r;
  if (!dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown output dtype");
  if (mode != RMM_SCORE_PRODUCT && mode != RMM_SCORE_A_ONLY) return fail(RMM_ERR_INVALID, "unknown score mode");
  if (d < 1) return fail(RMM_ERR_INVALID, "d must be >= 1");
  const int64_t k_keep = rmm_keep_count(rho, S_k);
  if (k_keep < 1) return fail(RMM_ERR_INVALID, "rho must lie in (0, 1] (got %g)", rho);
  if (bh > 0 && (!V || !P || (S_q > 0 && !O))) return fail(RMM_ERR_INVALID, "V, P or O is NULL");
  // P is the GEMM's A operand, read by TMA
  if ((reinterpret_cast<uintptr_t>(P) & 15u) || S_k % 8 != 0)
    return fail(RMM_ERR_UNSUPPORTED, "P must be 16-byte aligned and S_k a multiple of 8");
  if (!workspace) return fail(RMM_ERR_INVALID, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) & 1023u) return fail(RMM_ERR_INVALID, "workspace must be 1 KiB aligned");
  const SoftmaxWorkspace w = carve_softmax(workspace, bh, S_q, S_k, d, k_keep);
  if (workspace_bytes < w.bytes)
    return fail(RMM_ERR_INVALID, "workspace too small: %zu < %zu bytes", workspace_bytes, w.bytes);
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  cudaError_t ce = cudaMemsetAsync(w.status, 0, 4, stream);  // (the row-stats kernel clears it again)
  if (ce != cudaSuccess) return cuda_fail(ce, "cudaMemsetAsync(status)");
  if (bh == 0) return RMM_OK;
  int32_t* idx = idx_out ? idx_out : w.idx;
  if (S_q == 0) {  // no query: every score is 0, so the selection keeps the lowest indices
    ce = cudaMemsetAsync(w.s, 0, size_t(bh * S_k) * 4, stream);
    if (ce == cudaSuccess) ce = launch_select(w.s, bh, S_k, k_keep, idx, w.status, stream);
    return ce == cudaSuccess ? RMM_OK : cuda_fail(ce, "select kernel");
  }
  const ElemKind lk = kind(ldt);
  {
    StageRange range("rmm softmax row stats");
    ce = launch_softmax_stats(L, lk, bh, S_q, S_k, scale, causal, w.stats, w.status, 1, stream);
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "softmax row-stats kernel");
  {
    StageRange range("rmm softmax + score");
    ce = launch_softmax_score(L, lk, bh, S_q, S_k, scale, causal, w.stats, P, mode == RMM_SCORE_PRODUCT ? V : nullptr,
                              d, w.s, w.status, stream);
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "softmax + score kernel");
  GemmArgs g = gemm_args(P, w.v_m, 0, bh, S_q, d, S_k, O, d, S_q * d, out, w.status);
  g.lda = S_k;
  g.strideA = S_q * S_k;
  g.k_pad = S_k;
  if (causal) g.causal_off = S_k - S_q;  // P is zero above the mask: tiles skip those key blocks
  SplitZero z;
  const bool zero = gemm_tc_split_zero(g, &z);
  {
    StageRange range("rmm select");
    ce = launch_select(w.s, bh, S_k, k_keep, idx, w.status, stream, zero ? &z : nullptr, false);
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "select kernel");
  g.c_zeroed = zero ? 1 : 0;
  if ((r = do_mask(V, d, S_k * d, bh, S_k, d, idx, k_keep, RMM_BF16, w.v_m, stream))) return r;
  if ((r = do_gemm(g, RMM_BF16, stream))) return r;
  return debug_on() ? debug_call_status(w.status, stream) : RMM_OK;
}

static rmm_status check_bn(const float* bn, int64_t bn_stride, int64_t batch, int64_t K) {
  if (batch > 0 && !bn) return fail(RMM_ERR_INVALID, "b_norm is NULL");
  if (bn_stride < 0 || (batch > 1 && bn_stride != 0 && bn_stride < K))
    return fail(RMM_ERR_INVALID, "b_norm_stride must be 0 (shared) or >= K");
  return RMM_OK;
}

rmm_status rmm_matmul_reduced(const void* A, int64_t lda, const void* B, int64_t ldb, int64_t M, int64_t K, int64_t N,
                              double rho, rmm_dtype in, rmm_score_mode mode, void* C, int64_t ldc, rmm_dtype out,
                              int32_t* idx_out, void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  return rmm_matmul_reduced_batched(A, lda, 0, B, ldb, 0, 0, 1, M, K, N, rho, in, mode, C, ldc, 0, out, idx_out,
                                    workspace, workspace_bytes, stream);
}

rmm_status rmm_qk_reduced(const void* Q, const void* Kmat, int64_t bh, int64_t S_q, int64_t S_k, int64_t d, double rho,
                          rmm_dtype in, rmm_score_mode mode, void* S_out, rmm_dtype out, int32_t* idx_out,
                          void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  if (S_q < 0 || S_k < 0 || d < 1) return fail(RMM_ERR_INVALID, "need S_q, S_k >= 0 and d >= 1");
  return rmm_matmul_reduced_batched(Q, d, S_q * d, Kmat, d, S_k * d, 1, bh, S_q, d, S_k, rho, in, mode, S_out, S_k,
                                    S_q * S_k, out, idx_out, workspace, workspace_bytes, stream);
}

rmm_status rmm_pv_reduced(const void* P, const void* V, int64_t bh, int64_t S_q, int64_t S_k, int64_t d, double rho,
                          rmm_dtype in, rmm_score_mode mode, void* O, rmm_dtype out, int32_t* idx_out, void* workspace,
                          size_t workspace_bytes, cudaStream_t stream) {
  if (S_q < 0 || S_k < 1 || d < 0) return fail(RMM_ERR_INVALID, "need S_q, d >= 0 and S_k >= 1");
  return rmm_matmul_reduced_batched(P, S_k, S_q * S_k, V, d, S_k * d, 0, bh, S_q, S_k, d, rho, in, mode, O, d, S_q * d,
                                    out, idx_out, workspace, workspace_bytes, stream);
}

rmm_status rmm_check(void* status_word, cudaStream_t stream) {
  if (!status_word) return fail(RMM_ERR_INVALID, "status_word is NULL");
  DeviceGuard dg;
  rmm_status r = bind_device(stream, dg);
  if (r) return r;
  uint32_t w = 0;
  cudaError_t ce = cudaMemcpyAsync(&w, status_word, 4, cudaMemcpyDeviceToHost, stream);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(stream);
  if (ce == cudaSuccess) ce = cudaMemsetAsync(status_word, 0, 4, stream);
  if (ce == cudaSuccess) ce = cudaStreamSynchronize(stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "rmm_check");
  if (w & RMM_STATUS_BIT_TIMEOUT) return fail(RMM_ERR_TIMEOUT, "a pipeline wait in the GEMM ran out");
  if (w & RMM_STATUS_BIT_NONFINITE) return fail(RMM_ERR_NONFINITE, "a slice score was NaN or Inf");
  return RMM_OK;
}

const char* rmm_last_error_string(void) { return g_err; }

void rmm_set_wait_limit_ns(uint64_t ns) { g_wait_limit_ns.store(ns); }

void rmm_set_stall_producer_for_test(int on) { g_stall_producer.store(on ? 1 : 0); }

int rmm_set_gemm_cta_group(int cta_group) {
  if (cta_group != 1 && cta_group != 2) return g_cta_group.load();
  return g_cta_group.exchange(cta_group);
}

uint64_t rmm_launch_count(void) { return g_launches.load(); }

rmm_status rmm_softmax_row_stats(const void* L, rmm_dtype ldt, float scale, int causal, int64_t bh, int64_t S_q,
                                 int64_t S_k, float* stats, uint32_t* status_word, cudaStream_t stream) {
  rmm_status r = check_softmax(L, ldt, causal, bh, S_q, S_k);
  if (r) return r;
  if (bh == 0 || S_q == 0) return RMM_OK;
  if (!stats) return fail(RMM_ERR_INVALID, "stats is NULL");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  StageRange range("rmm softmax row stats");
  const cudaError_t ce = launch_softmax_stats(L, kind(ldt), bh, S_q, S_k, scale, causal, stats, status_word, 0, stream);
  return ce == cudaSuccess ? RMM_OK : cuda_fail(ce, "softmax row-stats kernel");
}

rmm_status rmm_softmax_score(const void* L, rmm_dtype ldt, float scale, int causal, const float* stats, const void* V,
                             int64_t d, int64_t bh, int64_t S_q, int64_t S_k, void* P, float* s,
                             uint32_t* status_word, cudaStream_t stream) {
  rmm_status r = check_softmax(L, ldt, causal, bh, S_q, S_k);
  if (r) return r;
  if (bh == 0) return RMM_OK;
  if (S_q > 0 && (!stats || !P)) return fail(RMM_ERR_INVALID, "stats or P is NULL");
  if (V && d < 1) return fail(RMM_ERR_INVALID, "d must be >= 1 when V is given");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  if (S_q == 0) {  // no query: every column of P is empty
    if (!s) return RMM_OK;
    const cudaError_t ce = cudaMemsetAsync(s, 0, size_t(bh * S_k) * 4, stream);
    return ce == cudaSuccess ? RMM_OK : cuda_fail(ce, "cudaMemsetAsync(s)");
  }
  StageRange range("rmm softmax + score");
  const cudaError_t ce = launch_softmax_score(L, kind(ldt), bh, S_q, S_k, scale, causal, stats, P, V, d, s,
                                              status_word, stream);
  return ce == cudaSuccess ? RMM_OK : cuda_fail(ce, "softmax + score kernel");
}

size_t rmm_pv_softmax_workspace_size(int64_t bh, int64_t S_q, int64_t S_k, int64_t d, int64_t k_keep) {
  if (bh < 0 || S_q < 0 || S_k < 0 || d < 0 || k_keep < 0) return 0;
  return carve_softmax(nullptr, bh, S_q, S_k, d, k_keep).bytes;
}

rmm_status rmm_pv_softmax_reduced(const void* L, rmm_dtype ldt, float scale, int causal, const void* V, int64_t bh,
                                  int64_t S_q, int64_t S_k, int64_t d, double rho, rmm_score_mode mode, void* P,
                                  void* O, rmm_dtype out, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                  cudaStream_t stream) {
  return fused_softmax_call(L, ldt, scale, causal, V, bh, S_q, S_k, d, rho, mode, P, O, out, idx_out, workspace,
                            workspace_bytes, stream);
}

int rmm_set_debug(int on) {
  const int prev = debug_on() ? 1 : 0;
  g_debug.store(on ? 1 : 0);
  return prev;
}

}  // extern "C"

void rmm_set_gemm_events(cudaEvent_t start, cudaEvent_t stop) {
  g_ev_start.store(start);
  g_ev_stop.store(stop);
}

rmm_status rmm_matmul_reduced_batched(const void* A, int64_t lda, int64_t strideA, const void* B, int64_t ldb,
                                      int64_t strideB, int b_kmajor, int64_t batch, int64_t M, int64_t K, int64_t N,
                                      double rho, rmm_dtype in, rmm_score_mode mode, void* C, int64_t ldc,
                                      int64_t strideC, rmm_dtype out, int32_t* idx_out, void* workspace,
                                      size_t workspace_bytes, cudaStream_t stream) {
  return fused_call(A, lda, strideA, B, ldb, strideB, b_kmajor, nullptr, 0, batch, M, K, N, rho, in, mode, C, ldc,
                    strideC, out, idx_out, workspace, workspace_bytes, stream);
}

rmm_status rmm_b_norms(const void* B, int64_t ldb, int64_t strideB, int b_kmajor, int64_t batch, int64_t K, int64_t N,
                       rmm_dtype in, float* b_norm, uint32_t* status_word, cudaStream_t stream) {
  rmm_status r = check_common(batch, 1, K, N, in);
  if (r) return r;
  const int64_t rows = b_kmajor ? N : K, cols = b_kmajor ? K : N;
  if (batch > 0 && (!B || !b_norm)) return fail(RMM_ERR_INVALID, "B or b_norm is NULL");
  if (!layout_ok(batch, rows, cols, ldb, strideB, true))
    return fail(RMM_ERR_INVALID, "B layout (ldb/strideB) is too small");
  if (batch == 0 || N == 0) {
    if (batch > 0 && N == 0 && b_norm) {
      DeviceGuard dg;
      if ((r = bind_device(stream, dg))) return r;
      cudaError_t ce = cudaMemsetAsync(b_norm, 0, size_t(batch * K) * 4, stream);
      if (ce != cudaSuccess) return cuda_fail(ce, "cudaMemsetAsync(b_norm)");
    }
    return RMM_OK;
  }
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  const cudaError_t ce = launch_b_norms(MatView{B, ldb, strideB, rows, cols}, b_kmajor, kind(in), batch, b_norm,
                                        status_word, stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "b_norms kernel");
  return RMM_OK;
}

rmm_status rmm_score_b_norms(const void* A, int64_t lda, int64_t strideA, const float* b_norm, int64_t b_norm_stride,
                             int64_t batch, int64_t M, int64_t K, rmm_dtype in, float* s, uint32_t* status_word,
                             cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, 1, in);
  if (r) return r;
  if ((r = check_bn(b_norm, b_norm_stride, batch, K))) return r;
  if (batch > 0 && M > 0 && !A) return fail(RMM_ERR_INVALID, "A is NULL");
  if (!layout_ok(batch, M, K, lda, strideA, true))
    return fail(RMM_ERR_INVALID, "A layout (lda/strideA) is too small");
  if (batch > 0 && !s) return fail(RMM_ERR_INVALID, "s is NULL");
  if (batch == 0) return RMM_OK;
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  return do_score(A, lda, strideA, nullptr, 0, 0, 0, batch, M, K, 0, in, RMM_SCORE_PRODUCT, s, status_word, stream,
                  b_norm, b_norm_stride);
}

rmm_status rmm_matmul_reduced_b_norms(const void* A, int64_t lda, int64_t strideA, const void* B, int64_t ldb,
                                      int64_t strideB, int b_kmajor, const float* b_norm, int64_t b_norm_stride,
                                      int64_t batch, int64_t M, int64_t K, int64_t N, double rho, rmm_dtype in,
                                      void* C, int64_t ldc, int64_t strideC, rmm_dtype out, int32_t* idx_out,
                                      void* workspace, size_t workspace_bytes, cudaStream_t stream) {
  rmm_status r = check_bn(b_norm, b_norm_stride, batch, K);
  if (r) return r;
  return fused_call(A, lda, strideA, B, ldb, strideB, b_kmajor, b_norm, b_norm_stride, batch, M, K, N, rho, in,
                    RMM_SCORE_PRODUCT, C, ldc, strideC, out, idx_out, workspace, workspace_bytes, stream);
}

rmm_status rmm_gemv_gather(const void* A, int64_t lda, int64_t strideA, const void* B, int64_t ldb, int64_t strideB,
                           int64_t batch, int64_t M, int64_t K, int64_t N, const int32_t* idx, int64_t k_keep,
                           rmm_dtype in, void* C, int64_t ldc, int64_t strideC, rmm_dtype out,
                           cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, in);
  if (r) return r;
  if (!dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown output dtype");
  if (M > kGemvMaxRows) return fail(RMM_ERR_INVALID, "M must be at most %lld", (long long)kGemvMaxRows);
  if (k_keep < 1 || k_keep > K) return fail(RMM_ERR_INVALID, "k_keep must be in [1, K]");
  r = check_ab(A, lda, strideA, B, ldb, strideB, 0, batch, M, K, N, true);
  if (r) return r;
  if (!layout_ok(batch, M, N, ldc, strideC)) return fail(RMM_ERR_INVALID, "C layout (ldc/strideC) is too small");
  if (batch == 0 || M == 0 || N == 0) return RMM_OK;
  if (!idx || !C) return fail(RMM_ERR_INVALID, "idx or C is NULL");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  if (debug_on() && (r = debug_check_indices(idx, batch, k_keep, K, "rmm_gemv_gather", stream))) return r;
  return do_gemv(A, lda, strideA, B, ldb, strideB, batch, M, N, idx, k_keep, in, C, ldc, strideC, out, stream);
}

// ---------------------------------------------------------------- INT8 weights
// need_align: the gather-GEMV copies 4 int8 at a time and needs Wq's rows
// 4-byte aligned; the norm and pack kernels take any alignment.
static rmm_status check_w8(const int8_t* Wq, int64_t ldw, int64_t strideW, const float* scale, int64_t scale_stride,
                           int64_t batch, int64_t K, int64_t N, bool need_align) {
  if (batch > 0 && N > 0 && (!Wq || !scale)) return fail(RMM_ERR_INVALID, "Wq or scale is NULL");
  if (!layout_ok(batch, K, N, ldw, strideW, true)) return fail(RMM_ERR_INVALID, "Wq layout (ldw/strideW) is too small");
  if (scale_stride < 0 || (batch > 1 && scale_stride != 0 && scale_stride < N))
    return fail(RMM_ERR_INVALID, "scale_stride must be 0 (shared) or >= N");
  if (need_align && ((reinterpret_cast<uintptr_t>(Wq) & 3u) || (ldw & 3) || (batch > 1 && (strideW & 3))))
    return fail(RMM_ERR_UNSUPPORTED, "Wq's rows must be 4-byte aligned for M <= 16 (the gather-GEMV)");
  return RMM_OK;
}

rmm_status rmm_b_norms_w8(const int8_t* Wq, int64_t ldw, int64_t strideW, const float* scale, int64_t scale_stride,
                          int64_t batch, int64_t K, int64_t N, float* b_norm, uint32_t* status_word,
                          cudaStream_t stream) {
  rmm_status r = check_common(batch, 1, K, N, RMM_BF16);
  if (r) return r;
  if ((r = check_w8(Wq, ldw, strideW, scale, scale_stride, batch, K, N, false))) return r;
  if (batch > 0 && !b_norm) return fail(RMM_ERR_INVALID, "b_norm is NULL");
  if (batch == 0) return RMM_OK;
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  cudaError_t ce = N == 0 ? cudaMemsetAsync(b_norm, 0, size_t(batch * K) * 4, stream)
                          : launch_b_norms_w8(Wq, ldw, strideW, scale, scale_stride, batch, K, N, b_norm,
                                              status_word, stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "b_norms_w8 kernel");
  return RMM_OK;
}

static rmm_status do_pack_w8(const void* A, int64_t lda, int64_t sA, const int8_t* Wq, int64_t ldw, int64_t sW,
                             const float* scale, int64_t s_stride, int64_t batch, int64_t M, int64_t K, int64_t N,
                             const int32_t* idx, int64_t k_keep, void* A_S, void* B_S, uint32_t* status,
                             cudaStream_t st) {
  StageRange range("rmm pack");
  const int64_t kp = round_up(k_keep, 64);
  cudaError_t ce = launch_pack_cols(MatView{A, lda, sA, M, K}, kBF16, batch, idx, k_keep, kp, A_S, status,
                                    wait_limit(), st);
  if (ce != cudaSuccess) return cuda_fail(ce, "pack kernel (A)");
  ce = launch_pack_rows_w8(Wq, ldw, sW, scale, s_stride, batch, N, idx, k_keep, kp, B_S, packed_b_ld(N), st);
  if (ce != cudaSuccess) return cuda_fail(ce, "pack kernel (INT8 weight)");
  return RMM_OK;
}

rmm_status rmm_pack_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw, int64_t strideW,
                       const float* scale, int64_t scale_stride, int64_t batch, int64_t M, int64_t K, int64_t N,
                       const int32_t* idx, int64_t k_keep, void* A_S, void* B_S, uint32_t* status_word,
                       cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, RMM_BF16);
  if (r) return r;
  if (k_keep < 1 || k_keep > K) return fail(RMM_ERR_INVALID, "k_keep must be in [1, K]");
  r = check_ab(A, lda, strideA, nullptr, 0, 0, 0, batch, M, K, N, false);
  if (r) return r;
  if ((r = check_w8(Wq, ldw, strideW, scale, scale_stride, batch, K, N, false))) return r;
  if (batch == 0) return RMM_OK;
  if (!idx || (M > 0 && !A_S) || !B_S) return fail(RMM_ERR_INVALID, "idx, A_S or B_S is NULL");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  if (debug_on() && (r = debug_check_indices(idx, batch, k_keep, K, "rmm_pack_w8", stream))) return r;
  return do_pack_w8(A, lda, strideA, Wq, ldw, strideW, scale, scale_stride, batch, M, K, N, idx, k_keep, A_S, B_S,
                    status_word, stream);
}

static rmm_status do_gemv_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                             int64_t strideW, const float* scale, int64_t scale_stride, int64_t batch, int64_t M,
                             int64_t N, const int32_t* idx, int64_t k_keep, void* C, int64_t ldc, int64_t strideC,
                             rmm_dtype out, cudaStream_t stream);

rmm_status rmm_matmul_reduced_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                                 int64_t strideW, const float* scale, int64_t scale_stride, const float* b_norm,
                                 int64_t b_norm_stride, int64_t batch, int64_t M, int64_t K, int64_t N, double rho,
                                 rmm_dtype in, rmm_score_mode mode, void* C, int64_t ldc, int64_t strideC,
                                 rmm_dtype out, int32_t* idx_out, void* workspace, size_t workspace_bytes,
                                 cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, in);
  if (r) return r;
  if (in != RMM_BF16) return fail(RMM_ERR_INVALID, "the INT8-weight path takes bf16 activations");
  if (!dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown output dtype");
  if (mode != RMM_SCORE_PRODUCT && mode != RMM_SCORE_A_ONLY) return fail(RMM_ERR_INVALID, "unknown score mode");
  if (mode == RMM_SCORE_PRODUCT && (r = check_bn(b_norm, b_norm_stride, batch, K))) return r;
  const int64_t k_keep = rmm_keep_count(rho, K);
  if (k_keep < 1) return fail(RMM_ERR_INVALID, "rho must lie in (0, 1] (got %g)", rho);
  r = check_ab(A, lda, strideA, nullptr, 0, 0, 0, batch, M, K, N, false);
  if (r) return r;
  if ((r = check_w8(Wq, ldw, strideW, scale, scale_stride, batch, K, N, M <= kGemvMaxRows))) return r;
  if (!layout_ok(batch, M, N, ldc, strideC)) return fail(RMM_ERR_INVALID, "C layout (ldc/strideC) is too small");
  if (batch > 0 && M > 0 && N > 0 && !C) return fail(RMM_ERR_INVALID, "C is NULL");
  if (!workspace) return fail(RMM_ERR_INVALID, "workspace is NULL");
  if (reinterpret_cast<uintptr_t>(workspace) & 1023u) return fail(RMM_ERR_INVALID, "workspace must be 1 KiB aligned");
  const Workspace w = carve(workspace, batch, M, K, N, k_keep, in);
  const size_t need = decode_route(M, 0) ? w.bytes_no_pack : w.bytes;
  if (workspace_bytes < need)
    return fail(RMM_ERR_INVALID, "workspace too small: %zu < %zu bytes", workspace_bytes, need);
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  cudaError_t ce = cudaSuccess;
  if (batch == 0) {
    ce = cudaMemsetAsync(w.status, 0, 4, stream);
    return ce == cudaSuccess ? RMM_OK : cuda_fail(ce, "cudaMemsetAsync(status)");
  }
  int32_t* idx = idx_out ? idx_out : w.idx;
  const float* bn = mode == RMM_SCORE_PRODUCT ? b_norm : nullptr;
  const bool gemv = decode_route(M, 0);
  const bool fold = select_scores(gemv, bn, mode, M, K);
  if (!fold && (r = do_score(A, lda, strideA, nullptr, 0, 0, 0, batch, M, K, N, in, mode, w.s, w.status, stream, bn,
                             b_norm_stride, 1)))
    return r;
  GemmArgs g = gemm_args(w.a_s, w.b_st, 0, batch, M, N, k_keep, C, ldc, strideC, out, w.status);
  SplitZero z;
  const bool zero = !gemv && gemm_tc_split_zero(g, &z);
  if (fold) {
    ce = select_with_scores(row_score(A, lda, strideA, batch, M, in, bn, b_norm_stride), w.s, batch, K, k_keep, idx,
                            w.status, stream);
  } else {
    StageRange range("rmm select");
    ce = launch_select(w.s, batch, K, k_keep, idx, w.status, stream, zero ? &z : nullptr, gemv);
  }
  if (ce != cudaSuccess) return cuda_fail(ce, "select kernel");
  g.c_zeroed = zero ? 1 : 0;
  if (M == 0 || N == 0) return debug_on() ? debug_call_status(w.status, stream) : RMM_OK;
  if (gemv) {
    if ((r = do_gemv_w8(A, lda, strideA, Wq, ldw, strideW, scale, scale_stride, batch, M, N, idx, k_keep, C, ldc,
                        strideC, out, stream)))
      return r;
  } else {
    if ((r = do_pack_w8(A, lda, strideA, Wq, ldw, strideW, scale, scale_stride, batch, M, K, N, idx, k_keep, w.a_s,
                        w.b_st, w.status, stream)))
      return r;
    if ((r = do_gemm(g, in, stream))) return r;
  }
  return debug_on() ? debug_call_status(w.status, stream) : RMM_OK;
}

static rmm_status do_gemv_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                             int64_t strideW, const float* scale, int64_t scale_stride, int64_t batch, int64_t M,
                             int64_t N, const int32_t* idx, int64_t k_keep, void* C, int64_t ldc, int64_t strideC,
                             rmm_dtype out, cudaStream_t stream) {
  StageRange range("rmm gather-gemv");
  GemvArgs v;
  v.a = A;
  v.b = Wq;
  v.lda = lda;
  v.strideA = strideA;
  v.ldb = ldw;
  v.strideB = strideW;
  v.idx = idx;
  v.k_keep = k_keep;
  v.c = C;
  v.ldc = ldc;
  v.strideC = strideC;
  v.batch = batch;
  v.M = M;
  v.N = N;
  v.in = kBF16;
  v.out = kind(out);
  const cudaError_t ce = launch_gemv_gather_w8(v, scale, scale_stride, stream);
  if (ce != cudaSuccess) return cuda_fail(ce, "gemv kernel (INT8 weight)");
  return RMM_OK;
}

rmm_status rmm_gemv_gather_w8(const void* A, int64_t lda, int64_t strideA, const int8_t* Wq, int64_t ldw,
                              int64_t strideW, const float* scale, int64_t scale_stride, int64_t batch, int64_t M,
                              int64_t K, int64_t N, const int32_t* idx, int64_t k_keep, void* C, int64_t ldc,
                              int64_t strideC, rmm_dtype out, cudaStream_t stream) {
  rmm_status r = check_common(batch, M, K, N, RMM_BF16);
  if (r) return r;
  if (!dtype_ok(out)) return fail(RMM_ERR_INVALID, "unknown output dtype");
  if (M > kGemvMaxRows) return fail(RMM_ERR_INVALID, "M must be at most %lld", (long long)kGemvMaxRows);
  if (k_keep < 1 || k_keep > K) return fail(RMM_ERR_INVALID, "k_keep must be in [1, K]");
  if ((r = check_ab(A, lda, strideA, nullptr, 0, 0, 0, batch, M, K, N, false))) return r;
  if ((r = check_w8(Wq, ldw, strideW, scale, scale_stride, batch, K, N, true))) return r;
  if (!layout_ok(batch, M, N, ldc, strideC)) return fail(RMM_ERR_INVALID, "C layout (ldc/strideC) is too small");
  if (batch == 0 || M == 0 || N == 0) return RMM_OK;
  if (!idx || !C) return fail(RMM_ERR_INVALID, "idx or C is NULL");
  DeviceGuard dg;
  if ((r = bind_device(stream, dg))) return r;
  if (debug_on() && (r = debug_check_indices(idx, batch, k_keep, K, "rmm_gemv_gather_w8", stream))) return r;
  return do_gemv_w8(A, lda, strideA, Wq, ldw, strideW, scale, scale_stride, batch, M, N, idx, k_keep, C, ldc,
                    strideC, out, stream);
}

