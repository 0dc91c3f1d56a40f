// C ABI of libtpmlp (declared in include/tp_mlp.h): argument validation,
// per-device state, and dispatch to the kernels.  No device memory is
// allocated here; the caller owns every buffer.
#include <cuda_runtime.h>

#include <atomic>
#include <cstdarg>
#include <cstdint>
#include <cstdio>
#include <mutex>

#include "tp_internal.h"
#include "tp_launch.cuh"
#include "tp_mlp.h"

// Per-device status word written by the bounded device-side waits.
__device__ unsigned int g_tp_status_word = 0;

namespace tpk {
namespace {

std::atomic<uint64_t> g_launches{0};
std::atomic<uint64_t> g_timeout_ns{2000000000ull};
std::atomic<int64_t> g_debug_drop{-1};
std::atomic<int> g_debug_skip{0};   // tensor-core launches to pass before the drop applies
thread_local char g_detail[512] = "";

constexpr int kMaxDevices = 64;
int g_num_sms[kMaxDevices] = {};
int g_cc_major[kMaxDevices] = {};
unsigned* g_status_addr[kMaxDevices] = {};
unsigned long long g_ctx_id[kMaxDevices] = {};   // context the entries above belong to
uint64_t g_epoch[kMaxDevices] = {};              // bumped whenever that context changes
std::mutex g_dev_mu;

tp_status fail(tp_status st, const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
  return st;
}

// Process-unique id of the calling thread's current CUDA context (0 if the
// driver cannot tell).  A device reset, or a context lost after an error,
// gives the device a new context with a new id, so per-device caches keyed
// on it are refilled instead of reusing addresses, streams or attributes of
// a context that no longer exists.
unsigned long long current_context_id() {
  using GetCurrent = CUresult (*)(CUcontext*);
  using GetId = CUresult (*)(CUcontext, unsigned long long*);
  static GetCurrent get_current = nullptr;
  static GetId get_id = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuCtxGetCurrent", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_current = reinterpret_cast<GetCurrent>(f);
    f = nullptr;
    if (cudaGetDriverEntryPoint("cuCtxGetId", &f, cudaEnableDefault, &q) == cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      get_id = reinterpret_cast<GetId>(f);
  });
  if (get_current == nullptr || get_id == nullptr) return 0;
  CUcontext ctx = nullptr;
  unsigned long long id = 0;
  if (get_current(&ctx) != CUDA_SUCCESS || ctx == nullptr) return 0;
  if (get_id(ctx, &id) != CUDA_SUCCESS) return 0;
  return id;
}

// Per-device properties and the device address of the status word, looked
// up with that device current, once per context of the device.
tp_status device_state(int* dev_out, int* sms, int* cc_major, unsigned** status,
                       uint64_t* epoch) {
  int dev = 0;
  cudaError_t e = cudaGetDevice(&dev);
  if (e != cudaSuccess) return fail(TP_ERR_CUDA, "cudaGetDevice: %s", cudaGetErrorString(e));
  if (dev < 0 || dev >= kMaxDevices) return fail(TP_ERR_UNSUPPORTED, "device index %d", dev);
  // A thread on which the runtime has not yet made the device's context
  // current reads id 0 here; the set-up below makes it current (looking up a
  // device symbol does), and the id read after it decides whether the
  // context really changed.  Where the driver cannot report ids at all, the
  // set-up runs once per device.
  unsigned long long ctx = current_context_id();
  std::lock_guard<std::mutex> lk(g_dev_mu);
  if (g_status_addr[dev] == nullptr || g_ctx_id[dev] != ctx) {
    int n = 0, major = 0;
    e = cudaDeviceGetAttribute(&n, cudaDevAttrMultiProcessorCount, dev);
    if (e == cudaSuccess) e = cudaDeviceGetAttribute(&major, cudaDevAttrComputeCapabilityMajor, dev);
    void* addr = nullptr;
    if (e == cudaSuccess) e = cudaGetSymbolAddress(&addr, g_tp_status_word);
    if (e != cudaSuccess)
      return fail(TP_ERR_CUDA, "device set-up: %s", cudaGetErrorString(e));
    ctx = current_context_id();
    if (g_status_addr[dev] == nullptr || g_ctx_id[dev] != ctx) ++g_epoch[dev];
    g_num_sms[dev] = n;
    g_cc_major[dev] = major;
    g_status_addr[dev] = static_cast<unsigned*>(addr);
    g_ctx_id[dev] = ctx;
  }
  *dev_out = dev;
  *sms = g_num_sms[dev];
  *cc_major = g_cc_major[dev];
  *status = g_status_addr[dev];
  if (epoch != nullptr) *epoch = g_epoch[dev];
  return TP_OK;
}

tp_status make_ctx(void* stream, bool tensor_core, LaunchCtx* c) {
  int cc = 0;
  tp_status st = device_state(&c->device, &c->num_sms, &cc, &c->err_word, &c->epoch);
  if (st != TP_OK) return st;
  if (tensor_core && cc != 10)
    return fail(TP_ERR_UNSUPPORTED, "bf16 path needs an sm_100 device (found sm_%d.x)", cc);
  c->stream = static_cast<cudaStream_t>(stream);
  c->timeout_ns = g_timeout_ns.load();
  c->debug_drop = -1;
  if (tensor_core && g_debug_drop.load() >= 0) {
    if (g_debug_skip.load() > 0)
      g_debug_skip.fetch_sub(1);
    else
      c->debug_drop = g_debug_drop.exchange(-1);
  }
  return TP_OK;
}

bool aligned16(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 15u) == 0; }
bool aligned4(const void* p) { return (reinterpret_cast<uintptr_t>(p) & 3u) == 0; }

tp_status check_shape(int64_t T, int64_t d, int64_t k, int p, int dtype) {
  if (p < 1) return fail(TP_ERR_INVALID_ARG, "p = %d, must be >= 1", p);
  if (T < 0 || d < 1 || k < 1)
    return fail(TP_ERR_INVALID_ARG, "sizes T=%lld d=%lld k=%lld", (long long)T, (long long)d,
                (long long)k);
  if (dtype != TP_F32 && dtype != TP_BF16) return fail(TP_ERR_INVALID_ARG, "dtype %d", dtype);
  if (k % p != 0)
    return fail(TP_ERR_INDIVISIBLE, "%lld features cannot be split evenly over %d shards",
                (long long)k, p);
  if (T > INT32_MAX || d > INT32_MAX || k > INT32_MAX || T * d > (int64_t(1) << 46) ||
      T * k > (int64_t(1) << 46) || d * k > (int64_t(1) << 46))
    return fail(TP_ERR_UNSUPPORTED, "sizes too large");
  if (dtype == TP_BF16 && (d % 8 != 0 || (k / p) % 8 != 0))
    return fail(TP_ERR_ALIGNMENT, "bf16 needs d %% 8 == 0 and k/p %% 8 == 0 (d=%lld, s=%lld)",
                (long long)d, (long long)(k / p));
  return TP_OK;
}

tp_status check_ptr(const void* ptr, const char* name, int dtype, bool tma) {
  if (ptr == nullptr) return fail(TP_ERR_INVALID_ARG, "%s is NULL", name);
  if (dtype == TP_BF16 && tma && !aligned16(ptr))
    return fail(TP_ERR_ALIGNMENT, "%s must be 16-byte aligned", name);
  if (dtype == TP_F32 && !aligned4(ptr)) return fail(TP_ERR_ALIGNMENT, "%s must be 4-byte aligned", name);
  return TP_OK;
}

tp_status check_act(int act, const void* W_up) {
  if (act < TP_ACT_GELU_TANH || act > TP_ACT_RELU) return fail(TP_ERR_INVALID_ARG, "act %d", act);
  if (act == TP_ACT_SWIGLU && W_up == nullptr)
    return fail(TP_ERR_INVALID_ARG, "SwiGLU needs W_up");
  return TP_OK;
}

tp_status cuda_status(cudaError_t e, const char* what) {
  if (e == cudaSuccess) return TP_OK;
  return fail(TP_ERR_CUDA, "%s: %s", what, cudaGetErrorString(e));
}

#define TP_TRY(expr)               \
  do {                             \
    const tp_status st_ = (expr);  \
    if (st_ != TP_OK) return st_;  \
  } while (0)

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Counters at the end of the workspace: the single-launch block's per-m-tile
// counters, or the row layer's per-region counters for the overlapped fold
// (never both in one call).
size_t counter_bytes(int64_t T, int64_t d) {
  const size_t a = block_counter_bytes(T, d), b = region_counter_bytes(T, d);
  return a > b ? a : b;
}

// Workspace layout: hidden shards Y, then (default mode) the fp32 partials,
// then the counters, each at a 256-byte boundary.
size_t workspace_bytes(int64_t T, int64_t d, int64_t k, int p, int dtype, int flags) {
  const size_t esize = dtype == TP_BF16 ? 2 : 4;
  size_t bytes = align256(static_cast<size_t>(T) * static_cast<size_t>(k) * esize);
  if (!(flags & (TP_FLAG_SPLITK_FUSED | TP_FLAG_ROW_FOLD)))
    bytes += align256(static_cast<size_t>(p) * static_cast<size_t>(T) * static_cast<size_t>(d) * 4);
  return bytes + counter_bytes(T, d);
}

tp_status column_impl(const void* X, const void* W1, const void* W_up, const void* b1, void* Y,
                      int64_t T, int64_t d, int64_t k, int p, int dtype, int act, void* stream,
                      int* zero_cnt = nullptr, int zero_n = 0) {
  TP_TRY(check_shape(T, d, k, p, dtype));
  TP_TRY(check_act(act, W_up));
  if (T == 0) return TP_OK;
  TP_TRY(check_ptr(X, "X", dtype, true));
  TP_TRY(check_ptr(W1, "W1", dtype, true));
  if (act == TP_ACT_SWIGLU) TP_TRY(check_ptr(W_up, "W_up", dtype, true));
  TP_TRY(check_ptr(Y, "Y", dtype, true));
  if (b1 != nullptr) TP_TRY(check_ptr(b1, "b1", dtype, dtype == TP_BF16));
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, dtype == TP_BF16, &c));
  if (dtype == TP_BF16)
    return launch_tc_column(c, X, W1, W_up, b1, Y, T, d, k, p, act, zero_cnt, zero_n);
  return cuda_status(launch_simt_column(c, static_cast<const float*>(X),
                                        static_cast<const float*>(W1),
                                        static_cast<const float*>(W_up),
                                        static_cast<const float*>(b1), static_cast<float*>(Y), T,
                                        d, k, p, act),
                     "fp32 column launch");
}

tp_status row_impl(const void* Y, const void* W2, float* partials, int64_t T, int64_t k,
                   int64_t d, int p, int dtype, void* stream) {
  TP_TRY(check_shape(T, d, k, p, dtype));
  if (T == 0) return TP_OK;
  TP_TRY(check_ptr(Y, "Y", dtype, true));
  TP_TRY(check_ptr(W2, "W2", dtype, true));
  if (partials == nullptr) return fail(TP_ERR_INVALID_ARG, "partials is NULL");
  if (!aligned16(partials) && dtype == TP_BF16)
    return fail(TP_ERR_ALIGNMENT, "partials must be 16-byte aligned");
  if (!aligned4(partials)) return fail(TP_ERR_ALIGNMENT, "partials must be 4-byte aligned");
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, dtype == TP_BF16, &c));
  if (dtype == TP_BF16) return launch_tc_row(c, Y, W2, partials, T, k, d, p);
  return cuda_status(launch_simt_row(c, static_cast<const float*>(Y),
                                     static_cast<const float*>(W2), partials, T, k, d, p),
                     "fp32 row launch");
}

tp_status reduce_impl(const float* partials, const float* b2, float* Z, int64_t T, int64_t d,
                      int p, void* stream) {
  if (p < 1) return fail(TP_ERR_INVALID_ARG, "p = %d, must be >= 1", p);
  if (T < 0 || d < 1) return fail(TP_ERR_INVALID_ARG, "sizes T=%lld d=%lld", (long long)T, (long long)d);
  if (T == 0) return TP_OK;
  if (partials == nullptr || Z == nullptr) return fail(TP_ERR_INVALID_ARG, "partials/Z is NULL");
  if (!aligned4(partials) || !aligned4(Z) || (b2 != nullptr && !aligned4(b2)))
    return fail(TP_ERR_ALIGNMENT, "fp32 buffers must be 4-byte aligned");
  const uintptr_t p0 = reinterpret_cast<uintptr_t>(partials);
  const uintptr_t p1 = p0 + static_cast<uintptr_t>(p) * T * d * 4;
  const uintptr_t z0 = reinterpret_cast<uintptr_t>(Z);
  const uintptr_t z1 = z0 + static_cast<uintptr_t>(T) * d * 4;
  if (z0 < p1 && p0 < z1) return fail(TP_ERR_INVALID_ARG, "Z overlaps the partials");
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, false, &c));
  return cuda_status(launch_reduce(c, partials, b2, Z, T, d, p), "reduce launch");
}

// True when [a, a + an) and [b, b + bn) share a byte.
bool ranges_overlap(const void* a, size_t an, const void* b, size_t bn) {
  const uintptr_t a0 = reinterpret_cast<uintptr_t>(a), b0 = reinterpret_cast<uintptr_t>(b);
  return a0 < b0 + bn && b0 < a0 + an;
}

// Counters at `at` for the fold beside the row layer, when that path
// applies: the bf16 path on an sm_100 device, b2 and R NULL or 16-byte
// aligned (the fold reads them as vectors).  *out is NULL otherwise, and
// *n the number of counters.  Nothing is enqueued here: the column layer
// launched before the row layer zeroes them (launch_tc_column's zero_cnt),
// or, where no column layer of this library comes first, regions_reset().
tp_status region_counters(void* at, int64_t T, int64_t d, const float* b2, const float* R,
                          int** out, int* n) {
  *out = nullptr;
  *n = 0;
  if (!region_fold_allowed() || (b2 != nullptr && !aligned16(b2)) ||
      (R != nullptr && !aligned16(R)))
    return TP_OK;
  LaunchCtx c{};
  int cc = 0;
  TP_TRY(device_state(&c.device, &c.num_sms, &cc, &c.err_word, &c.epoch));
  if (cc != 10) return TP_OK;
  *out = static_cast<int*>(at);
  *n = static_cast<int>(region_counter_bytes(T, d) / sizeof(int));
  return TP_OK;
}

// Zeroes the counters with a memset enqueued before the caller's first
// launch (so that nothing sits between the counting layer and the one
// before it).
tp_status regions_reset(int* cnt, int n, void* stream) {
  if (cnt == nullptr) return TP_OK;
  const cudaError_t e = cudaMemsetAsync(cnt, 0, static_cast<size_t>(n) * sizeof(int),
                                        static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(TP_ERR_CUDA, "counter reset: %s", cudaGetErrorString(e));
  return TP_OK;
}

tp_status fold_residual_impl(const float* partials, const float* bias, const float* R, float* H,
                             int64_t T, int64_t d, int p, const float* gamma, const float* beta,
                             void* Y, float eps, void* stream);

// bf16 row layer to partials, then the fixed-order fold of the partials
// (+ b2, + the residual R if given).  When `regions` came from
// region_counters (and were zeroed) and the layer runs on CTA pairs: inside
// the row layer (each shard's tile adds its partial to the running sum in Z,
// the last adds b2 and R; no partials written), or beside it with
// TP_DISABLE_ROW_CHAIN=1.  After it otherwise.  Same bits every way.
tp_status row_and_fold(const void* Y, const void* W2, float* P, const float* b2, float* Z,
                       int64_t T, int64_t k, int64_t d, int p, int* regions, void* stream,
                       const float* R = nullptr) {
  auto fold_after = [&]() {
    return R == nullptr ? reduce_impl(P, b2, Z, T, d, p, stream)
                        : fold_residual_impl(P, b2, R, Z, T, d, p, nullptr, nullptr, nullptr, 1e-5f,
                                             stream);
  };
  if (regions == nullptr) {
    TP_TRY(row_impl(Y, W2, P, T, k, d, p, TP_BF16, stream));
    return fold_after();
  }
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, true, &c));
  if (row_chain_allowed()) {
    bool done = false;
    TP_TRY(launch_tc_row_chain(c, Y, W2, b2, R, Z, T, k, d, p, regions, &done));
    if (done) return TP_OK;
  }
  RegionFold rf{};
  TP_TRY(launch_tc_row(c, Y, W2, P, T, k, d, p, regions, &rf));
  if (rf.cnt != nullptr)
    return cuda_status(launch_fold_regions(c, P, b2, Z, T, d, p, rf, R), "fold launch");
  return fold_after();
}

// The attention block's Q, K, V projections (identity column layers of the
// same input): one launch of CTA-pair tiles where the shapes suit it, else
// three.  The first launch zeroes `zero_cnt` (the row layer's counters).
tp_status qkv_impl(const void* X, const void* Wq, const void* Wk, const void* Wv, void* Q,
                   void* K, void* V, int64_t T, int64_t d, int64_t kq, int64_t kkv, int p,
                   void* stream, int* zero_cnt, int zero_n) {
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, true, &c));
  const void* W[3] = {Wq, Wk, Wv};
  void* Y[3] = {Q, K, V};
  const int64_t k[3] = {kq, kkv, kkv};
  bool done = false;
  TP_TRY(launch_tc_column_multi(c, X, W, Y, k, 3, T, d, p, zero_cnt, zero_n, &done));
  if (done) return TP_OK;
  const int ident = TP_ACT_IDENTITY;
  TP_TRY(launch_tc_column(c, X, Wq, nullptr, nullptr, Q, T, d, kq, p, ident, zero_cnt, zero_n));
  c.debug_drop = -1;   // an armed fault injection applies to the first launch only
  TP_TRY(launch_tc_column(c, X, Wk, nullptr, nullptr, K, T, d, kkv, p, ident));
  return launch_tc_column(c, X, Wv, nullptr, nullptr, V, T, d, kkv, p, ident);
}

tp_status check_heads(int p, int n_heads, int n_kv_heads, int head_dim) {
  if (p < 1) return fail(TP_ERR_INVALID_ARG, "p = %d, must be >= 1", p);
  if (n_heads < 1 || n_kv_heads < 1 || head_dim < 1)
    return fail(TP_ERR_INVALID_ARG, "heads %d / %d, head_dim %d", n_heads, n_kv_heads, head_dim);
  if (n_heads % p != 0 || n_kv_heads % p != 0)
    return fail(TP_ERR_INDIVISIBLE,
                "number of attention heads (%d) and key/value heads (%d) must be divisible by "
                "tensor_parallel_size (%d)",
                n_heads, n_kv_heads, p);
  if (n_heads % n_kv_heads != 0)
    return fail(TP_ERR_INVALID_ARG, "n_heads (%d) must be a multiple of n_kv_heads (%d)", n_heads,
                n_kv_heads);
  if (head_dim != 128) return fail(TP_ERR_UNSUPPORTED, "head_dim %d (128 is provided)", head_dim);
  return TP_OK;
}

tp_status attention_impl(const void* Q, const void* K, const void* V, void* O, int64_t T, int p,
                         int n_heads, int n_kv_heads, int head_dim, int causal, void* stream) {
  TP_TRY(check_heads(p, n_heads, n_kv_heads, head_dim));
  if (T < 0 || T > INT32_MAX) return fail(TP_ERR_INVALID_ARG, "T = %lld", (long long)T);
  if (T == 0) return TP_OK;
  TP_TRY(check_ptr(Q, "Q", TP_BF16, true));
  TP_TRY(check_ptr(K, "K", TP_BF16, true));
  TP_TRY(check_ptr(V, "V", TP_BF16, true));
  TP_TRY(check_ptr(O, "O", TP_BF16, true));
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, true, &c));
  return launch_tc_attention(c, Q, K, V, O, T, p, n_heads / p, n_kv_heads / p, causal);
}

tp_status check_rows(int64_t T, int64_t d) {
  if (T < 0 || d < 1) return fail(TP_ERR_INVALID_ARG, "sizes T=%lld d=%lld", (long long)T, (long long)d);
  if (T > INT32_MAX) return fail(TP_ERR_UNSUPPORTED, "T = %lld", (long long)T);
  if (d % 4 != 0 || d > 16384)
    return fail(TP_ERR_UNSUPPORTED, "row kernels need d %% 4 == 0 and d <= 16384 (d = %lld)",
                (long long)d);
  return TP_OK;
}

tp_status check_vec16(const void* ptr, const char* name, bool nullable) {
  if (ptr == nullptr) return nullable ? TP_OK : fail(TP_ERR_INVALID_ARG, "%s is NULL", name);
  if (!aligned16(ptr)) return fail(TP_ERR_ALIGNMENT, "%s must be 16-byte aligned", name);
  return TP_OK;
}

tp_status layer_norm_impl(const float* X, const float* gamma, const float* beta, void* Y, int64_t T,
                          int64_t d, float eps, void* stream) {
  TP_TRY(check_rows(T, d));
  if (!(eps > 0.0f)) return fail(TP_ERR_INVALID_ARG, "eps must be > 0");
  if (T == 0) return TP_OK;
  TP_TRY(check_vec16(X, "X", false));
  TP_TRY(check_vec16(gamma, "gamma", false));
  TP_TRY(check_vec16(beta, "beta", false));
  TP_TRY(check_vec16(Y, "Y", false));
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, false, &c));
  return cuda_status(launch_row_fold_ln(c, nullptr, 0, nullptr, X, nullptr, gamma, beta, Y, T, d, eps),
                     "layer norm launch");
}

tp_status fold_residual_impl(const float* P, const float* b, const float* R, float* Z, int64_t T,
                             int64_t d, int p, const float* gamma, const float* beta, void* Y,
                             float eps, void* stream) {
  if (p < 1) return fail(TP_ERR_INVALID_ARG, "p = %d, must be >= 1", p);
  TP_TRY(check_rows(T, d));
  if (T == 0) return TP_OK;
  TP_TRY(check_vec16(P, "partials", false));
  TP_TRY(check_vec16(b, "bias", true));
  TP_TRY(check_vec16(R, "residual", true));
  TP_TRY(check_vec16(Z, "Z", false));
  const uintptr_t p0 = reinterpret_cast<uintptr_t>(P);
  const uintptr_t p1 = p0 + static_cast<uintptr_t>(p) * T * d * 4;
  const uintptr_t z0 = reinterpret_cast<uintptr_t>(Z);
  const uintptr_t z1 = z0 + static_cast<uintptr_t>(T) * d * 4;
  if (z0 < p1 && p0 < z1) return fail(TP_ERR_INVALID_ARG, "Z overlaps the partials");
  if (R != nullptr && R != Z) {
    const uintptr_t r0 = reinterpret_cast<uintptr_t>(R);
    const uintptr_t r1 = r0 + static_cast<uintptr_t>(T) * d * 4;
    if (z0 < r1 && r0 < z1) return fail(TP_ERR_INVALID_ARG, "Z partly overlaps the residual");
  }
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, false, &c));
  return cuda_status(launch_row_fold_ln(c, P, p, b, R, Z, gamma, beta, Y, T, d, eps),
                     "fold launch");
}

size_t attn_workspace_bytes(int64_t T, int64_t d, int n_heads, int n_kv_heads, int head_dim, int p) {
  const size_t q = align256(static_cast<size_t>(T) * n_heads * head_dim * 2);
  const size_t kv = align256(static_cast<size_t>(T) * n_kv_heads * head_dim * 2);
  const size_t part = align256(static_cast<size_t>(p) * T * d * 4);
  return 2 * q + 2 * kv + part + region_counter_bytes(T, d);
}

struct BwdLayout {
  size_t dh, du, part, scratch, cnt, total;
};

BwdLayout bwd_layout(int64_t T, int64_t d, int64_t k, int p, bool swiglu) {
  BwdLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  const size_t t = static_cast<size_t>(T);
  const size_t chunks = (t + 127) / 128;
  const size_t s = static_cast<size_t>(k / p);
  L.dh = take(t * k * 2);
  L.du = swiglu ? take(t * k * 2) : 0;
  L.part = take(static_cast<size_t>(p) * t * d * 4);
  const size_t sc = chunks * (static_cast<size_t>(p) * s > static_cast<size_t>(d)
                                  ? static_cast<size_t>(p) * s : static_cast<size_t>(d));
  L.scratch = take(sc * 4);
  L.cnt = take(region_counter_bytes(T, d));
  L.total = off;
  return L;
}

struct BlockLayout {
  size_t a, h, q, k, v, o, y, p, cnt, total;
};

BlockLayout block_layout(int64_t T, int64_t d, int n_heads, int n_kv_heads, int head_dim,
                         int64_t k, int p) {
  BlockLayout L{};
  size_t off = 0;
  auto take = [&](size_t bytes) {
    const size_t at = off;
    off += align256(bytes);
    return at;
  };
  const size_t t = static_cast<size_t>(T);
  L.a = take(t * d * 2);
  L.h = take(t * d * 4);
  L.q = take(t * n_heads * head_dim * 2);
  L.k = take(t * n_kv_heads * head_dim * 2);
  L.v = take(t * n_kv_heads * head_dim * 2);
  L.o = take(t * n_heads * head_dim * 2);
  L.y = take(t * k * 2);
  L.p = take(static_cast<size_t>(p) * t * d * 4);
  L.cnt = take(region_counter_bytes(T, d));
  L.total = off;
  return L;
}


}  // namespace

tp_status current_device(int* dev, uint64_t* epoch) {
  int sms = 0, cc = 0;
  unsigned* addr = nullptr;
  return device_state(dev, &sms, &cc, &addr, epoch);
}

void note_launch() { g_launches.fetch_add(1, std::memory_order_relaxed); }

void set_error_detail(const char* fmt, ...) {
  va_list ap;
  va_start(ap, fmt);
  vsnprintf(g_detail, sizeof(g_detail), fmt, ap);
  va_end(ap);
}

}  // namespace tpk

using namespace tpk;

extern "C" {

tp_status tp_column_linear(const void* X, const void* W1, const void* W_up, const void* b1,
                           void* Y, int64_t T, int64_t d, int64_t k, int p, tp_dtype dtype,
                           tp_act act, void* stream) {
  g_detail[0] = 0;
  return column_impl(X, W1, W_up, b1, Y, T, d, k, p, dtype, act, stream);
}

tp_status tp_row_linear(const void* Y, const void* W2, float* partials, int64_t T, int64_t k,
                        int64_t d, int p, tp_dtype dtype, void* stream) {
  g_detail[0] = 0;
  return row_impl(Y, W2, partials, T, k, d, p, dtype, stream);
}

tp_status tp_reduce_partials(const float* partials, const float* b2, float* Z, int64_t T,
                             int64_t d, int p, void* stream) {
  g_detail[0] = 0;
  return reduce_impl(partials, b2, Z, T, d, p, stream);
}

size_t tp_mlp_block_workspace_size(int64_t T, int64_t d, int64_t k, int p, tp_dtype dtype,
                                   tp_act act, int flags) {
  if (check_shape(T, d, k, p, dtype) != TP_OK) return 0;
  if (act < TP_ACT_GELU_TANH || act > TP_ACT_RELU) return 0;
  return workspace_bytes(T, d, k, p, dtype, flags);
}

tp_status tp_mlp_block(const void* X, const void* W1, const void* W_up, const void* b1,
                       const void* W2, const float* b2, float* Z, void* workspace,
                       size_t workspace_size, int64_t T, int64_t d, int64_t k, int p,
                       tp_dtype dtype, tp_act act, int flags, void* stream) {
  g_detail[0] = 0;
  TP_TRY(check_shape(T, d, k, p, dtype));
  TP_TRY(check_act(act, W_up));
  if (flags & ~(TP_FLAG_SPLITK_FUSED | TP_FLAG_FUSED_LAUNCH | TP_FLAG_ROW_FOLD))
    return fail(TP_ERR_INVALID_ARG, "flags 0x%x", flags);
  const bool splitk = (flags & TP_FLAG_SPLITK_FUSED) != 0;
  const bool row_fold = (flags & TP_FLAG_ROW_FOLD) != 0;
  if (row_fold && (flags & (TP_FLAG_SPLITK_FUSED | TP_FLAG_FUSED_LAUNCH)))
    return fail(TP_ERR_INVALID_ARG, "TP_FLAG_ROW_FOLD combines with no other flag");
  if (row_fold && (dtype != TP_BF16 || (k / p) % 64 != 0))
    return fail(TP_ERR_UNSUPPORTED, "the epilogue fold needs bf16 and k/p %% 64 == 0");
  if (splitk && dtype == TP_BF16 && (k / p) % 64 != 0)
    return fail(TP_ERR_UNSUPPORTED, "split-K over shards needs k/p %% 64 == 0 for bf16");
  if (T == 0) return TP_OK;
  TP_TRY(check_ptr(X, "X", dtype, true));
  TP_TRY(check_ptr(W1, "W1", dtype, true));
  if (act == TP_ACT_SWIGLU) TP_TRY(check_ptr(W_up, "W_up", dtype, true));
  TP_TRY(check_ptr(W2, "W2", dtype, true));
  if (b1 != nullptr) TP_TRY(check_ptr(b1, "b1", dtype, dtype == TP_BF16));
  if (Z == nullptr) return fail(TP_ERR_INVALID_ARG, "Z is NULL");
  if (!aligned16(Z)) return fail(TP_ERR_ALIGNMENT, "Z must be 16-byte aligned");
  if (b2 != nullptr && !aligned4(b2)) return fail(TP_ERR_ALIGNMENT, "b2 must be 4-byte aligned");
  const size_t need = workspace_bytes(T, d, k, p, dtype, flags);
  if (workspace == nullptr || workspace_size < need)
    return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need,
                workspace == nullptr ? size_t(0) : workspace_size);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(TP_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  // Z is written while the row layer still reads the workspace (running sums
  // of the fold in its epilogue; partials read by the fold)
  if (ranges_overlap(Z, static_cast<size_t>(T) * d * 4, workspace, need))
    return fail(TP_ERR_INVALID_ARG, "Z overlaps the workspace");

  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* Y = ws;
  const size_t esize = dtype == TP_BF16 ? 2 : 4;
  const size_t y_bytes = align256(static_cast<size_t>(T) * k * esize);
  float* P = (splitk || row_fold) ? nullptr : reinterpret_cast<float*>(ws + y_bytes);
  if (dtype == TP_BF16 && (flags & TP_FLAG_FUSED_LAUNCH)) {
    // Both GEMM layers in one persistent launch (its tile counters start at
    // 0), then the fixed-order fold of the partials.  The device check comes
    // first, so that an unsupported device returns with nothing enqueued.
    LaunchCtx c{};
    TP_TRY(make_ctx(stream, true, &c));
    int* counters = reinterpret_cast<int*>(ws + need - counter_bytes(T, d));
    const cudaError_t e = cudaMemsetAsync(counters, 0, block_counter_bytes(T, d),
                                          static_cast<cudaStream_t>(stream));
    if (e != cudaSuccess) return fail(TP_ERR_CUDA, "counter reset: %s", cudaGetErrorString(e));
    TP_TRY(launch_tc_block(c, X, W1, W_up, b1, W2, b2, Y, P, Z, counters, T, d, k, p, act, splitk));
    if (splitk) return TP_OK;
    return reduce_impl(P, b2, Z, T, d, p, stream);
  }
  // Default bf16 mode: the fold runs beside the row layer where that
  // applies (region_counters); the column layer zeroes the counters.
  int* regions = nullptr;
  int n_regions = 0;
  if (!splitk && !row_fold && dtype == TP_BF16)
    TP_TRY(region_counters(ws + need - counter_bytes(T, d), T, d, b2, nullptr, &regions,
                           &n_regions));
  TP_TRY(column_impl(X, W1, W_up, b1, Y, T, d, k, p, dtype, act, stream, regions, n_regions));
  if (regions != nullptr) return row_and_fold(Y, W2, P, b2, Z, T, k, d, p, regions, stream);
  if (row_fold) {
    LaunchCtx c{};
    TP_TRY(make_ctx(stream, true, &c));
    return launch_tc_row_fold(c, Y, W2, b2, Z, T, k, d, p);
  }
  if (splitk) {
    LaunchCtx c{};
    TP_TRY(make_ctx(stream, dtype == TP_BF16, &c));
    if (dtype == TP_BF16) return launch_tc_row_splitk(c, Y, W2, b2, Z, T, k, d, p);
    return cuda_status(launch_simt_row_splitk(c, static_cast<const float*>(Y),
                                              static_cast<const float*>(W2), b2, Z, T, k, d, p),
                       "fp32 split-K launch");
  }
  TP_TRY(row_impl(Y, W2, P, T, k, d, p, dtype, stream));
  return reduce_impl(P, b2, Z, T, d, p, stream);
}

tp_status tp_attention_heads(const void* Q, const void* K, const void* V, void* O, int64_t T,
                             int p, int n_heads, int n_kv_heads, int head_dim, int causal,
                             void* stream) {
  g_detail[0] = 0;
  return attention_impl(Q, K, V, O, T, p, n_heads, n_kv_heads, head_dim, causal, stream);
}

size_t tp_attn_block_workspace_size(int64_t T, int64_t d, int n_heads, int n_kv_heads,
                                    int head_dim, int p) {
  if (check_heads(p, n_heads, n_kv_heads, head_dim) != TP_OK || T < 0 || d < 1) return 0;
  return attn_workspace_bytes(T, d, n_heads, n_kv_heads, head_dim, p);
}

tp_status tp_attn_block(const void* X, const void* Wq, const void* Wk, const void* Wv,
                        const void* Wo, const float* bo, float* Z, void* workspace,
                        size_t workspace_size, int64_t T, int64_t d, int n_heads, int n_kv_heads,
                        int head_dim, int p, int causal, void* stream) {
  g_detail[0] = 0;
  TP_TRY(check_heads(p, n_heads, n_kv_heads, head_dim));
  const int64_t kq = static_cast<int64_t>(n_heads) * head_dim;
  const int64_t kkv = static_cast<int64_t>(n_kv_heads) * head_dim;
  TP_TRY(check_shape(T, d, kq, p, TP_BF16));
  if (T == 0) return TP_OK;
  TP_TRY(check_ptr(X, "X", TP_BF16, true));
  TP_TRY(check_ptr(Wq, "Wq", TP_BF16, true));
  TP_TRY(check_ptr(Wk, "Wk", TP_BF16, true));
  TP_TRY(check_ptr(Wv, "Wv", TP_BF16, true));
  TP_TRY(check_ptr(Wo, "Wo", TP_BF16, true));
  if (Z == nullptr) return fail(TP_ERR_INVALID_ARG, "Z is NULL");
  if (!aligned16(Z)) return fail(TP_ERR_ALIGNMENT, "Z must be 16-byte aligned");
  if (bo != nullptr && !aligned4(bo)) return fail(TP_ERR_ALIGNMENT, "bo must be 4-byte aligned");
  const size_t need = attn_workspace_bytes(T, d, n_heads, n_kv_heads, head_dim, p);
  if (workspace == nullptr || workspace_size < need)
    return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need,
                workspace == nullptr ? size_t(0) : workspace_size);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(TP_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  if (ranges_overlap(Z, static_cast<size_t>(T) * d * 4, workspace, need))
    return fail(TP_ERR_INVALID_ARG, "Z overlaps the workspace");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t qb = align256(static_cast<size_t>(T) * kq * 2);
  const size_t kvb = align256(static_cast<size_t>(T) * kkv * 2);
  void* Q = ws;
  void* K = ws + qb;
  void* V = ws + qb + kvb;
  void* O = ws + qb + 2 * kvb;
  float* P = reinterpret_cast<float*>(ws + 2 * qb + 2 * kvb);
  int* regions = nullptr;
  int n_regions = 0;
  TP_TRY(region_counters(ws + need - region_counter_bytes(T, d), T, d, bo, nullptr, &regions,
                         &n_regions));
  TP_TRY(qkv_impl(X, Wq, Wk, Wv, Q, K, V, T, d, kq, kkv, p, stream, regions, n_regions));
  TP_TRY(attention_impl(Q, K, V, O, T, p, n_heads, n_kv_heads, head_dim, causal, stream));
  return row_and_fold(O, Wo, P, bo, Z, T, kq, d, p, regions, stream);
}

tp_status tp_layer_norm(const float* X, const float* gamma, const float* beta, void* Y, int64_t T,
                        int64_t d, float eps, void* stream) {
  g_detail[0] = 0;
  return layer_norm_impl(X, gamma, beta, Y, T, d, eps, stream);
}

tp_status tp_reduce_partials_residual(const float* partials, const float* bias,
                                      const float* residual, float* Z, int64_t T, int64_t d, int p,
                                      void* stream) {
  g_detail[0] = 0;
  return fold_residual_impl(partials, bias, residual, Z, T, d, p, nullptr, nullptr, nullptr, 1e-5f,
                            stream);
}


size_t tp_transformer_block_workspace_size(int64_t T, int64_t d, int n_heads, int n_kv_heads,
                                           int head_dim, int64_t k, int p) {
  if (check_heads(p, n_heads, n_kv_heads, head_dim) != TP_OK || T < 0 || d < 1 || k < 1) return 0;
  return block_layout(T, d, n_heads, n_kv_heads, head_dim, k, p).total;
}

tp_status tp_transformer_block(const float* X, const tp_block_params* prm, float* out,
                               void* workspace, size_t workspace_bytes, int64_t T, int64_t d,
                               int n_heads, int n_kv_heads, int head_dim, int64_t k, int p, int act,
                               int causal, float eps, void* stream) {
  g_detail[0] = 0;
  if (prm == nullptr) return fail(TP_ERR_INVALID_ARG, "params is NULL");
  TP_TRY(check_heads(p, n_heads, n_kv_heads, head_dim));
  TP_TRY(check_rows(T, d));
  TP_TRY(check_shape(T, d, k, p, TP_BF16));
  TP_TRY(check_act(act, prm->W_up));
  if (!(eps > 0.0f)) return fail(TP_ERR_INVALID_ARG, "eps must be > 0");
  if (T == 0) return TP_OK;
  TP_TRY(check_vec16(X, "X", false));
  TP_TRY(check_vec16(out, "out", false));
  TP_TRY(check_vec16(prm->ln1_gamma, "ln1_gamma", false));
  TP_TRY(check_vec16(prm->ln1_beta, "ln1_beta", false));
  TP_TRY(check_vec16(prm->ln2_gamma, "ln2_gamma", false));
  TP_TRY(check_vec16(prm->ln2_beta, "ln2_beta", false));
  TP_TRY(check_vec16(prm->bo, "bo", true));
  TP_TRY(check_vec16(prm->b2, "b2", true));
  const BlockLayout L = block_layout(T, d, n_heads, n_kv_heads, head_dim, k, p);
  if (workspace == nullptr || workspace_bytes < L.total)
    return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", L.total,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(TP_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  if (ranges_overlap(out, static_cast<size_t>(T) * d * 4, workspace, L.total))
    return fail(TP_ERR_INVALID_ARG, "out overlaps the workspace");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* A = ws + L.a;                       // LN1(X), later LN2(H): bf16 [T][d]
  float* H = reinterpret_cast<float*>(ws + L.h);
  void* Q = ws + L.q;
  void* K = ws + L.k;
  void* V = ws + L.v;
  void* O = ws + L.o;
  void* Yh = ws + L.y;
  float* P = reinterpret_cast<float*>(ws + L.p);
  const int64_t kq = static_cast<int64_t>(n_heads) * head_dim;
  const int64_t kkv = static_cast<int64_t>(n_kv_heads) * head_dim;
  const int ident = TP_ACT_IDENTITY;
  // The MLP's fold (+ b2 + the residual H) runs in its row layer's epilogue
  // where that applies; the counters are zeroed by the MLP's column layer.
  int* regions = nullptr;
  int n_regions = 0;
  TP_TRY(region_counters(ws + L.cnt, T, d, prm->b2, H, &regions, &n_regions));
  // LayerNorm -> attention (column Q, K, V by heads; local attention; row Wo)
  TP_TRY(layer_norm_impl(X, prm->ln1_gamma, prm->ln1_beta, A, T, d, eps, stream));
  TP_TRY(qkv_impl(A, prm->Wq, prm->Wk, prm->Wv, Q, K, V, T, d, kq, kkv, p, stream, nullptr, 0));
  TP_TRY(attention_impl(Q, K, V, O, T, p, n_heads, n_kv_heads, head_dim, causal, stream));
  TP_TRY(row_impl(O, prm->Wo, P, T, kq, d, p, TP_BF16, stream));
  // reduction #1 with the residual: H = X + fold + bo; then LayerNorm of H
  TP_TRY(fold_residual_impl(P, prm->bo, X, H, T, d, p, prm->ln2_gamma, prm->ln2_beta, A, eps,
                            stream));
  // MLP: column W1 (+ activation), row W2
  TP_TRY(column_impl(A, prm->W1, prm->W_up, prm->b1, Yh, T, d, k, p, TP_BF16, act, stream,
                     regions, n_regions));
  // row W2, then reduction #2 with the residual: out = fold + b2 + H
  return row_and_fold(Yh, prm->W2, P, prm->b2, out, T, k, d, p, regions, stream, H);
}

size_t tp_mlp_block_backward_workspace_size(int64_t T, int64_t d, int64_t k, int p, int act) {
  if (p < 1 || T < 0 || d < 1 || k < 1 || k % p != 0) return 0;
  return bwd_layout(T, d, k, p, act == TP_ACT_SWIGLU).total;
}

tp_status tp_mlp_block_backward(const void* X, const void* W1, const void* W_up, const void* W2,
                                const void* H, const void* H_up, const void* Y, const void* dZ,
                                float* dX, float* dW1, float* dW_up, float* db1, float* dW2,
                                float* db2, void* workspace, size_t workspace_bytes, int64_t T,
                                int64_t d, int64_t k, int p, int act, void* stream) {
  g_detail[0] = 0;
  TP_TRY(check_shape(T, d, k, p, TP_BF16));
  const bool swiglu = act == TP_ACT_SWIGLU;
  TP_TRY(check_act(act, W_up));
  if ((k / p) % 64 != 0)
    return fail(TP_ERR_UNSUPPORTED, "backward needs k/p %% 64 == 0 (k/p = %lld)",
                (long long)(k / p));
  if (T > 65535LL * 128) return fail(TP_ERR_UNSUPPORTED, "T = %lld", (long long)T);
  if (T == 0) return TP_OK;
  for (const void* ptr : {X, W1, W2, H, Y, dZ})
    if (ptr == nullptr || !aligned16(ptr))
      return fail(ptr == nullptr ? TP_ERR_INVALID_ARG : TP_ERR_ALIGNMENT,
                  "X, W1, W2, H, Y, dZ must be non-NULL and 16-byte aligned");
  if (swiglu && (H_up == nullptr || !aligned16(H_up) || !aligned16(W_up)))
    return fail(TP_ERR_INVALID_ARG, "SwiGLU needs W_up and H_up (16-byte aligned)");
  for (const float* ptr : {dX, dW1, dW_up, db1, dW2, db2})
    if (ptr != nullptr && !aligned16(ptr))
      return fail(TP_ERR_ALIGNMENT, "gradient outputs must be 16-byte aligned");
  const BwdLayout L = bwd_layout(T, d, k, p, swiglu);
  if (workspace == nullptr || workspace_bytes < L.total)
    return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", L.total,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(TP_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  void* dH = ws + L.dh;
  void* dU = swiglu ? ws + L.du : nullptr;
  float* part = reinterpret_cast<float*>(ws + L.part);
  float* scratch = reinterpret_cast<float*>(ws + L.scratch);
  const int64_t s = k / p;
  // The dX fold runs beside the dX partials' GEMM where that runs on
  // CTA-pair tiles; its counters are reset before the first launch.
  int* regions = nullptr;
  int n_regions = 0;
  if (dX != nullptr) {
    TP_TRY(region_counters(ws + L.cnt, T, d, nullptr, nullptr, &regions, &n_regions));
    if (regions != nullptr) {
      LaunchCtx q{};
      TP_TRY(make_ctx(stream, false, &q));
      if (bwd_dx_on_pairs(q, T, swiglu ? 2 * k : k, d, p))
        TP_TRY(regions_reset(regions, n_regions, stream));
      else
        regions = nullptr;
    }
  }
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, true, &c));
  // g backward (identity): every shard uses the whole dZ
  TP_TRY(launch_bwd_act_grad(c, dZ, W2, H, H_up, dH, dU, T, d, k, p, act));
  c.debug_drop = -1;   // an armed fault injection applies to the first launch only
  if (dW2 != nullptr) TP_TRY(launch_bwd_dw2(c, Y, dZ, dW2, T, d, k, p));
  if (dW1 != nullptr) TP_TRY(launch_bwd_dw1(c, X, dH, dU, dW1, swiglu ? dW_up : nullptr, T, d, k, p));
  if (swiglu && dW1 == nullptr && dW_up != nullptr)
    return fail(TP_ERR_INVALID_ARG, "dW_up without dW1 is not provided");
  if (db1 != nullptr)
    TP_TRY(cuda_status(launch_colsum(c, dH, db1, scratch, p, T, s, s), "bias gradient launch"));
  if (db2 != nullptr)
    TP_TRY(cuda_status(launch_colsum(c, dZ, db2, scratch, 1, T, d, d), "bias gradient launch"));
  if (dX != nullptr) {
    // f backward (all-reduce): p input-gradient partials, folded in shard order
    RegionFold rf{};
    TP_TRY(launch_bwd_dx_partials(c, dH, dU, W1, W_up, part, T, d, k, p, regions, &rf));
    if (rf.cnt != nullptr)
      TP_TRY(cuda_status(launch_fold_regions(c, part, nullptr, dX, T, d, p, rf), "fold launch"));
    else
      TP_TRY(cuda_status(launch_reduce(c, part, nullptr, dX, T, d, p), "fold launch"));
  }
  return TP_OK;
}

size_t tp_mlp_block_backward_recompute_workspace_size(int64_t T, int64_t d, int64_t k, int p,
                                                      int act) {
  const size_t base = tp_mlp_block_backward_workspace_size(T, d, k, p, act);
  if (base == 0) return 0;
  const size_t h = align256(static_cast<size_t>(T) * static_cast<size_t>(k) * 2);
  return base + h * (act == TP_ACT_SWIGLU ? 3 : 2);
}

tp_status tp_mlp_block_backward_recompute(const void* X, const void* W1, const void* W_up,
                                          const void* b1, const void* W2, const void* dZ,
                                          float* dX, float* dW1, float* dW_up, float* db1,
                                          float* dW2, float* db2, void* workspace,
                                          size_t workspace_bytes, int64_t T, int64_t d, int64_t k,
                                          int p, int act, void* stream) {
  g_detail[0] = 0;
  TP_TRY(check_shape(T, d, k, p, TP_BF16));
  TP_TRY(check_act(act, W_up));
  const size_t need = tp_mlp_block_backward_recompute_workspace_size(T, d, k, p, act);
  if (need == 0) return fail(TP_ERR_INVALID_ARG, "sizes");
  if (T == 0) return TP_OK;
  if (workspace == nullptr || workspace_bytes < need)
    return fail(TP_ERR_WORKSPACE, "workspace needs %zu bytes, got %zu", need,
                workspace == nullptr ? size_t(0) : workspace_bytes);
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0)
    return fail(TP_ERR_ALIGNMENT, "workspace must be 256-byte aligned");
  // Activation recomputation: the forward column layer again, keeping the
  // pre-activations (identity epilogue) and the activations, then the
  // backward pass proper in the rest of the workspace.
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  const size_t h = align256(static_cast<size_t>(T) * static_cast<size_t>(k) * 2);
  const bool swiglu = act == TP_ACT_SWIGLU;
  void* H = ws;
  void* Y = ws + h;
  void* Hu = swiglu ? ws + 2 * h : nullptr;
  uint8_t* rest = ws + h * (swiglu ? 3 : 2);
  TP_TRY(column_impl(X, W1, nullptr, b1, H, T, d, k, p, TP_BF16, TP_ACT_IDENTITY, stream));
  if (swiglu)
    TP_TRY(column_impl(X, W_up, nullptr, nullptr, Hu, T, d, k, p, TP_BF16, TP_ACT_IDENTITY, stream));
  TP_TRY(column_impl(X, W1, W_up, b1, Y, T, d, k, p, TP_BF16, act, stream));
  return tp_mlp_block_backward(X, W1, W_up, W2, H, Hu, Y, dZ, dX, dW1, dW_up, db1, dW2, db2, rest,
                               workspace_bytes - (rest - ws), T, d, k, p, act, stream);
}

tp_status tp_sync_status(void* stream) {
  g_detail[0] = 0;
  int dev = 0, sms = 0, cc = 0;
  unsigned* addr = nullptr;
  TP_TRY(device_state(&dev, &sms, &cc, &addr, nullptr));
  cudaError_t e = cudaStreamSynchronize(static_cast<cudaStream_t>(stream));
  if (e != cudaSuccess) return fail(TP_ERR_CUDA, "stream: %s", cudaGetErrorString(e));
  unsigned word = 0;
  e = cudaMemcpyFromSymbol(&word, g_tp_status_word, sizeof(word));
  if (e != cudaSuccess) return fail(TP_ERR_CUDA, "status read: %s", cudaGetErrorString(e));
  if (word != 0) {
    const unsigned zero = 0;
    e = cudaMemcpyToSymbol(g_tp_status_word, &zero, sizeof(zero));
    if (e != cudaSuccess) return fail(TP_ERR_CUDA, "status clear: %s", cudaGetErrorString(e));
    return fail(TP_ERR_DEVICE_TIMEOUT, "device wait gave up (status bits 0x%x)", word);
  }
  return TP_OK;
}

void tp_set_wait_timeout_ns(uint64_t ns) { g_timeout_ns.store(ns == 0 ? 2000000000ull : ns); }

tp_status tp_reduce_partials_gather(const float* const* partials, int p, const float* b2,
                                    float* const* outs, int n_out, int64_t row0, int64_t rows,
                                    int64_t d, void* stream) {
  g_detail[0] = 0;
  if (p < 1 || p > TP_GATHER_MAX) return fail(TP_ERR_INVALID_ARG, "p = %d (1..%d)", p, TP_GATHER_MAX);
  if (n_out < 1 || n_out > TP_GATHER_MAX)
    return fail(TP_ERR_INVALID_ARG, "n_out = %d (1..%d)", n_out, TP_GATHER_MAX);
  if (row0 < 0 || rows < 0 || d < 1 || row0 > (int64_t(1) << 40) || rows > (int64_t(1) << 40) ||
      d > (int64_t(1) << 30))
    return fail(TP_ERR_INVALID_ARG, "row0=%lld rows=%lld d=%lld", (long long)row0,
                (long long)rows, (long long)d);
  if (partials == nullptr || outs == nullptr)
    return fail(TP_ERR_INVALID_ARG, "pointer tables must not be NULL");
  for (int j = 0; j < p; ++j) {
    if (partials[j] == nullptr) return fail(TP_ERR_INVALID_ARG, "partials[%d] is NULL", j);
    if (!aligned4(partials[j])) return fail(TP_ERR_ALIGNMENT, "partials[%d] not 4-byte aligned", j);
  }
  if (b2 != nullptr && !aligned4(b2)) return fail(TP_ERR_ALIGNMENT, "b2 not 4-byte aligned");
  const uintptr_t lo = static_cast<uintptr_t>(row0 * d * 4);
  const uintptr_t hi = static_cast<uintptr_t>((row0 + rows) * d * 4);
  for (int q = 0; q < n_out; ++q) {
    if (outs[q] == nullptr) return fail(TP_ERR_INVALID_ARG, "outs[%d] is NULL", q);
    if (!aligned4(outs[q])) return fail(TP_ERR_ALIGNMENT, "outs[%d] not 4-byte aligned", q);
    const uintptr_t o0 = reinterpret_cast<uintptr_t>(outs[q]) + lo;
    const uintptr_t o1 = reinterpret_cast<uintptr_t>(outs[q]) + hi;
    for (int j = 0; j < p && rows > 0; ++j) {
      const uintptr_t p0 = reinterpret_cast<uintptr_t>(partials[j]) + lo;
      const uintptr_t p1 = reinterpret_cast<uintptr_t>(partials[j]) + hi;
      if (o0 < p1 && p0 < o1)
        return fail(TP_ERR_INVALID_ARG, "outs[%d] overlaps partials[%d] on the slab", q, j);
    }
  }
  if (rows == 0) return TP_OK;
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, false, &c));
  return cuda_status(launch_gather_fold(c, partials, p, b2, outs, n_out, row0, rows, d),
                     "gather-fold launch");
}

tp_status tp_ipc_export(const void* ptr, tp_ipc_handle* handle) {
  g_detail[0] = 0;
  if (ptr == nullptr || handle == nullptr) return fail(TP_ERR_INVALID_ARG, "NULL argument");
  return ipc_export(ptr, handle);
}

tp_status tp_ipc_import(const tp_ipc_handle* handle, void** ptr) {
  g_detail[0] = 0;
  if (ptr == nullptr || handle == nullptr) return fail(TP_ERR_INVALID_ARG, "NULL argument");
  return ipc_import(handle, ptr);
}

tp_status tp_ipc_release(const tp_ipc_handle* handle) {
  g_detail[0] = 0;
  if (handle == nullptr) return fail(TP_ERR_INVALID_ARG, "NULL argument");
  return ipc_release(handle);
}

tp_status tp_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream) {
  g_detail[0] = 0;
  if (n < 0 || n > (int64_t(1) << 40)) return fail(TP_ERR_INVALID_ARG, "n = %lld", (long long)n);
  if (n == 0) return TP_OK;
  if (x == nullptr || y == nullptr) return fail(TP_ERR_INVALID_ARG, "x or y is NULL");
  if (!aligned4(x) || !aligned4(y)) return fail(TP_ERR_ALIGNMENT, "x and y must be 4-byte aligned");
  LaunchCtx c{};
  TP_TRY(make_ctx(stream, true, &c));
  return cuda_status(launch_exp2_poly_probe(c, x, y, n), "exp2 probe launch");
}

void tp_debug_drop_load(int64_t stage_index) { tp_debug_drop_load_after(stage_index, 0); }

void tp_debug_drop_load_after(int64_t stage_index, int launches_to_skip) {
  g_debug_skip.store(launches_to_skip < 0 ? 0 : launches_to_skip);
  g_debug_drop.store(stage_index < 0 ? -1 : stage_index);
}

const char* tp_status_string(int status) {
  switch (status) {
    case TP_OK: return "TP_OK";
    case TP_ERR_INVALID_ARG: return "TP_ERR_INVALID_ARG: invalid argument";
    case TP_ERR_INDIVISIBLE: return "TP_ERR_INDIVISIBLE: k is not divisible by p";
    case TP_ERR_ALIGNMENT: return "TP_ERR_ALIGNMENT: pointer or pitch not aligned";
    case TP_ERR_UNSUPPORTED: return "TP_ERR_UNSUPPORTED: unsupported combination";
    case TP_ERR_CUDA: return "TP_ERR_CUDA: CUDA runtime error";
    case TP_ERR_DEVICE_TIMEOUT: return "TP_ERR_DEVICE_TIMEOUT: a bounded device wait gave up";
    case TP_ERR_WORKSPACE: return "TP_ERR_WORKSPACE: workspace missing or too small";
    default: return "unknown tp_status";
  }
}

const char* tp_last_error_detail(void) { return g_detail; }

uint64_t tp_kernel_launch_count(void) { return g_launches.load(); }

int tp_abi_version(void) { return TP_ABI_VERSION; }

}  // extern "C"
