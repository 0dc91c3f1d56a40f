// tp_mlp_block_host: the whole block with X and Z in host memory.
//
// The block is row-wise: output row t of Z depends only on row t of X
// ("Tensor parallel math", "The MLP block: column then row, one
// all-reduce": every step is a product with X's rows on the left, an
// element-wise activation, or the element-wise sum of partials).  So the
// token rows can be cut into a few chunks and the chunks pipelined across the
// GPU's engines: while chunk c is computed, chunk c+1 is copied in by one copy
// engine and chunk c-1 copied out by the other.  Every chunk runs the same
// kernels as tp_mlp_block on its rows, so Z has the same bits as copying X in,
// calling tp_mlp_block on all T rows and copying Z out.
//
// Streams and events.  Each device gets three non-blocking helper streams
// (one per copy direction and a second compute stream for every other chunk)
// and a set of events, created by the first call and kept for the process.  A call forks them from the caller's stream with an event
// and joins them back before returning, so all of its work is ordered on the
// caller's stream (and can be captured into a CUDA graph from it: the host
// buffers must then be pinned).  The events are reused by every call, so the
// enqueue sequence of one call holds a per-device lock.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "tp_internal.h"
#include "tp_mlp.h"

namespace {

constexpr int kMaxDevices = 64;
constexpr int kMaxChunks = 8;
constexpr int64_t kMinChunkRows = 256;   // smaller chunks cost more in launches than they hide
constexpr int64_t kRowAlign = 128;   // keeps every chunk's rows 256-byte aligned

struct Pipe {
  bool ready = false;
  uint64_t epoch = 0;   // context epoch the streams and events were created under
  cudaStream_t h2d = nullptr, d2h = nullptr;
  cudaStream_t cmp = nullptr;   // second compute stream: odd chunks run here
  cudaEvent_t fork = nullptr, join = nullptr;
  cudaEvent_t in[kMaxChunks] = {}, out[kMaxChunks] = {};
};

Pipe g_pipe[kMaxDevices];
std::mutex g_pipe_mu[kMaxDevices];

size_t align256(size_t n) { return (n + 255) & ~size_t(255); }

// Rows per chunk: up to kMaxChunks chunks, each a multiple of kRowAlign rows
// and at least kMinChunkRows long, except the last, which takes what is left.
int64_t chunk_rows(int64_t T) {
  if (T <= kMinChunkRows) return T;
  int64_t n = (T + kMinChunkRows - 1) / kMinChunkRows;
  if (n > kMaxChunks) n = kMaxChunks;
  int64_t rc = (T + n - 1) / n;
  rc = (rc + kRowAlign - 1) / kRowAlign * kRowAlign;
  return rc;
}

// Layout: X staging [T][d], Z staging [T][d] fp32, then the block workspace
// of one chunk -- of two when there is more than one chunk (consecutive
// chunks run on two streams, each with its own workspace) -- each at a
// 256-byte boundary.
struct HostLayout {
  size_t x_bytes = 0, z_bytes = 0, block_bytes = 0, total = 0;
  int64_t rc = 0;
  int n_ws = 1;
};

bool host_layout(int64_t T, int64_t d, int64_t k, int p, tp_dtype dtype, tp_act act, int flags,
                 HostLayout* L) {
  const size_t esize = dtype == TP_BF16 ? 2 : 4;
  L->rc = chunk_rows(T);
  L->block_bytes = tp_mlp_block_workspace_size(L->rc, d, k, p, dtype, act, flags);
  if (L->block_bytes == 0) return false;
  L->block_bytes = align256(L->block_bytes);
  L->x_bytes = align256(static_cast<size_t>(T) * static_cast<size_t>(d) * esize);
  L->z_bytes = align256(static_cast<size_t>(T) * static_cast<size_t>(d) * 4);
  L->n_ws = T > L->rc ? 2 : 1;
  L->total = L->x_bytes + L->z_bytes + L->n_ws * L->block_bytes;
  return true;
}

tp_status cuda_fail(cudaError_t e, const char* what) {
  tpk::set_error_detail("%s: %s", what, cudaGetErrorString(e));
  return TP_ERR_CUDA;
}

// The device's helper streams and events, created on first use and again
// if the device has since been given a new CUDA context (the old handles died
// with the old context and are dropped, not destroyed).
tp_status pipe_for(int dev, uint64_t epoch, Pipe** out) {
  Pipe& P = g_pipe[dev];
  if (P.ready && P.epoch != epoch) P = Pipe{};
  if (!P.ready) {
    cudaError_t e = cudaStreamCreateWithFlags(&P.h2d, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&P.d2h, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaStreamCreateWithFlags(&P.cmp, cudaStreamNonBlocking);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P.fork, cudaEventDisableTiming);
    if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P.join, cudaEventDisableTiming);
    for (int c = 0; c < kMaxChunks && e == cudaSuccess; ++c) {
      e = cudaEventCreateWithFlags(&P.in[c], cudaEventDisableTiming);
      if (e == cudaSuccess) e = cudaEventCreateWithFlags(&P.out[c], cudaEventDisableTiming);
    }
    if (e != cudaSuccess) return cuda_fail(e, "helper streams / events");
    P.ready = true;
    P.epoch = epoch;
  }
  *out = &P;
  return TP_OK;
}

}  // namespace

extern "C" {

size_t tp_mlp_block_host_workspace_size(int64_t T, int64_t d, int64_t k, int p, tp_dtype dtype,
                                        tp_act act, int flags) {
  if (T < 0) return 0;
  HostLayout L;
  if (!host_layout(T, d, k, p, dtype, act, flags, &L)) return 0;
  return L.total;
}

tp_status tp_mlp_block_host(const void* X_host, const void* W1, const void* W_up, const void* b1,
                            const void* W2, const float* b2, float* Z_host, void* workspace,
                            size_t workspace_bytes, int64_t T, int64_t d, int64_t k, int p,
                            tp_dtype dtype, tp_act act, int flags, void* stream) {
  // Shapes and flags are checked by the block itself on a zero-row problem
  // (no launch); the operands here, before anything is enqueued, so that an
  // argument error never leaves copies in flight.
  const tp_status st0 =
      tp_mlp_block(nullptr, W1, W_up, b1, W2, b2, nullptr, nullptr, 0, 0, d, k, p, dtype, act,
                   flags, stream);
  if (st0 != TP_OK) return st0;
  if (T < 0) {
    tpk::set_error_detail("T = %lld", static_cast<long long>(T));
    return TP_ERR_INVALID_ARG;
  }
  if (T == 0) return TP_OK;
  const struct {
    const void* ptr;
    const char* name;
    bool required;
    size_t align;
  } operands[] = {
      {X_host, "X_host", true, 1},
      {Z_host, "Z_host", true, 1},
      {W1, "W1", true, dtype == TP_BF16 ? 16u : 4u},
      {W_up, "W_up", act == TP_ACT_SWIGLU, dtype == TP_BF16 ? 16u : 4u},
      {W2, "W2", true, dtype == TP_BF16 ? 16u : 4u},
      {b1, "b1", false, dtype == TP_BF16 ? 16u : 4u},
      {b2, "b2", false, 4u},
  };
  for (const auto& o : operands) {
    if (o.ptr == nullptr) {
      if (!o.required) continue;
      tpk::set_error_detail("%s is NULL", o.name);
      return TP_ERR_INVALID_ARG;
    }
    if ((reinterpret_cast<uintptr_t>(o.ptr) & (o.align - 1)) != 0) {
      tpk::set_error_detail("%s must be %zu-byte aligned", o.name, o.align);
      return TP_ERR_ALIGNMENT;
    }
  }
  HostLayout L;
  if (!host_layout(T, d, k, p, dtype, act, flags, &L)) {
    tpk::set_error_detail("no workspace layout for these sizes");
    return TP_ERR_INVALID_ARG;
  }
  if (workspace == nullptr || workspace_bytes < L.total) {
    tpk::set_error_detail("workspace needs %zu bytes, got %zu", L.total,
                          workspace == nullptr ? size_t(0) : workspace_bytes);
    return TP_ERR_WORKSPACE;
  }
  if ((reinterpret_cast<uintptr_t>(workspace) & 255u) != 0) {
    tpk::set_error_detail("workspace must be 256-byte aligned");
    return TP_ERR_ALIGNMENT;
  }
  int dev = 0;
  uint64_t epoch = 0;
  const tp_status sd = tpk::current_device(&dev, &epoch);
  if (sd != TP_OK) return sd;
  if (dev >= kMaxDevices) {
    tpk::set_error_detail("device index %d", dev);
    return TP_ERR_UNSUPPORTED;
  }
  cudaError_t e = cudaSuccess;

  const size_t esize = dtype == TP_BF16 ? 2 : 4;
  uint8_t* ws = static_cast<uint8_t*>(workspace);
  uint8_t* Xd = ws;
  float* Zd = reinterpret_cast<float*>(ws + L.x_bytes);
  void* block_ws = ws + L.x_bytes + L.z_bytes;
  const uint8_t* Xh = static_cast<const uint8_t*>(X_host);
  const cudaStream_t s = static_cast<cudaStream_t>(stream);
  const int64_t n_chunks = (T + L.rc - 1) / L.rc;

  std::lock_guard<std::mutex> lk(g_pipe_mu[dev]);
  Pipe* P = nullptr;
  const tp_status sp = pipe_for(dev, epoch, &P);
  if (sp != TP_OK) return sp;

  // Fork: the copies and the second compute stream start after the caller's
  // earlier work on `s`.
  const int n_streams = L.n_ws;
  if ((e = cudaEventRecord(P->fork, s)) != cudaSuccess) return cuda_fail(e, "fork record");
  if ((e = cudaStreamWaitEvent(P->h2d, P->fork, 0)) != cudaSuccess) return cuda_fail(e, "fork");
  if ((e = cudaStreamWaitEvent(P->d2h, P->fork, 0)) != cudaSuccess) return cuda_fail(e, "fork");
  if ((e = cudaStreamWaitEvent(P->cmp, P->fork, 0)) != cudaSuccess) return cuda_fail(e, "fork");
  // From here on every exit joins the helper streams back into `s`, so the
  // caller's stream never runs ahead of work this call has enqueued.
  auto join = [&](tp_status st) {
    cudaError_t j = cudaSuccess;
    for (cudaStream_t h : {P->h2d, P->d2h, P->cmp}) {
      if (j == cudaSuccess) j = cudaEventRecord(P->join, h);
      if (j == cudaSuccess) j = cudaStreamWaitEvent(s, P->join, 0);
    }
    if (st == TP_OK && j != cudaSuccess) return cuda_fail(j, "join");
    return st;
  };
  // All input copies first: they run ahead of the compute.
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int64_t r0 = c * L.rc;
    const int64_t rows = (T - r0) < L.rc ? (T - r0) : L.rc;
    const size_t off = static_cast<size_t>(r0) * static_cast<size_t>(d) * esize;
    const size_t bytes = static_cast<size_t>(rows) * static_cast<size_t>(d) * esize;
    if ((e = cudaMemcpyAsync(Xd + off, Xh + off, bytes, cudaMemcpyDefault, P->h2d)) != cudaSuccess)
      return join(cuda_fail(e, "X copy in"));
    if ((e = cudaEventRecord(P->in[c], P->h2d)) != cudaSuccess)
      return join(cuda_fail(e, "in record"));
  }
  // Each chunk's block once its rows have arrived, even chunks on the
  // caller's stream and odd ones on the second compute stream, each stream
  // with its own workspace: a chunk's kernels can then take the SMs the
  // other chunk's last wave of tiles leaves idle.  Its Z rows leave on the
  // other copy engine as soon as they are final.
  for (int64_t c = 0; c < n_chunks; ++c) {
    const int64_t r0 = c * L.rc;
    const int64_t rows = (T - r0) < L.rc ? (T - r0) : L.rc;
    const size_t xoff = static_cast<size_t>(r0) * static_cast<size_t>(d) * esize;
    const size_t zoff = static_cast<size_t>(r0) * static_cast<size_t>(d);
    const int lane = n_streams == 2 ? static_cast<int>(c & 1) : 0;
    const cudaStream_t cs = lane == 0 ? s : P->cmp;
    uint8_t* const ws_c = static_cast<uint8_t*>(block_ws) + lane * L.block_bytes;
    if ((e = cudaStreamWaitEvent(cs, P->in[c], 0)) != cudaSuccess)
      return join(cuda_fail(e, "in wait"));
    const tp_status st = tp_mlp_block(Xd + xoff, W1, W_up, b1, W2, b2, Zd + zoff, ws_c,
                                      L.block_bytes, rows, d, k, p, dtype, act, flags, cs);
    if (st != TP_OK) return join(st);
    if ((e = cudaEventRecord(P->out[c], cs)) != cudaSuccess)
      return join(cuda_fail(e, "out record"));
    if ((e = cudaStreamWaitEvent(P->d2h, P->out[c], 0)) != cudaSuccess)
      return join(cuda_fail(e, "out wait"));
    if ((e = cudaMemcpyAsync(Z_host + zoff, Zd + zoff,
                             static_cast<size_t>(rows) * static_cast<size_t>(d) * 4,
                             cudaMemcpyDefault, P->d2h)) != cudaSuccess)
      return join(cuda_fail(e, "Z copy out"));
  }
  return join(TP_OK);
}

}  // extern "C"
