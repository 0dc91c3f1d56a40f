// The all-reduce of the p partials when the p shards live on p GPUs.
//
// On p GPUs shard i sits on GPU i: X is replicated, W1's column block i and
// W2's row block i are local, every GPU forms its own full-shape partial
// P_i = act(X W1_i + b1_i) W2_i, and the partials are summed across GPUs by
// one all-reduce (day-41 post, "Simulating row parallel linear", where the
// sum of partials is the NCCL all-reduce over NVLink; "Building GPT from
// Scratch -- Part 9", "Implementation Sketch", RowParallelLinear.forward
// calls dist.all_reduce and adds the bias afterwards).
//
// This file holds the device half of that all-reduce, written so that the
// result is bit-identical to the single-GPU fixed-order fold: GPU r owns the
// token-row slab [row0, row0 + rows) of Z and
//   - reads that slab of every P_j, j = 0..p-1, in shard order -- its own
//     from local memory, the others through peer mappings over NVLink
//     (plain vector loads; no TMA, no multicast),
//   - folds them left to right with single fp32 round-to-nearest-even adds
//     (then + b2), exactly as tp_reduce_partials does,
//   - and stores the folded slab into every destination it is given: its
//     own Z and, through peer mappings, every other GPU's Z (the all-gather
//     half of the all-reduce in the same pass).
// Each GPU therefore reads (p-1)/p of a partial's bytes from its peers and
// writes as many to them: the bandwidth-optimal reduce-scatter + all-gather
// volume, in one kernel.
//
// The kernel does not wait on other GPUs: the caller orders it after every
// GPU's partial is complete and before any GPU reads Z (a stream-ordered
// barrier on each side, e.g. a one-element NCCL all-reduce).  The kernel
// ends with a system-scope fence, so its peer stores are performed before
// the kernel is seen as complete.
//
// Also in this file: export / import of device buffers between processes
// (CUDA IPC), so that the ranks can map each other's P and Z.
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <map>
#include <mutex>
#include <string>

#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {
namespace {

struct GatherPtrs {
  const float* part[TP_GATHER_MAX];
  float* out[TP_GATHER_MAX];
};

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                     __fadd_rn(a.w, b.w));
}

// Vector path: d % 4 == 0, every pointer 16-byte aligned.  `off4` is the
// slab's first float4 (row0 * d / 4), `n4` its length in float4.
template <int P>
__global__ void __launch_bounds__(256) gather_fold_vec_kernel(const GatherPtrs ptrs, int p_runtime,
                                                              int n_out,
                                                              const float* __restrict__ b2,
                                                              int64_t off4, int64_t n4,
                                                              int64_t d4) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  const int np = P > 0 ? P : p_runtime;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += stride) {
    const int64_t e = off4 + i;
    float4 acc;
    if constexpr (P > 0) {
      float4 v[P];
#pragma unroll
      for (int s = 0; s < P; ++s) v[s] = __ldcs(reinterpret_cast<const float4*>(ptrs.part[s]) + e);
      acc = v[0];
#pragma unroll
      for (int s = 1; s < P; ++s) acc = add4(acc, v[s]);
    } else {
      acc = __ldcs(reinterpret_cast<const float4*>(ptrs.part[0]) + e);
      for (int s = 1; s < np; ++s)
        acc = add4(acc, __ldcs(reinterpret_cast<const float4*>(ptrs.part[s]) + e));
    }
    if (b2 != nullptr) acc = add4(acc, __ldg(reinterpret_cast<const float4*>(b2) + (e % d4)));
    for (int q = 0; q < n_out; ++q) __stcs(reinterpret_cast<float4*>(ptrs.out[q]) + e, acc);
  }
  __threadfence_system();
}

// Scalar path for any d and 4-byte alignment.
__global__ void __launch_bounds__(256) gather_fold_scalar_kernel(const GatherPtrs ptrs, int p,
                                                                 int n_out,
                                                                 const float* __restrict__ b2,
                                                                 int64_t off, int64_t n,
                                                                 int64_t d) {
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    const int64_t e = off + i;
    float acc = ptrs.part[0][e];
    for (int s = 1; s < p; ++s) acc = __fadd_rn(acc, ptrs.part[s][e]);
    if (b2 != nullptr) acc = __fadd_rn(acc, b2[e % d]);
    for (int q = 0; q < n_out; ++q) ptrs.out[q][e] = acc;
  }
  __threadfence_system();
}

bool al16(const void* q) { return (reinterpret_cast<uintptr_t>(q) & 15u) == 0; }

// ---- CUDA IPC bookkeeping: one mapping per exported allocation and
// process, shared by every import of a buffer inside it.
using GetRange = CUresult (*)(CUdeviceptr*, size_t*, CUdeviceptr);

GetRange get_range_fn() {
  static GetRange fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* f = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuMemGetAddressRange", &f, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<GetRange>(f);
  });
  return fn;
}

struct Mapping {
  void* base;
  int refs;
};
std::mutex g_ipc_mu;
std::map<std::string, Mapping> g_by_handle;   // handle bytes -> mapping

}  // namespace

cudaError_t launch_gather_fold(const LaunchCtx& c, const float* const* parts, int p,
                               const float* b2, float* const* outs, int n_out, int64_t row0,
                               int64_t rows, int64_t d) {
  GatherPtrs g{};
  bool aligned = d % 4 == 0 && (b2 == nullptr || al16(b2));
  for (int j = 0; j < p; ++j) {
    g.part[j] = parts[j];
    aligned = aligned && al16(parts[j]);
  }
  for (int q = 0; q < n_out; ++q) {
    g.out[q] = outs[q];
    aligned = aligned && al16(outs[q]);
  }
  const int threads = 256;
  const int64_t cap = static_cast<int64_t>(c.num_sms) * 8;
  cudaError_t e = cudaSuccess;
  if (aligned) {
    const int64_t n4 = rows * d / 4, off4 = row0 * d / 4, d4 = d / 4;
    int64_t blocks = (n4 + threads - 1) / threads;
    if (blocks > cap) blocks = cap;
    const dim3 gr(static_cast<unsigned>(blocks)), bl(threads);
    switch (p) {
      case 1: gather_fold_vec_kernel<1><<<gr, bl, 0, c.stream>>>(g, p, n_out, b2, off4, n4, d4); break;
      case 2: gather_fold_vec_kernel<2><<<gr, bl, 0, c.stream>>>(g, p, n_out, b2, off4, n4, d4); break;
      case 4: gather_fold_vec_kernel<4><<<gr, bl, 0, c.stream>>>(g, p, n_out, b2, off4, n4, d4); break;
      case 8: gather_fold_vec_kernel<8><<<gr, bl, 0, c.stream>>>(g, p, n_out, b2, off4, n4, d4); break;
      default: gather_fold_vec_kernel<0><<<gr, bl, 0, c.stream>>>(g, p, n_out, b2, off4, n4, d4); break;
    }
  } else {
    const int64_t n = rows * d, off = row0 * d;
    int64_t blocks = (n + threads - 1) / threads;
    if (blocks > cap) blocks = cap;
    gather_fold_scalar_kernel<<<static_cast<unsigned>(blocks), threads, 0, c.stream>>>(
        g, p, n_out, b2, off, n, d);
  }
  e = cudaGetLastError();
  note_launch();
  return e;
}

tp_status ipc_export(const void* ptr, tp_ipc_handle* h) {
  GetRange range = get_range_fn();
  if (range == nullptr) {
    set_error_detail("cuMemGetAddressRange is not available");
    return TP_ERR_CUDA;
  }
  CUdeviceptr base = 0;
  size_t size = 0;
  if (range(&base, &size, reinterpret_cast<CUdeviceptr>(ptr)) != CUDA_SUCCESS) {
    set_error_detail("cuMemGetAddressRange failed: not a device allocation");
    return TP_ERR_INVALID_ARG;
  }
  cudaIpcMemHandle_t mh;
  const cudaError_t e = cudaIpcGetMemHandle(&mh, reinterpret_cast<void*>(base));
  if (e != cudaSuccess) {
    set_error_detail("cudaIpcGetMemHandle: %s (the buffer must come from cudaMalloc)",
                     cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  static_assert(sizeof(mh) <= sizeof(h->bytes), "IPC handle size");
  std::memset(h, 0, sizeof(*h));
  std::memcpy(h->bytes, &mh, sizeof(mh));
  h->offset = static_cast<uint64_t>(reinterpret_cast<uintptr_t>(ptr) - base);
  h->size = static_cast<uint64_t>(size);
  return TP_OK;
}

tp_status ipc_import(const tp_ipc_handle* h, void** ptr) {
  const std::string key(reinterpret_cast<const char*>(h->bytes), sizeof(cudaIpcMemHandle_t));
  std::lock_guard<std::mutex> lk(g_ipc_mu);
  auto it = g_by_handle.find(key);
  if (it == g_by_handle.end()) {
    cudaIpcMemHandle_t mh;
    std::memcpy(&mh, h->bytes, sizeof(mh));
    void* base = nullptr;
    const cudaError_t e = cudaIpcOpenMemHandle(&base, mh, cudaIpcMemLazyEnablePeerAccess);
    if (e != cudaSuccess) {
      set_error_detail("cudaIpcOpenMemHandle: %s", cudaGetErrorString(e));
      return TP_ERR_CUDA;
    }
    it = g_by_handle.emplace(key, Mapping{base, 0}).first;
  }
  ++it->second.refs;
  *ptr = static_cast<uint8_t*>(it->second.base) + h->offset;
  return TP_OK;
}

tp_status ipc_release(const tp_ipc_handle* h) {
  const std::string key(reinterpret_cast<const char*>(h->bytes), sizeof(cudaIpcMemHandle_t));
  std::lock_guard<std::mutex> lk(g_ipc_mu);
  auto it = g_by_handle.find(key);
  if (it == g_by_handle.end()) {
    set_error_detail("this handle is not imported");
    return TP_ERR_INVALID_ARG;
  }
  if (--it->second.refs > 0) return TP_OK;
  void* base = it->second.base;
  g_by_handle.erase(it);
  const cudaError_t e = cudaIpcCloseMemHandle(base);
  if (e != cudaSuccess) {
    set_error_detail("cudaIpcCloseMemHandle: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

}  // namespace tpk
