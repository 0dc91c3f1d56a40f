// tp_mlp_block_noalloc: the whole block for callers that cannot allocate
// device memory.
//
// Some callers have no way to obtain a device workspace: a plugin inside a
// host framework that owns the whole device memory pool and forbids other
// allocations, or a latency-critical loop where cudaMalloc's implicit device
// synchronisation is not acceptable.  This entry point takes the block's
// scratch (hidden shards, then fp32 partials) from one fixed array in device
// global memory that lives in this library, so the caller passes only inputs
// and outputs and nothing is allocated per call.
//
// Costs and limits:
//   - every GPU that loads the library holds kNoAllocScratchBytes (16 MiB)
//     until the process exits;
//   - a problem whose scratch exceeds that is rejected (TP_ERR_WORKSPACE);
//   - all calls share the one array: calls whose kernels overlap on the same
//     GPU (other streams, other host threads) overwrite each other's scratch.
//     Issue them on one stream, one after the other.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "tp_internal.h"
#include "tp_mlp.h"

namespace {

constexpr size_t kNoAllocScratchBytes = size_t(16) << 20;

// Device code could name this array directly; host code must not: on the
// host the name is only a stand-in, not a device address, and handing it to a
// kernel would fault (or silently touch the wrong memory where the GPU can
// reach host memory).  Host code uses the address cudaGetSymbolAddress
// returns for the current device.
static __device__ __align__(256) unsigned char g_noalloc_scratch[kNoAllocScratchBytes];

constexpr int kMaxDevices = 64;
void* g_scratch_addr[kMaxDevices] = {};
uint64_t g_scratch_epoch[kMaxDevices] = {};   // context epoch the address belongs to
std::mutex g_scratch_mu;

// Device address of the scratch array on the current device.  It is looked
// up with cudaGetSymbolAddress once per device, at the first call on that
// device (make that first call before any stream capture begins), and again
// only if the device has since been given a new CUDA context (after a device
// reset, say), whose copy of the array sits at a different address.
tp_status scratch_address(void** out) {
  int dev = 0;
  uint64_t epoch = 0;
  const tp_status st = tpk::current_device(&dev, &epoch);
  if (st != TP_OK) return st;
  std::lock_guard<std::mutex> lk(g_scratch_mu);
  if (g_scratch_addr[dev] == nullptr || g_scratch_epoch[dev] != epoch) {
    void* p = nullptr;
    const cudaError_t e = cudaGetSymbolAddress(&p, g_noalloc_scratch);
    if (e != cudaSuccess || p == nullptr) {
      tpk::set_error_detail("cudaGetSymbolAddress(scratch): %s", cudaGetErrorString(e));
      return TP_ERR_CUDA;
    }
    g_scratch_addr[dev] = p;
    g_scratch_epoch[dev] = epoch;
  }
  *out = g_scratch_addr[dev];
  return TP_OK;
}

}  // namespace

extern "C" {

tp_status tp_mlp_block_noalloc(const void* X, const void* W1, const void* W_up, const void* b1,
                               const void* W2, const float* b2, float* Z, int64_t T, int64_t d,
                               int64_t k, int p, tp_dtype dtype, tp_act act, int flags,
                               void* stream) {
  const size_t need = tp_mlp_block_workspace_size(T, d, k, p, dtype, act, flags);
  if (need > kNoAllocScratchBytes) {
    tpk::set_error_detail(
        "tp_mlp_block_noalloc: this problem needs %zu bytes of scratch; the static scratch holds "
        "%zu bytes (use tp_mlp_block with a caller workspace)",
        need, kNoAllocScratchBytes);
    return TP_ERR_WORKSPACE;
  }
  // need == 0 means invalid arguments or T == 0: tp_mlp_block reports which.
  void* scratch = nullptr;
  if (need > 0 && T > 0) {
    const tp_status st = scratch_address(&scratch);
    if (st != TP_OK) return st;
  }
  // Nothing in the scratch has to start at zero: every byte the kernels read
  // (hidden shards, partials) is written earlier in the same call.
  return tp_mlp_block(X, W1, W_up, b1, W2, b2, Z, scratch, need > 0 ? kNoAllocScratchBytes : 0, T,
                      d, k, p, dtype, act, flags, stream);
}

}  // extern "C"
