// Kernel launch with programmatic dependent launch allowed: the kernel may
// start while the previous kernel in the stream finishes; every kernel of
// this library calls griddepcontrol.wait before its first global memory
// access, so the overlap only covers launch latency and prologues.
// Setting TP_DISABLE_PDL=1 in the environment launches them plainly.
#pragma once

#include <cuda_runtime.h>

#include <cstdlib>

namespace tpk {

inline bool pdl_allowed() {
  static const bool on = [] {
    const char* e = std::getenv("TP_DISABLE_PDL");
    return !(e != nullptr && e[0] == '1');
  }();
  return on;
}

// CTA-pair (cta_group::2) GEMMs for wide tiles; TP_DISABLE_PAIR=1 keeps the
// one-CTA kernel (for comparisons).
inline bool pair_allowed() {
  static const bool on = [] {
    const char* e = std::getenv("TP_DISABLE_PAIR");
    return !(e != nullptr && e[0] == '1');
  }();
  return on;
}

// tp_mlp_block's fold overlapped with its row layer (CTA-pair row tiles);
// TP_DISABLE_REGION_FOLD=1 folds after the row layer instead (for
// comparisons; same bits).
inline bool region_fold_allowed() {
  static const bool on = [] {
    const char* e = std::getenv("TP_DISABLE_REGION_FOLD");
    return !(e != nullptr && e[0] == '1');
  }();
  return on;
}

// TP_DISABLE_COOP=1 launches the folding row layer like the other layers
// (programmatic serialization, no co-residency guarantee): for profilers
// that cannot launch a cooperative cluster grid, and for comparisons.
inline bool coop_allowed() {
  static const bool on = [] {
    const char* e = std::getenv("TP_DISABLE_COOP");
    return !(e != nullptr && e[0] == '1');
  }();
  return on;
}

// TP_DISABLE_ROW_CHAIN=1 keeps the partials and the fold beside the row layer
// where the chain fold would run (for comparisons; same bits).
inline bool row_chain_allowed() {
  static const bool on = [] {
    const char* e = std::getenv("TP_DISABLE_ROW_CHAIN");
    return !(e != nullptr && e[0] == '1');
  }();
  return on;
}

template <typename... KArgs, typename... Args>
cudaError_t launch_pdl(void (*kernel)(KArgs...), dim3 grid, dim3 block, size_t smem,
                       cudaStream_t stream, Args&&... args) {
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = grid;
  cfg.blockDim = block;
  cfg.dynamicSmemBytes = smem;
  cfg.stream = stream;
  cudaLaunchAttribute attr[1];
  attr[0].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[0].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_allowed() ? 1 : 0;
  return cudaLaunchKernelEx(&cfg, kernel, static_cast<Args&&>(args)...);
}

}  // namespace tpk
