// The sum of partials that stands in for the all-reduce on one device:
//   Z = ((P_0 + P_1) + ...) + P_{p-1}  [+ b2]
// (day-41 post on tensor parallelism, "Simulating row parallel linear":
// sum(partial_sums) + bias).  One thread owns a 4-element column group of
// one row and folds the p shards into it in index order, so vector width and
// grid shape never change the order of any addition: the result is
// bit-reproducible.  Pure HBM streaming: (p + 1) * T * d * 4 bytes.
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

__device__ __forceinline__ float4 ld_stream(const float4* p) { return __ldcs(p); }

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  // __fadd_rn: one IEEE round-to-nearest-even add, never contracted.
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                     __fadd_rn(a.w, b.w));
}

// Vector path: T*d % 4 == 0, d % 4 == 0, 16-byte aligned P and Z.
template <int P>
__global__ void __launch_bounds__(256) reduce_vec_kernel(const float4* __restrict__ part,
                                                         const float* __restrict__ b2,
                                                         float4* __restrict__ Z, int64_t n4,
                                                         int64_t d4, int p_runtime) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n4;
       i += stride) {
    float4 acc;
    if constexpr (P > 0) {
      float4 v[P];
#pragma unroll
      for (int s = 0; s < P; ++s) v[s] = ld_stream(part + s * n4 + i);
      acc = v[0];
#pragma unroll
      for (int s = 1; s < P; ++s) acc = add4(acc, v[s]);
    } else {
      acc = ld_stream(part + i);
      for (int s = 1; s < p_runtime; ++s) acc = add4(acc, ld_stream(part + s * n4 + i));
    }
    if (b2 != nullptr) {
      const float4 b = __ldg(reinterpret_cast<const float4*>(b2) + (i % d4));
      acc = add4(acc, b);
    }
    __stcs(Z + i, acc);
  }
}

// Scalar path for any size / alignment.
__global__ void __launch_bounds__(256) reduce_scalar_kernel(const float* __restrict__ part,
                                                            const float* __restrict__ b2,
                                                            float* __restrict__ Z, int64_t n,
                                                            int64_t d, int p) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t stride = static_cast<int64_t>(gridDim.x) * blockDim.x;
  for (int64_t i = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x; i < n;
       i += stride) {
    float acc = part[i];
    for (int s = 1; s < p; ++s) acc = __fadd_rn(acc, part[s * n + i]);
    if (b2 != nullptr) acc = __fadd_rn(acc, b2[i % d]);
    Z[i] = acc;
  }
}

// The same fold, region by region, while the row layer is still running:
// launched right behind it (programmatic dependent launch, so its CTAs
// become resident beside the row layer's as soon as those have started),
// each CTA takes regions in the order the row layer finishes their tiles,
// waits (bounded) until the region's counter shows every shard's tile in
// memory, and folds it (then b2, then the residual R if given: the order of
// the row-wise fold with residual).  It has no griddepcontrol.wait: the
// counters, a release per producer and an acquire here, order it after the
// stores it reads, and the row layer itself ran after everything before it
// (R included).  Vector path only (d % 4 == 0, 16-byte aligned P, Z, b2, R).
struct RegionArgs {
  const float4* part;
  const float* b2;
  const float4* R;     // residual added last, or null
  float4* Z;
  const int* cnt;
  int64_t T, d4, n4;   // rows, float4 per row, float4 per shard
  int32_t rows, cols4, m_regions, n_regions, target, m_group;
  WaitCtl wait;
};

// The r-th region in the order the row layer completes them: group by
// group of m_group m-regions, within a group n slowest, m fastest.  Returns
// the region's counter index n * m_regions + m.
__device__ __forceinline__ int32_t region_in_order(const RegionArgs& a, int32_t r, int32_t& m,
                                                   int32_t& n) {
  const int32_t mg_full = a.m_group > 0 ? a.m_group : a.m_regions;
  const int32_t g = r / (mg_full * a.n_regions);
  const int32_t m0 = g * mg_full;
  const int32_t mg = a.m_regions - m0 < mg_full ? a.m_regions - m0 : mg_full;
  const int32_t q = r - g * mg_full * a.n_regions;
  n = q / mg;
  m = m0 + q - n * mg;
  return n * a.m_regions + m;
}

__device__ __forceinline__ bool wait_region(const int* cnt, int target, const WaitCtl& w) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (ld_acquire_gpu(cnt) < target) {
    if (globaltimer_ns() - t0 > w.timeout_ns) {
      atomicOr(w.err, kErrWaitRegion);
      return false;
    }
    __nanosleep(500);
  }
  return true;
}

// 512 threads (16 warps of at most 64 registers: 32K registers) fit beside
// a row-layer CTA (12 warps); 1024 would not.
constexpr int kFoldThreads = 512;
// Work unit: a quarter of a region's rows (64 of 256), so that the units
// spread evenly over the CTAs and a region that completes is folded by
// several CTAs at once.
constexpr int kUnitsPerRegion = 4;

template <int P>
__global__ void __launch_bounds__(kFoldThreads, 2) fold_regions_kernel(const RegionArgs a, int p_runtime) {
  pdl_launch_dependents();
  __shared__ int s_ok;
  const int32_t units = a.m_regions * a.n_regions * kUnitsPerRegion;
  const int32_t sub = a.rows / kUnitsPerRegion;
  for (int32_t u = blockIdx.x; u < units; u += gridDim.x) {
    const int32_t r = u / kUnitsPerRegion, q = u - r * kUnitsPerRegion;
    int32_t m, n;
    const int32_t ci = region_in_order(a, r, m, n);
    if (threadIdx.x == 0) s_ok = wait_region(a.cnt + ci, a.target, a.wait) ? 1 : 0;
    __syncthreads();
    if (!s_ok) return;   // block-uniform
    const int64_t r0 = static_cast<int64_t>(m) * a.rows + static_cast<int64_t>(q) * sub;
    const int64_t nrows = a.T - r0 < sub ? a.T - r0 : sub;   // may be <= 0 at the ragged end
    const int64_t c0 = static_cast<int64_t>(n) * a.cols4;
    const int32_t w4 = static_cast<int32_t>(a.d4 - c0 < a.cols4 ? a.d4 - c0 : a.cols4);
    const int64_t count = nrows > 0 ? nrows * w4 : 0;
    for (int64_t e = threadIdx.x; e < count; e += blockDim.x) {
      const int64_t row = r0 + e / w4;
      const int64_t col = c0 + e % w4;
      const int64_t i = row * a.d4 + col;
      float4 acc;
      if constexpr (P > 0) {
        float4 v[P];
#pragma unroll
        for (int s = 0; s < P; ++s) v[s] = ld_stream(a.part + s * a.n4 + i);
        acc = v[0];
#pragma unroll
        for (int s = 1; s < P; ++s) acc = add4(acc, v[s]);
      } else {
        acc = ld_stream(a.part + i);
        for (int s = 1; s < p_runtime; ++s) acc = add4(acc, ld_stream(a.part + s * a.n4 + i));
      }
      if (a.b2 != nullptr) acc = add4(acc, __ldg(reinterpret_cast<const float4*>(a.b2) + col));
      if (a.R != nullptr) acc = add4(acc, ld_stream(a.R + i));
      __stcs(a.Z + i, acc);
    }
    __syncthreads();   // s_ok is rewritten for the next unit
  }
}

}  // namespace

cudaError_t launch_fold_regions(const LaunchCtx& c, const float* P, const float* b2, float* Z,
                                int64_t T, int64_t d, int p, const RegionFold& rf, const float* R) {
  if (T == 0) return cudaSuccess;
  RegionArgs a{};
  a.part = reinterpret_cast<const float4*>(P);
  a.b2 = b2;
  a.R = reinterpret_cast<const float4*>(R);
  a.Z = reinterpret_cast<float4*>(Z);
  a.cnt = rf.cnt;
  a.T = T;
  a.d4 = d / 4;
  a.n4 = T * d / 4;
  a.rows = rf.rows;
  a.cols4 = rf.cols / 4;
  a.m_regions = rf.m_regions;
  a.n_regions = rf.n_regions;
  a.target = rf.target;
  a.m_group = rf.m_group;
  a.wait.err = c.err_word;
  a.wait.timeout_ns = c.timeout_ns;
  // One CTA per SM at most: beside a row-layer CTA only one more CTA fits
  // (shared memory, registers), and the carve-out must match the row
  // layer's for the two to share an SM.
  int blocks = rf.m_regions * rf.n_regions * kUnitsPerRegion;
  if (blocks > c.num_sms) blocks = c.num_sms;
  static uint64_t attr_epoch[64] = {};
  static std::mutex mu;
  auto kern = p == 2 ? fold_regions_kernel<2>
            : p == 4 ? fold_regions_kernel<4>
            : p == 8 ? fold_regions_kernel<8>
                     : fold_regions_kernel<0>;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      for (auto k : {fold_regions_kernel<0>, fold_regions_kernel<2>, fold_regions_kernel<4>,
                     fold_regions_kernel<8>}) {
        const cudaError_t e = cudaFuncSetAttribute(
            k, cudaFuncAttributePreferredSharedMemoryCarveout, cudaSharedmemCarveoutMaxShared);
        if (e != cudaSuccess) return e;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  const cudaError_t e =
      launch_pdl(kern, dim3(static_cast<unsigned>(blocks)), dim3(kFoldThreads), 0, c.stream, a, p);
  note_launch();
  return e;
}

cudaError_t launch_reduce(const LaunchCtx& c, const float* P, const float* b2, float* Z, int64_t T,
                          int64_t d, int p) {
  const int64_t n = T * d;
  if (n == 0) return cudaSuccess;
  const bool aligned = (reinterpret_cast<uintptr_t>(P) % 16 == 0) &&
                       (reinterpret_cast<uintptr_t>(Z) % 16 == 0) &&
                       (b2 == nullptr || reinterpret_cast<uintptr_t>(b2) % 16 == 0);
  const int threads = 256;
  cudaError_t e = cudaSuccess;
  if (aligned && d % 4 == 0) {
    const int64_t n4 = n / 4;
    // Enough resident threads to keep ~p loads in flight per thread on every
    // SM; grid-stride beyond that.
    int64_t blocks = (n4 + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(c.num_sms) * 8;
    if (blocks > cap) blocks = cap;
    const float4* P4 = reinterpret_cast<const float4*>(P);
    float4* Z4 = reinterpret_cast<float4*>(Z);
    const int64_t d4 = d / 4;
    dim3 g(static_cast<unsigned>(blocks));
    switch (p) {
      case 1: e = launch_pdl(reduce_vec_kernel<1>, g, dim3(threads), 0, c.stream, P4, b2, Z4, n4, d4, p); break;
      case 2: e = launch_pdl(reduce_vec_kernel<2>, g, dim3(threads), 0, c.stream, P4, b2, Z4, n4, d4, p); break;
      case 3: e = launch_pdl(reduce_vec_kernel<3>, g, dim3(threads), 0, c.stream, P4, b2, Z4, n4, d4, p); break;
      case 4: e = launch_pdl(reduce_vec_kernel<4>, g, dim3(threads), 0, c.stream, P4, b2, Z4, n4, d4, p); break;
      case 8: e = launch_pdl(reduce_vec_kernel<8>, g, dim3(threads), 0, c.stream, P4, b2, Z4, n4, d4, p); break;
      default: e = launch_pdl(reduce_vec_kernel<0>, g, dim3(threads), 0, c.stream, P4, b2, Z4, n4, d4, p); break;
    }
  } else {
    int64_t blocks = (n + threads - 1) / threads;
    const int64_t cap = static_cast<int64_t>(c.num_sms) * 8;
    if (blocks > cap) blocks = cap;
    e = launch_pdl(reduce_scalar_kernel, dim3(static_cast<unsigned>(blocks)), dim3(threads), 0,
                   c.stream, P, b2, Z, n, d, p);
  }
  note_launch();
  return e;
}

}  // namespace tpk
