// The sum of partials that stands in for the all-reduce on one device:
//   Z = ((P_0 + P_1) + ...) + P_{p-1}  [+ b2]
// (day-41 post on tensor parallelism, "Simulating row parallel linear":
// sum(partial_sums) + bias).  One thread owns a 4-element column group of
// one row and folds the p shards into it in index order, so vector width and
// grid shape never change the order of any addition: the result is
// bit-reproducible.  Pure HBM streaming: (p + 1) * T * d * 4 bytes.
#include <cuda_runtime.h>

#include <cstdint>

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

}  // namespace

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
