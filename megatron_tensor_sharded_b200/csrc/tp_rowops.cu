// Row-wise steps of the tensor-parallel transformer block ("Building GPT from
// Scratch -- Part 9", "Communication Pattern per Transformer Block"):
//
//   H = ((P_0 + P_1) + ... + P_{p-1}) [+ b] [+ R]     the reduction that ends
//                                                      each block, with the
//                                                      residual add fused;
//   Y = LayerNorm(H) * gamma + beta  (bf16)           the next block's input.
//
// One CTA per row: the row's fold is done element by element in shard order
// (the same order as the vector reduction kernel, so the sum is bit-exact),
// the row stays in registers, and the LayerNorm statistics are two block
// reductions over it (mean, then the mean square of x - mean).  With p = 0
// and R = X the kernel is a plain LayerNorm of X.  Pure HBM streaming:
// (p + 1) * d * 4 bytes read (+ d * 4 written for H, + d * 2 for Y) per row.
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <atomic>
#include <cstdint>
#include <cstring>
#include <type_traits>

#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

constexpr int kThreads = 256;
constexpr int kMaxV = 16;   // float4 chunks per thread: d <= 16384

__device__ __forceinline__ float4 add4(float4 a, float4 b) {
  return make_float4(__fadd_rn(a.x, b.x), __fadd_rn(a.y, b.y), __fadd_rn(a.z, b.z),
                     __fadd_rn(a.w, b.w));
}

__device__ __forceinline__ float block_sum(float v, float* red) {
#pragma unroll
  for (int o = 16; o > 0; o >>= 1) v += __shfl_xor_sync(0xffffffffu, v, o);
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  __syncthreads();   // `red` may still be read from the previous reduction
  if (lane == 0) red[warp] = v;
  __syncthreads();
  float s = 0.0f;
#pragma unroll
  for (int w = 0; w < kThreads / 32; ++w) s += red[w];
  return s;
}

// FOLD = false is the plain LayerNorm of R (p == 0): no partial loads, so
// the instance needs fewer registers and more CTAs stay resident.
template <int NV, bool FOLD>
__global__ void __launch_bounds__(kThreads) row_fold_ln_kernel(
    const float* __restrict__ part, int p, int64_t part_stride, const float* __restrict__ bias,
    const float* R, float* H, const float* __restrict__ gamma, const float* __restrict__ beta,
    __nv_bfloat16* __restrict__ Y, int64_t T, int64_t d, float eps) {
  __shared__ float red[kThreads / 32];
  pdl_wait();
  pdl_launch_dependents();
  const int64_t d4 = d / 4;
  // persistent: a fixed grid of resident CTAs walks the rows
  for (int64_t row = blockIdx.x; row < T; row += gridDim.x) {
  const int64_t base = row * d;
  // The fold, shard by shard over the whole row: each shard's NV vectors are
  // loaded together (NV loads in flight per thread, not one), and every
  // element still takes its additions in shard order, then bias, then R.
  float4 h[NV];
  const float4* src = reinterpret_cast<const float4*>((FOLD ? part : R) + base);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int64_t c = threadIdx.x + static_cast<int64_t>(k) * kThreads;
    h[k] = c < d4 ? (FOLD ? __ldcs(src + c) : src[c]) : make_float4(0.f, 0.f, 0.f, 0.f);
  }
  if constexpr (FOLD) {
    for (int s = 1; s < p; ++s) {
      const float4* ps = reinterpret_cast<const float4*>(part + s * part_stride + base);
      float4 v[NV];
#pragma unroll
      for (int k = 0; k < NV; ++k) {
        const int64_t c = threadIdx.x + static_cast<int64_t>(k) * kThreads;
        if (c < d4) v[k] = __ldcs(ps + c);
      }
#pragma unroll
      for (int k = 0; k < NV; ++k)
        if (threadIdx.x + static_cast<int64_t>(k) * kThreads < d4) h[k] = add4(h[k], v[k]);
    }
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int64_t c = threadIdx.x + static_cast<int64_t>(k) * kThreads;
      if (c < d4) {
        if (bias != nullptr) h[k] = add4(h[k], __ldg(reinterpret_cast<const float4*>(bias) + c));
        if (R != nullptr) h[k] = add4(h[k], reinterpret_cast<const float4*>(R + base)[c]);
      }
    }
  }
  if (H != nullptr) {
#pragma unroll
    for (int k = 0; k < NV; ++k) {
      const int64_t c = threadIdx.x + static_cast<int64_t>(k) * kThreads;
      if (c < d4) reinterpret_cast<float4*>(H + base)[c] = h[k];
    }
  }
  if (Y == nullptr) continue;
  float s = 0.0f;
#pragma unroll
  for (int k = 0; k < NV; ++k) s += (h[k].x + h[k].y) + (h[k].z + h[k].w);
  const float mean = block_sum(s, red) / static_cast<float>(d);
  float q = 0.0f;
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int64_t c = threadIdx.x + static_cast<int64_t>(k) * kThreads;
    if (c < d4) {
      const float a = h[k].x - mean, b = h[k].y - mean, e = h[k].z - mean, f = h[k].w - mean;
      q += (a * a + b * b) + (e * e + f * f);
    }
  }
  const float var = block_sum(q, red) / static_cast<float>(d);
  const float rstd = rsqrtf(var + eps);
#pragma unroll
  for (int k = 0; k < NV; ++k) {
    const int64_t c = threadIdx.x + static_cast<int64_t>(k) * kThreads;
    if (c < d4) {
      const float4 g = __ldg(reinterpret_cast<const float4*>(gamma) + c);
      const float4 bt = __ldg(reinterpret_cast<const float4*>(beta) + c);
      const __nv_bfloat162 lo =
          __floats2bfloat162_rn((h[k].x - mean) * rstd * g.x + bt.x, (h[k].y - mean) * rstd * g.y + bt.y);
      const __nv_bfloat162 hi =
          __floats2bfloat162_rn((h[k].z - mean) * rstd * g.z + bt.z, (h[k].w - mean) * rstd * g.w + bt.w);
      uint2 u;
      memcpy(&u.x, &lo, 4);
      memcpy(&u.y, &hi, 4);
      reinterpret_cast<uint2*>(Y + base)[c] = u;
    }
  }
  }
}

// Column sums of bf16 matrices [batches][R][n] (bias gradients: db = sum over
// tokens), in two fixed-order passes so the result is reproducible: pass 1
// sums chunks of kChunkRows rows per column pair into fp32 partials
// [batches][chunks][n]; pass 2 adds the chunks in order.
constexpr int kChunkRows = 128;

__global__ void __launch_bounds__(128) colsum_partial_kernel(const __nv_bfloat16* __restrict__ A,
                                                             float* __restrict__ part, int64_t R,
                                                             int64_t n, int chunks) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t j = (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x) * 2;
  const int chunk = blockIdx.y;
  const int64_t b = blockIdx.z;
  if (j >= n) return;
  const int64_t r0 = static_cast<int64_t>(chunk) * kChunkRows;
  const int64_t r1 = r0 + kChunkRows < R ? r0 + kChunkRows : R;
  const __nv_bfloat16* src = A + b * R * n + j;
  float s0 = 0.0f, s1 = 0.0f;
  for (int64_t r = r0; r < r1; ++r) {
    const __nv_bfloat162 v = *reinterpret_cast<const __nv_bfloat162*>(src + r * n);
    s0 += __bfloat162float(v.x);
    s1 += __bfloat162float(v.y);
  }
  float* dst = part + (b * chunks + chunk) * n + j;
  dst[0] = s0;
  dst[1] = s1;
}

__global__ void __launch_bounds__(256) colsum_final_kernel(const float* __restrict__ part,
                                                           float* __restrict__ out, int64_t n,
                                                           int chunks, int64_t out_batch_stride) {
  pdl_wait();
  pdl_launch_dependents();
  const int64_t j = static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x;
  const int64_t b = blockIdx.y;
  if (j >= n) return;
  float s = 0.0f;
  for (int c = 0; c < chunks; ++c) s += part[(b * chunks + c) * n + j];
  out[b * out_batch_stride + j] = s;
}

}  // namespace

// out[b * out_batch_stride + j] = sum_r A[b][r][j]; `scratch` holds
// batches * ceil(R / 128) * n floats.  n even.
cudaError_t launch_colsum(const LaunchCtx& c, const void* A, float* out, float* scratch,
                          int64_t batches, int64_t R, int64_t n, int64_t out_batch_stride) {
  if (batches == 0 || n == 0) return cudaSuccess;
  const int chunks = static_cast<int>((R + kChunkRows - 1) / kChunkRows);
  if (chunks == 0) {
    cudaError_t e = cudaSuccess;
    for (int64_t b = 0; b < batches && e == cudaSuccess; ++b)
      e = cudaMemsetAsync(out + b * out_batch_stride, 0, n * sizeof(float), c.stream);
    return e;
  }
  const dim3 g1(static_cast<unsigned>((n / 2 + 127) / 128), static_cast<unsigned>(chunks),
                static_cast<unsigned>(batches));
  cudaError_t e = launch_pdl(colsum_partial_kernel, g1, dim3(128), 0, c.stream,
                             static_cast<const __nv_bfloat16*>(A), scratch, R, n, chunks);
  note_launch();
  if (e != cudaSuccess) return e;
  const dim3 g2(static_cast<unsigned>((n + 255) / 256), static_cast<unsigned>(batches));
  e = launch_pdl(colsum_final_kernel, g2, dim3(256), 0, c.stream,
                 static_cast<const float*>(scratch), out, n, chunks, out_batch_stride);
  note_launch();
  return e;
}

// H = fold(P) [+ bias] [+ R] (written when H != nullptr); Y = LN(H) (when
// Y != nullptr).  p == 0: H = R.  Requires d % 4 == 0, d <= 16384 and
// 16-byte aligned rows (checked by the caller).
cudaError_t launch_row_fold_ln(const LaunchCtx& c, const float* P, int p, const float* bias,
                               const float* R, float* H, const float* gamma, const float* beta,
                               void* Y, int64_t T, int64_t d, float eps) {
  if (T == 0) return cudaSuccess;
  const int64_t d4 = d / 4;
  const int nv = static_cast<int>((d4 + kThreads - 1) / kThreads);
  __nv_bfloat16* y = static_cast<__nv_bfloat16*>(Y);
  const int64_t ps = T * d;
  // a persistent grid: as many CTAs as fit on the SMs at once (by the
  // kernel's register use), each walking rows blockIdx.x, + gridDim.x, ...
  // Residency is looked up once per instantiation: every instantiation has
  // the same function type, so each gets its own slot (index `slot`).
  static std::atomic<int> per_sm_cache[10];
  auto go = [&](auto kern, int slot) {
    int per_sm = per_sm_cache[slot].load(std::memory_order_relaxed);
    if (per_sm == 0) {
      if (cudaOccupancyMaxActiveBlocksPerMultiprocessor(&per_sm, kern, kThreads, 0) != cudaSuccess ||
          per_sm < 1)
        per_sm = 1;
      per_sm_cache[slot].store(per_sm, std::memory_order_relaxed);
    }
    const int64_t resident = static_cast<int64_t>(c.num_sms) * per_sm;
    const dim3 g(static_cast<unsigned>(T < resident ? T : resident)), b(kThreads);
    return launch_pdl(kern, g, b, 0, c.stream, P, p, ps, bias, R, H, gamma, beta, y, T, d, eps);
  };
  auto pick = [&](auto fold) {
    constexpr bool F = decltype(fold)::value;
    constexpr int f = F ? 5 : 0;
    if (nv <= 1) return go(row_fold_ln_kernel<1, F>, f + 0);
    if (nv <= 2) return go(row_fold_ln_kernel<2, F>, f + 1);
    if (nv <= 4) return go(row_fold_ln_kernel<4, F>, f + 2);
    if (nv <= 8) return go(row_fold_ln_kernel<8, F>, f + 3);
    return go(row_fold_ln_kernel<kMaxV, F>, f + 4);
  };
  const cudaError_t e = p > 0 ? pick(std::true_type{}) : pick(std::false_type{});
  note_launch();
  return e;
}

}  // namespace tpk
