// fp32 path of the block (TF32 off): plain fp32 FMA on the CUDA cores.
// Used for the fp32 configurations (the day-41 walkthrough's own shape,
// X[4,512] x W[512,2048], p = 4), where a tensor-core tile would be >95%
// padding and fp32 accuracy (1e-5) is required.
//
// One 64x64 output tile per block of 256 threads; each thread owns a 4x4
// strided sub-tile and sums k in ascending order with fmaf, so the result
// is deterministic.  Very few rows take the skinny kernel below.
#include <cuda_runtime.h>

#include <cstdint>

#include "tp_act.cuh"
#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

constexpr int TM = 64, TN = 64, TK = 16;

enum SimtKind : int { kCol = 0, kColSwiglu = 1, kRowPartial = 2, kRowSplitK = 3 };

struct SimtArgs {
  const float* A;    // X (column) or Y [p][T][s] (row)
  const float* B0;   // W1 / W_gate (column) or W2 (row)
  const float* B1;   // W_up (SwiGLU)
  const float* bias; // b1 (column) or b2 (row split-K); may be null
  float* out;        // Y [p][T][s], P [p][T][d] or Z [T][d]
  int64_t M, N, K;   // output rows, output cols, reduction length
  int64_t lda;       // row pitch of A (d or s)
  int64_t ldb;       // row pitch of B (k or d)
  int64_t s;         // shard width
  int act;
};

template <int KIND>
__device__ __forceinline__ float load_a(const SimtArgs& a, int64_t batch, int64_t r, int64_t kk) {
  if (r >= a.M || kk >= a.K) return 0.0f;
  if constexpr (KIND == kCol || KIND == kColSwiglu) {
    return a.A[r * a.lda + kk];
  } else if constexpr (KIND == kRowPartial) {
    return a.A[(batch * a.M + r) * a.s + kk];
  } else {  // split-K over shards: hidden column kk lives in shard kk / s
    const int64_t i = kk / a.s, j = kk - i * a.s;
    return a.A[(i * a.M + r) * a.s + j];
  }
}

template <int KIND>
__device__ __forceinline__ float load_b(const float* B, const SimtArgs& a, int64_t batch,
                                        int64_t kk, int64_t c) {
  if (kk >= a.K || c >= a.N) return 0.0f;
  if constexpr (KIND == kRowPartial) {
    return B[(batch * a.s + kk) * a.ldb + c];  // shard i's rows of W2
  } else {
    return B[kk * a.ldb + c];
  }
}

template <int KIND>
__global__ void __launch_bounds__(256) simt_gemm_kernel(SimtArgs a) {
  constexpr bool kTwo = (KIND == kColSwiglu);
  __shared__ float As[TK][TM + 1];
  __shared__ float Bs[TK][TN];
  __shared__ float Us[kTwo ? TK : 1][kTwo ? TN : 1];

  const int tid = threadIdx.x;
  const int tx = tid % 16, ty = tid / 16;
  const int64_t m0 = static_cast<int64_t>(blockIdx.y) * TM;
  const int64_t n0 = static_cast<int64_t>(blockIdx.x) * TN;
  const int64_t batch = blockIdx.z;
  pdl_wait();
  pdl_launch_dependents();

  float acc[4][4], accu[4][4];
#pragma unroll
  for (int i = 0; i < 4; ++i)
#pragma unroll
    for (int j = 0; j < 4; ++j) acc[i][j] = accu[i][j] = 0.0f;

  for (int64_t k0 = 0; k0 < a.K; k0 += TK) {
#pragma unroll
    for (int q = 0; q < 4; ++q) {
      const int e = tid + 256 * q;
      const int ar = e / TK, ak = e % TK;
      As[ak][ar] = load_a<KIND>(a, batch, m0 + ar, k0 + ak);
      const int bk = e / TN, bc = e % TN;
      Bs[bk][bc] = load_b<KIND>(a.B0, a, batch, k0 + bk, n0 + bc);
      if constexpr (kTwo) Us[bk][bc] = load_b<KIND>(a.B1, a, batch, k0 + bk, n0 + bc);
    }
    __syncthreads();
#pragma unroll
    for (int kk = 0; kk < TK; ++kk) {
      float av[4], bv[4];
#pragma unroll
      for (int i = 0; i < 4; ++i) av[i] = As[kk][ty + 16 * i];
#pragma unroll
      for (int j = 0; j < 4; ++j) bv[j] = Bs[kk][tx + 16 * j];
#pragma unroll
      for (int i = 0; i < 4; ++i)
#pragma unroll
        for (int j = 0; j < 4; ++j) acc[i][j] = fmaf(av[i], bv[j], acc[i][j]);
      if constexpr (kTwo) {
#pragma unroll
        for (int j = 0; j < 4; ++j) bv[j] = Us[kk][tx + 16 * j];
#pragma unroll
        for (int i = 0; i < 4; ++i)
#pragma unroll
          for (int j = 0; j < 4; ++j) accu[i][j] = fmaf(av[i], bv[j], accu[i][j]);
      }
    }
    __syncthreads();
  }

#pragma unroll
  for (int i = 0; i < 4; ++i) {
    const int64_t r = m0 + ty + 16 * i;
    if (r >= a.M) continue;
#pragma unroll
    for (int j = 0; j < 4; ++j) {
      const int64_t c = n0 + tx + 16 * j;
      if (c >= a.N) continue;
      float v = acc[i][j];
      if constexpr (KIND == kCol || KIND == kColSwiglu) {
        if (a.bias != nullptr) v = v + a.bias[c];
        if constexpr (kTwo) {
          v = silu_f32(v) * accu[i][j];
        } else {
          v = act_unary(a.act, v);
        }
        const int64_t shard = c / a.s, cc = c - shard * a.s;
        a.out[(shard * a.M + r) * a.s + cc] = v;
      } else if constexpr (KIND == kRowPartial) {
        a.out[(batch * a.M + r) * a.N + c] = v;
      } else {
        if (a.bias != nullptr) v = __fadd_rn(v, a.bias[c]);
        a.out[r * a.N + c] = v;
      }
    }
  }
}

// Few rows (T <= 32, e.g. the day-41 walkthrough's X[4,512]): a 64x64 tile
// would be mostly padding and its k loop pays one memory latency per step.
// Instead a block owns 32 output columns (one per lane) and splits k across
// its 8 warps, each streaming its k range with many weight loads in flight;
// the 8 warp sums are then added in warp order, so the result is
// deterministic.
constexpr int kSkinnyRows = 8;

template <int KIND>
__global__ void __launch_bounds__(256) skinny_f32_kernel(SimtArgs a) {
  constexpr bool kTwo = (KIND == kColSwiglu);
  __shared__ float part[8][kSkinnyRows][33];
  __shared__ float partu[kTwo ? 8 : 1][kTwo ? kSkinnyRows : 1][33];
  const int lane = threadIdx.x % 32, w = threadIdx.x / 32;
  const int64_t c = static_cast<int64_t>(blockIdx.x) * 32 + lane;
  const int64_t batch = blockIdx.z;
  pdl_wait();
  pdl_launch_dependents();
  const int64_t kchunk = (a.K + 7) / 8;
  const int64_t k0 = w * kchunk;
  const int64_t k1 = k0 + kchunk < a.K ? k0 + kchunk : a.K;
  for (int64_t r0 = 0; r0 < a.M; r0 += kSkinnyRows) {
    float acc[kSkinnyRows], accu[kSkinnyRows];
#pragma unroll
    for (int r = 0; r < kSkinnyRows; ++r) acc[r] = accu[r] = 0.0f;
    if (c < a.N) {
#pragma unroll 8
      for (int64_t kk = k0; kk < k1; ++kk) {
        const float b = load_b<KIND>(a.B0, a, batch, kk, c);
        float u = 0.0f;
        if constexpr (kTwo) u = load_b<KIND>(a.B1, a, batch, kk, c);
#pragma unroll
        for (int r = 0; r < kSkinnyRows; ++r) {
          const float x = load_a<KIND>(a, batch, r0 + r, kk);
          acc[r] = fmaf(x, b, acc[r]);
          if constexpr (kTwo) accu[r] = fmaf(x, u, accu[r]);
        }
      }
    }
#pragma unroll
    for (int r = 0; r < kSkinnyRows; ++r) {
      part[w][r][lane] = acc[r];
      if constexpr (kTwo) partu[w][r][lane] = accu[r];
    }
    __syncthreads();
    {
      const int r = threadIdx.x / 32;   // 8 rows x 32 columns, one per thread
      const int64_t row = r0 + r;
      if (row < a.M && c < a.N) {
        float v = part[0][r][lane], vu = 0.0f;
        if constexpr (kTwo) vu = partu[0][r][lane];
#pragma unroll
        for (int q = 1; q < 8; ++q) {
          v += part[q][r][lane];
          if constexpr (kTwo) vu += partu[q][r][lane];
        }
        if constexpr (KIND == kCol || KIND == kColSwiglu) {
          if (a.bias != nullptr) v = v + a.bias[c];
          if constexpr (kTwo) {
            v = silu_f32(v) * vu;
          } else {
            v = act_unary(a.act, v);
          }
          const int64_t shard = c / a.s, cc = c - shard * a.s;
          a.out[(shard * a.M + row) * a.s + cc] = v;
        } else if constexpr (KIND == kRowPartial) {
          a.out[(batch * a.M + row) * a.N + c] = v;
        } else {
          if (a.bias != nullptr) v = __fadd_rn(v, a.bias[c]);
          a.out[row * a.N + c] = v;
        }
      }
    }
    __syncthreads();
  }
}

template <int KIND>
cudaError_t run(const LaunchCtx& c, const SimtArgs& a, int64_t batches) {
  cudaError_t e;
  if (a.M <= 32) {
    dim3 grid(static_cast<unsigned>((a.N + 31) / 32), 1, static_cast<unsigned>(batches));
    e = launch_pdl(skinny_f32_kernel<KIND>, grid, dim3(256), 0, c.stream, a);
  } else {
    dim3 grid(static_cast<unsigned>((a.N + TN - 1) / TN), static_cast<unsigned>((a.M + TM - 1) / TM),
              static_cast<unsigned>(batches));
    e = launch_pdl(simt_gemm_kernel<KIND>, grid, dim3(256), 0, c.stream, a);
  }
  note_launch();
  return e;
}

}  // namespace

cudaError_t launch_simt_column(const LaunchCtx& c, const float* X, const float* W1,
                               const float* Wup, const float* b1, float* Y, int64_t T, int64_t d,
                               int64_t k, int p, int act) {
  SimtArgs a{X, W1, Wup, b1, Y, T, k, d, d, k, k / p, act};
  if (act == kActSwiglu) return run<kColSwiglu>(c, a, 1);
  return run<kCol>(c, a, 1);
}

cudaError_t launch_simt_row(const LaunchCtx& c, const float* Y, const float* W2, float* P,
                            int64_t T, int64_t k, int64_t d, int p) {
  const int64_t s = k / p;
  SimtArgs a{Y, W2, nullptr, nullptr, P, T, d, s, s, d, s, kActIdentity};
  return run<kRowPartial>(c, a, p);
}

cudaError_t launch_simt_row_splitk(const LaunchCtx& c, const float* Y, const float* W2,
                                   const float* b2, float* Z, int64_t T, int64_t k, int64_t d,
                                   int p) {
  const int64_t s = k / p;
  SimtArgs a{Y, W2, nullptr, b2, Z, T, d, k, s, d, s, kActIdentity};
  return run<kRowSplitK>(c, a, 1);
}

}  // namespace tpk
