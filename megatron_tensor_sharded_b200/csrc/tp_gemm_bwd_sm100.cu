// Backward pass of the sharded MLP block on sm_100a tensor cores.
//
// The f / g conjugate operators ("Tensor parallel math", "The f and g
// conjugate operators"): g after the row-parallel layer is the identity in
// the backward pass, so every shard takes the whole upstream gradient dZ;
// everything up to the column-parallel layer's input is local to the shard;
// f before the column-parallel layer is the all-reduce, here the sum of p
// full-shape input-gradient partials folded in shard order.
//
// Four batched GEMMs (batch = shard), one persistent warp-specialised kernel
// template with the operand layouts as parameters:
//
//   G1  dH_i = (dZ W2_i^T) * act'(H_i)   A = dZ [T x d] K-major,
//                                        B = W2_i (rows of W2) K-major;
//                                        epilogue reads H_i (and the up
//                                        projection for SwiGLU) and writes
//                                        dH_i (and dU_i), bf16 [p][T][s]
//   G2  dX_i = dH_i W1_i^T (+ dU_i Wup_i^T)   A = dH_i K-major, B = W1_i
//                                        (column block of W1) K-major; the
//                                        SwiGLU pair is one K loop over both
//                                        halves; fp32 partials [p][T][d]
//   G3  dW1_i = X^T dH_i                 A = X^T (M-major), B = dH_i
//                                        N-major; written into the column
//                                        block i of dW1 [d][k] (SwiGLU: a
//                                        second half of batches for dW_up)
//   G4  dW2_i = Y_i^T dZ                 A = Y_i^T (M-major), B = dZ
//                                        N-major; written into row block i
//                                        of dW2 [k][d]
//
// Every operand is a 3-D tensor map (inner, outer, batch) with the shard as
// the batch, except W1's column blocks, read from the whole [d][k] map at a
// K offset of s per shard (s is a multiple of 64, so no K block crosses into
// the next shard).  TMA zero-fills beyond each extent, so ragged M, N and K
// need no special code.  Roles as in the forward GEMM:
// warp 0 TMA, warp 1 MMA (two TMEM accumulators), warp 2 TMEM allocation,
// warps 4..11 epilogue; every wait bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstring>
#include <mutex>

#include "tp_gemm_parts.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

using namespace gemm;

constexpr int A_CHUNK_BYTES = BK * 64 * 2;   // M-major A: one 64-wide M atom column, 8 KiB

enum BwdEpi : int { kEpiF32 = 0, kEpiActGrad = 1, kEpiSwigluGrad = 2 };

struct GParams {
  int32_t M, N, K;              // per batch
  int32_t p, halves;            // batch b -> shard b % p, half b / p
  int32_t m_tiles, n_tiles, num_tiles, k_blocks, kb_half;  // kb_half > 0: K-concat of two sources
  int32_t a_batched, b_batched; // operand batch coordinate = shard (else 0)
  int32_t b_koff;               // K-major B: K coordinate offset per shard (W1's column blocks)
  int32_t act;
  int32_t bulk_out;             // fp32 epilogue through shared memory + TMA tensor stores
  int* region_cnt;              // fp32 partials on CTA pairs (bulk_out): per-tile completion
                                // counters [n_tiles][m_tiles] for the fold beside it; or null
  int32_t m_group;              // > 0: tiles walk groups of this many m-tiles, group slowest
  // epilogue
  void* out[2];                 // per half
  int64_t out_shard_stride;     // elements
  int64_t ldc;                  // elements
  const void* aux0;             // H (pre-activation / gate) bf16, same layout as out
  const void* aux1;             // up projection (SwiGLU)
  WaitCtl wait;
  int64_t debug_drop;
};

struct GTile {
  int32_t b, shard, half, m, n;
};

__device__ __forceinline__ GTile decode(const GParams& P, int32_t t) {
  // Within a group of m-tiles (all of them when m_group == 0): batch
  // slowest, then n, m fastest.  Every group but the last is full.
  const int32_t mg_full = P.m_group > 0 ? P.m_group : P.m_tiles;
  const int32_t batches = P.p * P.halves;
  const int32_t group_tiles = mg_full * P.n_tiles * batches;
  const int32_t grp = t / group_tiles;
  const int32_t m0 = grp * mg_full;
  const int32_t mg = P.m_tiles - m0 < mg_full ? P.m_tiles - m0 : mg_full;
  int32_t r = t - grp * group_tiles;
  GTile g;
  g.b = r / (mg * P.n_tiles);
  r -= g.b * mg * P.n_tiles;
  g.n = r / mg;
  g.m = m0 + r - g.n * mg;
  g.shard = g.b % P.p;
  g.half = g.b / P.p;
  return g;
}

template <int AMN, int BMN, int BN>
__device__ __forceinline__ void issue(const GParams& P, const CUtensorMap* mA0,
                                      const CUtensorMap* mA1, const CUtensorMap* mB0,
                                      const CUtensorMap* mB1, const GTile& g, int32_t kb,
                                      uint32_t sa, uint32_t sb, uint32_t bar) {
  // K-concat (kb_half > 0): the second half of the K loop reads the second
  // sources; halves > 1: the second half of the batches reads B1.
  bool second = false;
  if (P.kb_half > 0 && kb >= P.kb_half) {
    second = true;
    kb -= P.kb_half;
  }
  const CUtensorMap* mA = second ? mA1 : mA0;
  const CUtensorMap* mB = (second || g.half > 0) ? mB1 : mB0;
  const int32_t za = P.a_batched ? g.shard : 0;
  const int32_t zb = P.b_batched ? g.shard : 0;
  const int32_t m0 = g.m * BM, n0 = g.n * BN, k0 = kb * BK;
  if constexpr (AMN == 0) {
    tma_load_3d(sa, mA, bar, k0, m0, za);
  } else {
#pragma unroll
    for (int c = 0; c < BM / 64; ++c) tma_load_3d(sa + c * A_CHUNK_BYTES, mA, bar, m0 + c * 64, k0, za);
  }
  if constexpr (BMN == 0) {
    tma_load_3d(sb, mB, bar, k0 + g.shard * P.b_koff, n0, zb);
  } else {
#pragma unroll
    for (int c = 0; c < BN / 64; ++c) tma_load_3d(sb + c * B_CHUNK_BYTES, mB, bar, n0 + c * 64, k0, zb);
  }
}

__device__ __forceinline__ void store_bf16x8_at(__nv_bfloat16* dst, const float (&y)[8]) {
  const uint4 pk = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                              pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
  *reinterpret_cast<uint4*>(dst) = pk;
}

// fp32 outputs through shared memory: per 32-column chunk the warp's 32 rows
// go into its 4 KiB staging tile (128-byte swizzle) and one lane issues a TMA
// tensor store of the box at (column, row, shard) of the half's output map,
// which clips it at the shard's extents.
template <int BN>
__device__ __forceinline__ void epilogue_f32_bulk(const GParams& P, const GTile& g, uint32_t tacc,
                                                  int32_t row0, int half, uint32_t stage,
                                                  const CUtensorMap* mapC, int lane) {
#pragma unroll 1
  for (int q = 0; q < BN / 64; ++q) {
    const int c0 = half * (BN / 2) + q * 32;
    const int32_t j0 = g.n * BN + c0;
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + c0, v);
    tmem_ld_wait();
    if (j0 >= P.N) continue;   // warp-uniform
    if (lane == 0) bulk_wait_read0();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 8; ++c) {
      const uint32_t addr = stage + lane * 128 + ((c ^ (lane & 7)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[4 * c]),
                   "r"(v[4 * c + 1]), "r"(v[4 * c + 2]), "r"(v[4 * c + 3])
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      tma_store_3d(mapC, stage, j0, row0, g.shard);
      bulk_commit();
    }
  }
}

template <int EPI, int BN>
__device__ __forceinline__ void epilogue(const GParams& P, const GTile& g, uint32_t tacc, int row,
                                         int half) {
  const bool row_ok = row < P.M;
  const int64_t rbase = static_cast<int64_t>(g.shard) * P.out_shard_stride +
                        static_cast<int64_t>(row) * P.ldc;
#pragma unroll 1
  for (int q = 0; q < BN / 64; ++q) {
    const int c0 = half * (BN / 2) + q * 32;
    const int32_t j0 = g.n * BN + c0;
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + c0, v);
    tmem_ld_wait();
    if (!row_ok) continue;
    if constexpr (EPI == kEpiF32) {
      float* dst = static_cast<float*>(P.out[g.half]) + rbase;
#pragma unroll
      for (int e4 = 0; e4 < 8; ++e4) {
        const int32_t j = j0 + e4 * 4;
        if (j >= P.N) break;
        *reinterpret_cast<float4*>(dst + j) =
            make_float4(__uint_as_float(v[e4 * 4 + 0]), __uint_as_float(v[e4 * 4 + 1]),
                        __uint_as_float(v[e4 * 4 + 2]), __uint_as_float(v[e4 * 4 + 3]));
      }
    } else {
      const __nv_bfloat16* H = static_cast<const __nv_bfloat16*>(P.aux0) + rbase;
      __nv_bfloat16* dH = static_cast<__nv_bfloat16*>(P.out[0]) + rbase;
#pragma unroll
      for (int e8 = 0; e8 < 4; ++e8) {
        const int32_t j = j0 + e8 * 8;
        if (j >= P.N) break;
        float h[8], dy[8], o[8];
        unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(H + j)), h);
#pragma unroll
        for (int e = 0; e < 8; ++e) dy[e] = __uint_as_float(v[e8 * 8 + e]);
        if constexpr (EPI == kEpiActGrad) {
#pragma unroll
          for (int e = 0; e < 8; ++e) o[e] = dy[e] * act_grad_unary_mufu(P.act, h[e]);
          store_bf16x8_at(dH + j, o);
        } else {
          const __nv_bfloat16* U = static_cast<const __nv_bfloat16*>(P.aux1) + rbase;
          __nv_bfloat16* dU = static_cast<__nv_bfloat16*>(P.out[1]) + rbase;
          float u[8], ou[8];
          unpack_bf16x8(__ldg(reinterpret_cast<const uint4*>(U + j)), u);
#pragma unroll
          for (int e = 0; e < 8; ++e) {
            const float sg = sigmoid_mufu(h[e]);
            o[e] = dy[e] * u[e] * (sg * (1.0f + h[e] * (1.0f - sg)));   // d gate
            ou[e] = dy[e] * (h[e] * sg);                                // d up
          }
          store_bf16x8_at(dH + j, o);
          store_bf16x8_at(dU + j, ou);
        }
      }
    }
  }
}

template <int EPI, int BN>
using BCfg = Cfg<BN, EPI == kEpiF32 ? EPI_STAGE_BYTES : 0>;

template <int AMN, int BMN, int EPI, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_bwd_kernel(const __grid_constant__ CUtensorMap mapA0, const __grid_constant__ CUtensorMap mapA1,
                       const __grid_constant__ CUtensorMap mapB0, const __grid_constant__ CUtensorMap mapB1,
                       const __grid_constant__ CUtensorMap mapC0, const __grid_constant__ CUtensorMap mapC1,
                       const GParams P) {
  using C = BCfg<EPI, BN>;
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, AMN, BMN);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t epi_stage = base + STAGES * C::STAGE_BYTES;   // C::EPI_BYTES of staging
  uint8_t* const ctrl = smem_raw + (base - raw) + STAGES * C::STAGE_BYTES + C::EPI_BYTES;
  uint64_t* const bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * STAGES + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full_bar = [&](uint32_t s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](uint32_t s) { return smem_u32(&bars[STAGES + s]); };
  auto accf_bar = [&](uint32_t b) { return smem_u32(&bars[2 * STAGES + b]); };
  auto acce_bar = [&](uint32_t b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * STAGES + 4]);
  auto slot_a = [&](uint32_t s) { return base + s * C::STAGE_BYTES; };
  auto slot_b = [&](uint32_t s) { return base + s * C::STAGE_BYTES + A_BYTES; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), NUM_EPI_WARPS * 32);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA0);
    tma_prefetch_map(&mapB0);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; ok && t < P.num_tiles; t += gridDim.x) {
        const GTile g = decode(P, t);
        for (int32_t kb = 0; kb < P.k_blocks; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, P.wait, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (issued != P.debug_drop) {
            mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
            issue<AMN, BMN, BN>(P, &mapA0, &mapA1, &mapB0, &mapB1, g, kb, slot_a(stage),
                                slot_b(stage), full_bar(stage));
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      const int64_t first = issued > STAGES ? issued - STAGES : 0;
      for (int64_t q = first; q < issued; ++q) {
        if (q == P.debug_drop) continue;
        wait_teardown(full_bar(static_cast<uint32_t>(q % STAGES)),
                      static_cast<uint32_t>((q / STAGES) & 1), P.wait);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int32_t lt = 0;
      for (int32_t t = blockIdx.x; ok && t < P.num_tiles; t += gridDim.x, ++lt) {
        const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
        if (!wait_bounded(acce_bar(b), ap ^ 1u, abort_flag, P.wait, kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BN;
        for (int32_t kb = 0; kb < P.k_blocks; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, P.wait, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = slot_a(stage), sb = slot_b(stage);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            // K-major: a 16-element k step is 32 B inside the 128-byte swizzle
            // row; M/N-major: 64-wide atoms a chunk apart, a k step is 16
            // rows of 128 B.
            const uint64_t adesc = AMN == 0 ? smem_desc_sw128(sa + kk * UK * 2, 16, 1024)
                                            : smem_desc_sw128(sa + kk * UK * 128, A_CHUNK_BYTES, 1024);
            const uint64_t bdesc = BMN == 0 ? smem_desc_sw128(sb + kk * UK * 2, 16, 1024)
                                            : smem_desc_sw128(sb + kk * UK * 128, B_CHUNK_BYTES, 1024);
            tc_mma_f16(d_tmem, adesc, bdesc, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(accf_bar(b));
      }
      tc_commit(drain_bar);
      wait_teardown(drain_bar, 0, P.wait);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;
    int32_t lt = 0;
    for (int32_t t = blockIdx.x; t < P.num_tiles; t += gridDim.x, ++lt) {
      const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
      const GTile g = decode(P, t);
      bool ok = wait_bounded(accf_bar(b), ap, abort_flag, P.wait, kErrWaitAccFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * BN;
      if (EPI == kEpiF32 && P.bulk_out)
        epilogue_f32_bulk<BN>(P, g, tacc, g.m * BM + quad * 32, half,
                              epi_stage + (warp - 4) * EPI_WARP_STAGE_BYTES,
                              g.half > 0 ? &mapC1 : &mapC0, lane);
      else
        epilogue<EPI, BN>(P, g, tacc, g.m * BM + quad * 32 + lane, half);
      tc_fence_before();
      mbar_arrive(acce_bar(b));
    }
    if (lane == 0) bulk_wait_all0();   // staging read out before shared memory is released
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ CTA pairs
// The same four GEMMs on CTA pairs (tcgen05 cta_group::2) for layers large
// enough to fill the SMs with 256-row tiles: a cluster of two CTAs computes a
// 256 x PBN tile; each CTA loads its own 128 rows of A and half (PBN/2
// columns) of B, the even CTA's MMA thread issues M = 256 products that read
// both CTAs' shared memory and write each CTA's 128 accumulator rows into its
// own TMEM, and each CTA's epilogue stores its own rows.  Per SM the operand
// bytes per MMA cycle drop from 96 to 64 at width 256.  Barriers as in the
// forward pair kernel: the even CTA's full barrier counts both CTAs' bytes,
// the MMA commits multicast to both CTAs, every epilogue warp of both CTAs
// arrives on the even CTA's accumulator-empty barrier.  No load uses cluster
// multicast.  Every wait is bounded.
template <int PBN>
struct PairB {
  static constexpr int B_HALF_BYTES = (PBN / 2) * BK * 2;   // this CTA's half of B per slot
};

template <int AMN, int BMN, int PBN>
__device__ __forceinline__ void issue_pair(const GParams& P, const CUtensorMap* mA0,
                                           const CUtensorMap* mA1, const CUtensorMap* mB0,
                                           const CUtensorMap* mB1, const GTile& g, int32_t kb,
                                           uint32_t rank, uint32_t sa, uint32_t sb, uint32_t bar) {
  bool second = false;
  if (P.kb_half > 0 && kb >= P.kb_half) {
    second = true;
    kb -= P.kb_half;
  }
  const CUtensorMap* mA = second ? mA1 : mA0;
  const CUtensorMap* mB = (second || g.half > 0) ? mB1 : mB0;
  const int32_t za = P.a_batched ? g.shard : 0;
  const int32_t zb = P.b_batched ? g.shard : 0;
  const int32_t m0 = g.m * 2 * BM + static_cast<int32_t>(rank) * BM;
  const int32_t n0 = g.n * PBN + static_cast<int32_t>(rank) * (PBN / 2);
  const int32_t k0 = kb * BK;
  if constexpr (AMN == 0) {
    tma_load_3d_pair(sa, mA, bar, k0, m0, za);
  } else {
#pragma unroll
    for (int c = 0; c < BM / 64; ++c)
      tma_load_3d_pair(sa + c * A_CHUNK_BYTES, mA, bar, m0 + c * 64, k0, za);
  }
  if constexpr (BMN == 0) {
    tma_load_3d_pair(sb, mB, bar, k0 + g.shard * P.b_koff, n0, zb);
  } else {
#pragma unroll
    for (int c = 0; c < PBN / 2 / 64; ++c)
      tma_load_3d_pair(sb + c * B_CHUNK_BYTES, mB, bar, n0 + c * 64, k0, zb);
  }
}

template <int EPI, int PBN>
struct PBCfg {
  static constexpr int EPI_BYTES = EPI == kEpiF32 ? EPI_STAGE_BYTES : 0;
  static constexpr int STAGE_BYTES = A_BYTES + PairB<PBN>::B_HALF_BYTES;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - CTRL_BYTES - EPI_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + CTRL_BYTES;
  static constexpr int TMEM_COLS = 2 * PBN <= 256 ? 256 : 512;
  static_assert(PBN == 128 || PBN == 256, "pair tile width");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
  static_assert(8 * (2 * STAGES + 5) + 16 <= CTRL_BYTES, "control block");
};

template <int AMN, int BMN, int EPI, int PBN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_bwd_pair_kernel(const __grid_constant__ CUtensorMap mapA0,
                            const __grid_constant__ CUtensorMap mapA1,
                            const __grid_constant__ CUtensorMap mapB0,
                            const __grid_constant__ CUtensorMap mapB1,
                            const __grid_constant__ CUtensorMap mapC0,
                            const __grid_constant__ CUtensorMap mapC1, const GParams P) {
  using C = PBCfg<EPI, PBN>;
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t IDESC = idesc_bf16_f32(2 * BM, PBN, AMN, BMN);
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t epi_stage = base + STAGES * C::STAGE_BYTES;
  uint8_t* const ctrl = smem_raw + (base - raw) + STAGES * C::STAGE_BYTES + C::EPI_BYTES;
  uint64_t* const bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * STAGES + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  auto full_bar = [&](uint32_t s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](uint32_t s) { return smem_u32(&bars[STAGES + s]); };
  auto accf_bar = [&](uint32_t b) { return smem_u32(&bars[2 * STAGES + b]); };
  auto acce_bar = [&](uint32_t b) { return smem_u32(&bars[2 * STAGES + 2 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * STAGES + 4]);
  auto slot_a = [&](uint32_t s) { return base + s * C::STAGE_BYTES; };
  auto slot_b = [&](uint32_t s) { return base + s * C::STAGE_BYTES + A_BYTES; };
  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int32_t cluster = blockIdx.x / 2;
  const int32_t nclusters = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < STAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 2 * NUM_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA0);
    tma_prefetch_map(&mapB0);
  }
  if (warp == 2) {
    tmem_alloc_pair(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish_pair();
  }
  tc_fence_before();
  cluster_sync();  // both CTAs' barriers initialised and TMEM allocated
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  pdl_wait();
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      uint32_t stage = 0, phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int32_t t = cluster; ok && t < P.num_tiles; t += nclusters) {
        const GTile g = decode(P, t);
        for (int32_t kb = 0; kb < P.k_blocks; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, P.wait, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          // fault injection (tests of the bounded waits): the first pair only
          if (issued != P.debug_drop || cluster != 0) {
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * C::STAGE_BYTES);
            issue_pair<AMN, BMN, PBN>(P, &mapA0, &mapA1, &mapB0, &mapB1, g, kb, rank,
                                      slot_a(stage), slot_b(stage),
                                      mapa_shared(full_bar(stage), 0));
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // our last loads must have landed before this CTA's shared memory is
      // released: the even CTA sees that on its full barriers, the odd CTA
      // on its empty barriers (the MMA consumed the slot)
      const int64_t first = issued > STAGES ? issued - STAGES : 0;
      for (int64_t q = first; q < issued; ++q) {
        if (q == P.debug_drop && cluster == 0) continue;
        const uint32_t s = static_cast<uint32_t>(q % STAGES);
        const uint32_t ph = static_cast<uint32_t>((q / STAGES) & 1);
        wait_teardown(rank == 0 ? full_bar(s) : empty_bar(s), ph, P.wait);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int32_t lt = 0;
      for (int32_t t = cluster; ok && t < P.num_tiles; t += nclusters, ++lt) {
        const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
        if (!wait_bounded(acce_bar(b), ap ^ 1u, abort_flag, P.wait, kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * PBN;
        for (int32_t kb = 0; kb < P.k_blocks; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, P.wait, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = slot_a(stage), sb = slot_b(stage);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t adesc = AMN == 0 ? smem_desc_sw128(sa + kk * UK * 2, 16, 1024)
                                            : smem_desc_sw128(sa + kk * UK * 128, A_CHUNK_BYTES, 1024);
            const uint64_t bdesc = BMN == 0 ? smem_desc_sw128(sb + kk * UK * 2, 16, 1024)
                                            : smem_desc_sw128(sb + kk * UK * 128, B_CHUNK_BYTES, 1024);
            tc_mma_f16_pair(d_tmem, adesc, bdesc, IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair_mc(empty_bar(stage), 0x3);
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit_pair_mc(accf_bar(b), 0x3);
      }
      tc_commit_pair_mc(drain_bar, 0x1);
      wait_teardown(drain_bar, 0, P.wait);
    }
    __syncwarp();
  } else if (warp >= 4) {
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;
    int32_t lt = 0;
    for (int32_t t = cluster; t < P.num_tiles; t += nclusters, ++lt) {
      const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
      const GTile g = decode(P, t);
      bool ok = wait_bounded(accf_bar(b), ap, abort_flag, P.wait, kErrWaitAccFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * PBN;
      const int32_t row0 = g.m * 2 * BM + static_cast<int32_t>(rank) * BM + quad * 32;
      if (EPI == kEpiF32 && P.bulk_out)
        epilogue_f32_bulk<PBN>(P, g, tacc, row0, half,
                               epi_stage + (warp - 4) * EPI_WARP_STAGE_BYTES,
                               g.half > 0 ? &mapC1 : &mapC0, lane);
      else
        epilogue<EPI, PBN>(P, g, tacc, row0 + lane, half);
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(acce_bar(b), 0));
      if constexpr (EPI == kEpiF32) {
        if (P.region_cnt != nullptr) {
          // Publish this warp's part of the tile to the fold beside this
          // layer (as the forward row layer does): bulk stores complete,
          // ordered for generic-proxy readers, one release increment.
          if (lane == 0) {
            bulk_wait_all0();
            fence_proxy_async_global();
            red_release_gpu_add(P.region_cnt + g.n * P.m_tiles + g.m, 1);
          }
          __syncwarp();
        }
      }
    }
    if (lane == 0) bulk_wait_all0();   // staging read out before shared memory is released
  }

  tc_fence_before();
  cluster_sync();  // the pair's MMAs, commits and arrivals are done with both CTAs
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

template <int AMN, int BMN, int EPI, int PBN>
tp_status launch_gp(const LaunchCtx& c, const CUtensorMap* maps, GParams prm) {
  using Cf = PBCfg<EPI, PBN>;
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_gemm_bwd_pair_kernel<AMN, BMN, EPI, PBN>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  prm.m_tiles = ceil_div(prm.M, 2 * BM);
  prm.n_tiles = ceil_div(prm.N, PBN);
  prm.num_tiles = prm.m_tiles * prm.n_tiles * prm.p * prm.halves;
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  if (prm.num_tiles == 0) return TP_OK;
  int clusters = c.num_sms / 2;
  if (clusters > prm.num_tiles) clusters = prm.num_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = Cf::SMEM_BYTES;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
  attr[1].val.programmaticStreamSerializationAllowed = 1;
  cfg.attrs = attr;
  cfg.numAttrs = pdl_allowed() ? 2 : 1;
  const cudaError_t e = cudaLaunchKernelEx(&cfg, tc_gemm_bwd_pair_kernel<AMN, BMN, EPI, PBN>,
                                           maps[0], maps[1], maps[2], maps[3], maps[4], maps[5],
                                           prm);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("paired backward GEMM launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

template <int AMN, int BMN, int EPI, int BN>
tp_status launch_g(const LaunchCtx& c, const CUtensorMap* maps, GParams prm) {
  using Cf = BCfg<EPI, BN>;
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_gemm_bwd_kernel<AMN, BMN, EPI, BN>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  prm.n_tiles = ceil_div(prm.N, BN);
  prm.num_tiles = prm.m_tiles * prm.n_tiles * prm.p * prm.halves;
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  if (prm.num_tiles == 0) return TP_OK;
  const int grid = prm.num_tiles < c.num_sms ? prm.num_tiles : c.num_sms;
  const cudaError_t e = launch_pdl(tc_gemm_bwd_kernel<AMN, BMN, EPI, BN>, dim3(grid),
                                   dim3(NUM_THREADS), Cf::SMEM_BYTES, c.stream, maps[0], maps[1],
                                   maps[2], maps[3], maps[4], maps[5], prm);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("backward GEMM launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

// Tile shape for an (M x N) x batches problem with K / 64 slots: the
// forward's cost model (single-CTA widths 64, 128, 256; CTA-pair tiles of
// 256 rows x 128 or 256 once single-CTA tiles take more than one wave).
TileChoice choose_tile(int64_t M, int64_t N, int64_t batches, int64_t k_blocks, int num_sms) {
  // the backward kernels have no 192-wide single-CTA tile
  return pick_tile(M, N, batches, k_blocks, num_sms, false, pair_allowed(), false);
}

// Width of a K-major B operand's TMA box: the tile width, or its half on
// CTA pairs (each CTA loads half of B's columns).
uint32_t b_box(const TileChoice& t) { return static_cast<uint32_t>(t.pair ? t.bn / 2 : t.bn); }

template <int AMN, int BMN, int EPI>
tp_status dispatch(const LaunchCtx& c, const CUtensorMap* maps, const GParams& prm,
                   const TileChoice& t) {
  if (t.pair) {
    if (t.bn == 256) return launch_gp<AMN, BMN, EPI, 256>(c, maps, prm);
    return launch_gp<AMN, BMN, EPI, 128>(c, maps, prm);
  }
  if (t.bn == 256) return launch_g<AMN, BMN, EPI, 256>(c, maps, prm);
  if (t.bn == 128) return launch_g<AMN, BMN, EPI, 128>(c, maps, prm);
  return launch_g<AMN, BMN, EPI, 64>(c, maps, prm);
}

// 3-D bf16 map: dims (inner, outer, batch), row stride and batch stride in
// elements; box (inner 64, outer box_outer).
bool map3(CUtensorMap* m, const void* g, int64_t inner, int64_t outer, int64_t batch,
          int64_t row_stride, int64_t batch_stride, uint32_t box_outer) {
  const uint64_t dims[3] = {static_cast<uint64_t>(inner), static_cast<uint64_t>(outer),
                            static_cast<uint64_t>(batch)};
  const uint64_t strides[2] = {static_cast<uint64_t>(row_stride) * 2,
                               static_cast<uint64_t>(batch > 1 ? batch_stride : row_stride * outer) * 2};
  const uint32_t box[3] = {64, box_outer, 1};
  return make_map(m, g, 3, dims, strides, box);
}

GParams base_params(int64_t M, int64_t N, int64_t K, int p, int halves) {
  GParams prm{};
  prm.M = static_cast<int32_t>(M);
  prm.N = static_cast<int32_t>(N);
  prm.K = static_cast<int32_t>(K);
  prm.p = p;
  prm.halves = halves;
  prm.m_tiles = ceil_div(M, BM);
  prm.k_blocks = ceil_div(K, BK);
  return prm;
}

}  // namespace

// G1: dH_i = (dZ W2_i^T) * act'(H_i)   [SwiGLU: dG_i, dU_i]
tp_status launch_bwd_act_grad(const LaunchCtx& c, const void* dZ, const void* W2, const void* H,
                              const void* Hup, void* dH, void* dU, int64_t T, int64_t d, int64_t k,
                              int p, int act) {
  const int64_t s = k / p;
  GParams prm = base_params(T, s, d, p, 1);
  prm.a_batched = 0;
  prm.b_batched = 1;
  prm.act = act;
  prm.out[0] = dH;
  prm.out[1] = dU;
  prm.out_shard_stride = T * s;
  prm.ldc = s;
  prm.aux0 = H;
  prm.aux1 = Hup;
  const TileChoice tch = choose_tile(T, s, p, prm.k_blocks, c.num_sms);
  CUtensorMap maps[6];
  // A = dZ [T][d] K-major; B = W2 rows of shard i: [p][s][d] K-major (N rows)
  if (!map3(&maps[0], dZ, d, T, 1, d, 0, BM) || !map3(&maps[2], W2, d, s, p, d, s * d, b_box(tch)))
    return TP_ERR_CUDA;
  maps[1] = maps[0];
  maps[3] = maps[2];
  maps[4] = maps[5] = maps[0];   // bf16 outputs: per-thread stores
  if (act == kActSwiglu) return dispatch<0, 0, kEpiSwigluGrad>(c, maps, prm, tch);
  return dispatch<0, 0, kEpiActGrad>(c, maps, prm, tch);
}

// G2: dX partials P_i = dH_i W1_i^T (+ dU_i Wup_i^T), fp32 [p][T][d]
bool bwd_dx_on_pairs(const LaunchCtx& c, int64_t T, int64_t k_eff, int64_t d, int p) {
  return choose_tile(T, d, p, ceil_div(k_eff / p, BK), c.num_sms).pair;
}

tp_status launch_bwd_dx_partials(const LaunchCtx& c, const void* dH, const void* dU,
                                 const void* W1, const void* Wup, float* P, int64_t T, int64_t d,
                                 int64_t k, int p, int* region_cnt, RegionFold* rf) {
  const int64_t s = k / p;
  const bool two = dU != nullptr;
  GParams prm = base_params(T, d, two ? 2 * s : s, p, 1);
  if (two) {
    prm.kb_half = ceil_div(s, BK);
    prm.k_blocks = 2 * prm.kb_half;
  }
  prm.a_batched = 1;
  prm.b_batched = 0;
  prm.b_koff = static_cast<int32_t>(s);
  prm.out[0] = P;
  prm.out[1] = P;
  prm.out_shard_stride = T * d;
  prm.ldc = d;
  const TileChoice tch = choose_tile(T, d, p, prm.k_blocks, c.num_sms);
  CUtensorMap maps[6];
  // A = dH [p][T][s] K-major; B = W1 [d][k] K-major (inner k, outer d = N
  // rows), shard i's block at K offset i s
  if (!map3(&maps[0], dH, s, T, p, s, T * s, BM) || !map3(&maps[2], W1, k, d, 1, k, 0, b_box(tch)))
    return TP_ERR_CUDA;
  if (two) {
    if (!map3(&maps[1], dU, s, T, p, s, T * s, BM) ||
        !map3(&maps[3], Wup, k, d, 1, k, 0, b_box(tch)))
      return TP_ERR_CUDA;
  } else {
    maps[1] = maps[0];
    maps[3] = maps[2];
  }
  if (!make_map_f32_out(&maps[4], P, d, T, p)) return TP_ERR_CUDA;
  maps[5] = maps[4];
  prm.bulk_out = 1;
  if (rf != nullptr) *rf = RegionFold{};
  if (tch.pair && region_cnt != nullptr && rf != nullptr) {
    // regions = the pair tiles, taken in two halves of the m-tiles as in the
    // forward row layer; 16 epilogue warps count once per tile and shard
    const int32_t m_tiles = ceil_div(T, 2 * BM);
    prm.region_cnt = region_cnt;
    prm.m_group = m_tiles >= 4 ? ceil_div(m_tiles, 2) : 0;
    *rf = RegionFold{region_cnt, 2 * BM, tch.bn, m_tiles, ceil_div(d, tch.bn),
                     2 * NUM_EPI_WARPS * p, prm.m_group};
  }
  return dispatch<0, 0, kEpiF32>(c, maps, prm, tch);
}

// G3: dW1[:, i s:(i+1) s] = X^T dH_i  (SwiGLU: dW_up from dU as a second
// half of the batches), fp32 [d][k]
tp_status launch_bwd_dw1(const LaunchCtx& c, const void* X, const void* dH, const void* dU,
                         float* dW1, float* dWup, int64_t T, int64_t d, int64_t k, int p) {
  const int64_t s = k / p;
  const bool two = dU != nullptr && dWup != nullptr;
  GParams prm = base_params(d, s, T, p, two ? 2 : 1);
  prm.a_batched = 0;
  prm.b_batched = 1;
  prm.out[0] = dW1;
  prm.out[1] = two ? dWup : dW1;
  prm.out_shard_stride = s;
  prm.ldc = k;
  const TileChoice tch = choose_tile(d, s, p * prm.halves, prm.k_blocks, c.num_sms);
  CUtensorMap maps[6];
  // A = X^T: M-major view of X [T][d] (inner d = M, outer T = K);
  // B = dH [p][T][s] N-major (inner s = N, outer T = K)
  if (!map3(&maps[0], X, d, T, 1, d, 0, BK) || !map3(&maps[2], dH, s, T, p, s, T * s, BK))
    return TP_ERR_CUDA;
  maps[1] = maps[0];
  if (two) {
    if (!map3(&maps[3], dU, s, T, p, s, T * s, BK)) return TP_ERR_CUDA;
  } else {
    maps[3] = maps[2];
  }
  // dW1's column block i: (s columns, d rows, shard i at a column offset of
  // i s); the bulk path needs the driver to accept the interleaved batch
  // stride, else the per-thread epilogue writes it
  prm.bulk_out = make_map_f32_strided(&maps[4], dW1, s, d, p, k, s) ? 1 : 0;
  if (prm.bulk_out && two) prm.bulk_out = make_map_f32_strided(&maps[5], dWup, s, d, p, k, s) ? 1 : 0;
  if (!prm.bulk_out) maps[4] = maps[0];
  if (!two || !prm.bulk_out) maps[5] = maps[4];
  return dispatch<1, 1, kEpiF32>(c, maps, prm, tch);
}

// G4: dW2[i s:(i+1) s, :] = Y_i^T dZ, fp32 [k][d]
tp_status launch_bwd_dw2(const LaunchCtx& c, const void* Y, const void* dZ, float* dW2, int64_t T,
                         int64_t d, int64_t k, int p) {
  const int64_t s = k / p;
  GParams prm = base_params(s, d, T, p, 1);
  prm.a_batched = 1;
  prm.b_batched = 0;
  prm.out[0] = dW2;
  prm.out[1] = dW2;
  prm.out_shard_stride = s * d;
  prm.ldc = d;
  const TileChoice tch = choose_tile(s, d, p, prm.k_blocks, c.num_sms);
  CUtensorMap maps[6];
  // A = Y_i^T: M-major view of Y [p][T][s]; B = dZ [T][d] N-major
  if (!map3(&maps[0], Y, s, T, p, s, T * s, BK) || !map3(&maps[2], dZ, d, T, 1, d, 0, BK))
    return TP_ERR_CUDA;
  maps[1] = maps[0];
  maps[3] = maps[2];
  // dW2's row block i as shard i of a [p][s][d] tensor
  if (!make_map_f32_out(&maps[4], dW2, d, s, p)) return TP_ERR_CUDA;
  maps[5] = maps[4];
  prm.bulk_out = 1;
  return dispatch<1, 1, kEpiF32>(c, maps, prm, tch);
}

}  // namespace tpk
