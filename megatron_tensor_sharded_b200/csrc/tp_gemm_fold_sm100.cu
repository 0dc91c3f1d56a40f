// Row-parallel layer with the reduction in its epilogue (sm_100a).
//
// The row-parallel layer produces one full-shape partial per shard, P_i =
// Y_i W2_i, and the all-reduce sums them ("Tensor parallel math",
// "Row-parallel: split the weight by input rows"; day-41 post, "Simulating
// row parallel linear": sum(partial_sums) + bias).  Here one CTA owns an
// output tile of Z and computes the p partials of that tile one after the
// other, each in its own TMEM accumulator (K loop over shard i's rows of W2
// only), and its epilogue folds them in shard order as they complete:
//
//   R = P_0;  R = R + P_1;  ...;  Z = (R + P_{p-1}) [+ b2]
//
// every addition one fp32 round-to-nearest-even operation, the running sum R
// kept in TMEM.  Each P_i is the same fp32 accumulator the partials layer
// would store, and the additions are those of the fold kernel in the same
// order, so Z is bit-identical to tp_row_linear + tp_reduce_partials -- the
// p partials simply never leave the SM.
//
// Roles (384 threads): warp 0 TMA (A = Y_i tile of the shard the K block
// belongs to, B = the matching 64 rows of W2), warp 1 MMA into a 2-deep ring
// of accumulators (shard i+1 accumulates while the epilogue folds shard i),
// warp 2 TMEM, warps 4..11 fold + bias + bulk tensor store of Z.  TMEM: two
// accumulators and the running sum, 3 * BN columns.  Every wait is bounded.
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

template <int BN>
using FCfg = Cfg<BN, EPI_STAGE_BYTES>;

template <int BN>
constexpr int kFoldTmemCols = 3 * BN <= 256 ? 256 : 512;

template <int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_row_fold_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB,
                       const __grid_constant__ CUtensorMap mapZ, const TcParams P) {
  using C = FCfg<BN>;
  constexpr int STAGES = C::STAGES;
  constexpr int TMEM_COLS = kFoldTmemCols<BN>;
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
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB);
    tma_prefetch_map(&mapZ);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), TMEM_COLS);
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
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; ok && t < P.num_tiles; t += gridDim.x) {
        const TileCoord tc = decode_tile(P, t);
        for (int32_t kb = 0; kb < P.k_blocks; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, P.wait, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (issued != P.debug_drop) {
            mbar_arrive_expect_tx(full_bar(stage), C::STAGE_BYTES);
            // shard kb / kb_per_shard: its Y tile and W2 rows [kb*64, kb*64+64)
            issue_slot<kModeRowSplitK, BN>(P, &mapA, &mapB, &mapB, tc, kb, slot_a(stage),
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
      // ---------------------------------------------------------- MMA issuer
      // one accumulator use per (tile, shard); uses alternate between the
      // two buffers
      uint32_t stage = 0, phase = 0, use = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; ok && t < P.num_tiles; t += gridDim.x) {
        for (int32_t i = 0; ok && i < P.p; ++i, ++use) {
          const uint32_t b = use & 1, ap = (use >> 1) & 1;
          if (!wait_bounded(acce_bar(b), ap ^ 1u, abort_flag, P.wait, kErrWaitAccEmpty)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t d_tmem = tmem_base + b * BN;
          for (int32_t kin = 0; kin < P.kb_per_shard; ++kin) {
            if (!wait_bounded(full_bar(stage), phase, abort_flag, P.wait, kErrWaitFull)) {
              ok = false;
              break;
            }
            tc_fence_after();
            const uint32_t sa = slot_a(stage), sb = slot_b(stage);
#pragma unroll
            for (int kk = 0; kk < BK / UK; ++kk) {
              const uint64_t adesc = smem_desc_sw128(sa + kk * UK * 2, 16, 1024);
              const uint64_t bdesc = smem_desc_sw128(sb + kk * UK * 128, B_CHUNK_BYTES, 1024);
              tc_mma_f16(d_tmem, adesc, bdesc, C::IDESC, (kin > 0 || kk > 0) ? 1u : 0u);
            }
            tc_commit(empty_bar(stage));
            if (++stage == STAGES) {
              stage = 0;
              phase ^= 1u;
            }
          }
          if (!ok) break;
          tc_commit(accf_bar(b));   // partial P_i of this tile complete
        }
      }
      tc_commit(drain_bar);
      wait_teardown(drain_bar, 0, P.wait);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------ fold + epilogue
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t trun = tmem_base + lane_off + 2 * BN;   // running sum
    const uint32_t stage_w = epi_stage + (warp - 4) * EPI_WARP_STAGE_BYTES;
    const float* __restrict__ bias = static_cast<const float*>(P.bias);
    uint32_t use = 0;
    bool ok = true;
    for (int32_t t = blockIdx.x; ok && t < P.num_tiles; t += gridDim.x) {
      const TileCoord tc = decode_tile(P, t);
      const int32_t row0 = tc.m * BM + quad * 32;
      for (int32_t i = 0; i < P.p; ++i, ++use) {
        const uint32_t b = use & 1, ap = (use >> 1) & 1;
        ok = wait_bounded(accf_bar(b), ap, abort_flag, P.wait, kErrWaitAccFull);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tacc = tmem_base + lane_off + b * BN;
        const bool last = (i == P.p - 1);
#pragma unroll 1
        for (int q = 0; q < BN / 64; ++q) {
          const int c0 = half * (BN / 2) + q * 32;
          const int32_t j0 = tc.n * BN + c0;
          float bv[32];
          if (last && bias != nullptr) {
#pragma unroll
            for (int e = 0; e < 32; ++e) bv[e] = (j0 + e < P.n_total) ? __ldg(bias + j0 + e) : 0.0f;
          }
          uint32_t v[32], r[32];
          tmem_ld_32x32b_x32(tacc + c0, v);
          if (i > 0) tmem_ld_32x32b_x32(trun + c0, r);
          tmem_ld_wait();
          if (i > 0) {
#pragma unroll
            for (int e = 0; e < 32; ++e)
              v[e] = __float_as_uint(__fadd_rn(__uint_as_float(r[e]), __uint_as_float(v[e])));
          }
          if (!last) {
            tmem_st_32x32b_x32(trun + c0, v);
            continue;
          }
          if (bias != nullptr) {
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__fadd_rn(__uint_as_float(v[e]), bv[e]));
          }
          if (j0 >= P.n_total) continue;   // warp-uniform
          if (lane == 0) bulk_wait_read0();
          __syncwarp();
#pragma unroll
          for (int c = 0; c < 8; ++c) {
            const uint32_t addr = stage_w + lane * 128 + ((c ^ (lane & 7)) << 4);
            asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(v[4 * c]),
                         "r"(v[4 * c + 1]), "r"(v[4 * c + 2]), "r"(v[4 * c + 3])
                         : "memory");
          }
          fence_proxy_async_smem();
          __syncwarp();
          if (lane == 0) {
            tma_store_3d(&mapZ, stage_w, j0, row0, 0);
            bulk_commit();
          }
        }
        if (!last) tmem_st_wait();   // the running sum is in place before the buffer is released
        tc_fence_before();
        mbar_arrive(acce_bar(b));
      }
    }
    if (lane == 0) bulk_wait_all0();
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

template <int BN>
tp_status launch_fold(const LaunchCtx& c, const CUtensorMap& a, const CUtensorMap& b,
                      const CUtensorMap& z, TcParams prm) {
  using Cf = FCfg<BN>;
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_row_fold_kernel<BN>, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  prm.n_tiles = ceil_div(prm.n_total, BN);
  prm.num_tiles = prm.m_tiles * prm.n_tiles;
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  const int grid = prm.num_tiles < c.num_sms ? prm.num_tiles : c.num_sms;
  const cudaError_t e = launch_pdl(tc_row_fold_kernel<BN>, dim3(grid), dim3(NUM_THREADS),
                                   Cf::SMEM_BYTES, c.stream, a, b, z, prm);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("row-fold GEMM launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

}  // namespace

// Z = fold_i(Y_i W2_i) [+ b2] in shard order, bit-identical to the partials
// layer followed by the fixed-order reduction.  Needs k/p % 64 == 0.
tp_status launch_tc_row_fold(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                             float* Z, int64_t T, int64_t k, int64_t d, int p) {
  const int64_t s = k / p;
  CUtensorMap mA, mB, mZ;
  if (!make_map_a(&mA, Y, s, T, p) || !make_map_b(&mB, W2, d, k) ||
      !make_map_f32_out(&mZ, Z, d, T, 1))
    return TP_ERR_CUDA;
  TcParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.n_total = static_cast<int32_t>(d);
  prm.s = static_cast<int32_t>(s);
  prm.p = p;
  prm.m_tiles = ceil_div(T, BM);
  prm.batches = 1;
  prm.kb_per_shard = static_cast<int32_t>(s / BK);
  prm.k_blocks = prm.kb_per_shard * p;
  prm.act = kActIdentity;
  prm.bias = b2;
  prm.out = Z;
  // 128-column tiles when they alone fill the SMs, else 64 (twice the tiles)
  const int64_t tiles128 = static_cast<int64_t>(prm.m_tiles) * ((d + 127) / 128);
  if (tiles128 >= c.num_sms) return launch_fold<128>(c, mA, mB, mZ, prm);
  return launch_fold<64>(c, mA, mB, mZ, prm);
}

}  // namespace tpk
