// bf16 tensor-core GEMMs of the sharded MLP block for sm_100a.
//
// One persistent, warp-specialised kernel template serves every GEMM of the
// block; the tile scheduler walks (shard, m-tile, n-tile) units so that all p
// simulated shards of a layer run in a single launch:
//
//   column-parallel layer (day-41 post, "Simulating column parallel linear";
//   "Tensor parallel math", "Column-parallel: split the weight by output
//   columns"):  Y_i = act(X W1_i + b1_i)  -- the shard index only decides
//   where an output column is stored, [p][T][s];
//   SwiGLU variant ("Tensor Parallelism Explained", 2.B): one accumulator of
//   BN columns holds BN/2 gate and the matching BN/2 up columns, and the
//   epilogue writes SiLU(gate) * up;
//   row-parallel layer ("Simulating row parallel linear"; "Row-parallel:
//   split the weight by input rows"): P_i = Y_i W2_i, full-shape fp32
//   partials; or, split-K over shards, Z = sum_i Y_i W2_i accumulated in one
//   TMEM accumulator and written once (+ b2).
//
// Roles (384 threads):
//   warp 0 lane 0  TMA producer: A tile [128 x 64] (K-major) and B tile
//                  [64 x BN] (N-major, BN/64 boxes of 64 columns) per slot,
//                  128-byte swizzle, STAGES-deep ring;
//   warp 1 lane 0  MMA issuer: tcgen05.mma M=128 N=BN K=16, fp32 in TMEM,
//                  two accumulators so the epilogue of one tile overlaps the
//                  main loop of the next;
//   warp 2         TMEM allocation / release;
//   warps 4..11    epilogue: warp w reads TMEM lanes 32*(w%4).. (the lane
//                  quadrant it may access) and one half of the columns;
//                  bias + activation (or none), convert, then stages 32 x 32
//                  tiles in shared memory and bulk-stores them with TMA
//                  tensor stores (per-thread stores for column layers whose
//                  shard width is not a multiple of 32).
// Tile width BN (64..256) is picked per problem so that the tiles of a small
// problem still cover the SMs.  Every barrier wait is bounded.  Launches use
// programmatic dependent launch: the prologue overlaps the previous kernel,
// and every global access comes after griddepcontrol.wait.
#include <cuda.h>
#include <cudaTypedefs.h>
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

// Epilogues store through shared memory with bulk tensor stores (the column
// layers when every shard is a whole number of 32-column chunks).
template <int MODE>
constexpr bool kBulkOut = (MODE == kModeRowPartial || MODE == kModeRowSplitK);

template <int MODE, int BN>
using KCfg = Cfg<BN, EPI_STAGE_BYTES>;

template <int MODE, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                   const __grid_constant__ CUtensorMap mapB1, const __grid_constant__ CUtensorMap mapC,
                   const TcParams P) {
  using C = KCfg<MODE, BN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
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

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;

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
    tma_prefetch_map(&mapB0);
    if (MODE == kModeColumnSwiglu) tma_prefetch_map(&mapB1);
    if (kBulkOut<MODE> || P.bulk_out) tma_prefetch_map(&mapC);
  }
  if (warp == 2) {
    tmem_alloc(smem_u32(tmem_slot), C::TMEM_COLS);
    tmem_relinquish();
  }
  tc_fence_before();
  __syncthreads();
  tc_fence_after();
  const uint32_t tmem_base = *reinterpret_cast<volatile uint32_t*>(tmem_slot);
  // Everything above overlaps the previous kernel; from here on global
  // memory is read and written.
  pdl_wait();
  zero_counters(P, warp, lane);
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
            issue_slot<MODE, BN>(P, &mapA, &mapB0, &mapB1, tc, kb, slot_a(stage), slot_b(stage),
                                 full_bar(stage));
          }
          ++issued;
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Teardown: the last (up to STAGES) loads must land before the CTA's
      // shared memory is released.
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
            // A: K-major, 128-byte swizzle; 8-row groups 1024 B apart; a
            // 16-element k step is 32 B inside the swizzle row.
            const uint64_t adesc = smem_desc_sw128(sa + kk * UK * 2, 16, 1024);
            // B: N-major, 128-byte swizzle; 64-column atoms B_CHUNK_BYTES
            // apart (leading), 8 k-rows 1024 B apart (stride); a 16-row k step
            // is 16 * 128 B.
            const uint64_t bdesc = smem_desc_sw128(sb + kk * UK * 128, B_CHUNK_BYTES, 1024);
            tc_mma_f16(d_tmem, adesc, bdesc, C::IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(empty_bar(stage));  // slot free once these MMAs have read it
          if (++stage == STAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
        if (!ok) break;
        tc_commit(accf_bar(b));  // accumulator b complete
      }
      // Teardown: every MMA issued above must finish before TMEM is freed.
      tc_commit(drain_bar);
      wait_teardown(drain_bar, 0, P.wait);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;          // TMEM lane quadrant this warp may access
    const int half = (warp - 4) >> 2;   // which half of the accumulator columns
    uint32_t nchunk = 0;   // bf16 chunks this warp has staged (alternating halves)
    int32_t lt = 0;
    for (int32_t t = blockIdx.x; t < P.num_tiles; t += gridDim.x, ++lt) {
      const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
      const TileCoord tc = decode_tile(P, t);
      EpiBias<MODE, BN> eb;
      load_epi_bias<MODE, BN>(P, tc, half, eb);
      bool ok = wait_bounded(accf_bar(b), ap, abort_flag, P.wait, kErrWaitAccFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * BN;
      const uint32_t stage_w = epi_stage + (warp - 4) * EPI_WARP_STAGE_BYTES;
      if constexpr (kBulkOut<MODE>) {
        epilogue_tile_bulk<MODE, BN>(P, tc, tacc, tc.m * BM + quad * 32, half, stage_w, &mapC,
                                     lane);
      } else {
        if (P.bulk_out)
          epilogue_tile_bulk_col<MODE, BN>(P, tc, tacc, tc.m * BM + quad * 32, half, eb, stage_w,
                                           &mapC, lane, nchunk);
        else
          epilogue_tile<MODE, BN>(P, tc, tacc, tc.m * BM + quad * 32 + lane, half, eb);
      }
      tc_fence_before();
      mbar_arrive(acce_bar(b));
    }
    // the staging tiles must be read out before shared memory is released
    if (lane == 0) bulk_wait_all0();
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

template <int MODE, int BN>
tp_status launch_mode(const LaunchCtx& c, const CUtensorMap& a, const CUtensorMap& b0,
                      const CUtensorMap& b1, const CUtensorMap& cm, TcParams prm) {
  using Cf = KCfg<MODE, BN>;
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_gemm_kernel<MODE, BN>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  const int grid = prm.num_tiles < c.num_sms ? prm.num_tiles : c.num_sms;
  const cudaError_t e = launch_pdl(tc_gemm_kernel<MODE, BN>, dim3(grid), dim3(NUM_THREADS),
                                   Cf::SMEM_BYTES, c.stream, a, b0, b1, cm, prm);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("tensor-core GEMM launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

template <int MODE>
tp_status launch_bn(const LaunchCtx& c, int bn, const CUtensorMap& a, const CUtensorMap& b0,
                    const CUtensorMap& b1, const CUtensorMap& cm, TcParams prm) {
  const int out_cols = MODE == kModeColumnSwiglu ? bn / 2 : bn;
  prm.n_tiles = ceil_div(prm.n_total, out_cols);
  prm.num_tiles = prm.m_tiles * prm.n_tiles * prm.batches;
  switch (bn) {
    case 256: return launch_mode<MODE, 256>(c, a, b0, b1, cm, prm);
    case 128: return launch_mode<MODE, 128>(c, a, b0, b1, cm, prm);
    default: break;
  }
  if constexpr (MODE != kModeColumnSwiglu) {
    if (bn == 192) return launch_mode<MODE, 192>(c, a, b0, b1, cm, prm);
    if (bn == 64) return launch_mode<MODE, 64>(c, a, b0, b1, cm, prm);
  }
  set_error_detail("no tile width %d", bn);
  return TP_ERR_UNSUPPORTED;
}

}  // namespace

tp_status launch_tc_column(const LaunchCtx& c, const void* X, const void* W1, const void* Wup,
                           const void* b1, void* Y, int64_t T, int64_t d, int64_t k, int p,
                           int act, int* zero_cnt, int zero_n) {
  CUtensorMap mA, mB0, mB1, mY;
  if (!make_map_a(&mA, X, d, T, 1) || !make_map_b(&mB0, W1, k, d)) return TP_ERR_CUDA;
  const bool bulk = (k / p) % 32 == 0;
  if (bulk && !make_map_bf16_out(&mY, Y, k / p, T, p)) return TP_ERR_CUDA;
  if (!bulk) mY = mA;
  const bool swiglu = (act == kActSwiglu);
  if (swiglu) {
    if (!make_map_b(&mB1, Wup, k, d)) return TP_ERR_CUDA;
  } else {
    mB1 = mB0;
  }
  TcParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.n_total = static_cast<int32_t>(k);
  prm.s = static_cast<int32_t>(k / p);
  prm.p = p;
  prm.m_tiles = ceil_div(T, BM);
  prm.batches = 1;
  prm.k_blocks = ceil_div(d, BK);
  prm.kb_per_shard = 0;
  prm.act = act;
  prm.bias = b1;
  prm.out = Y;
  prm.bulk_out = bulk ? 1 : 0;
  prm.zero_cnt = zero_cnt;
  prm.zero_n = zero_n;
  const TileChoice tch = pick_tile(T, k, 1, prm.k_blocks, c.num_sms, swiglu, pair_allowed());
  const int mode = swiglu ? kModeColumnSwiglu : kModeColumn;
  if (tch.pair) return launch_tc_pair(c, mode, tch.bn, mA, mB0, mB1, mY, prm);
  if (swiglu) return launch_bn<kModeColumnSwiglu>(c, tch.bn, mA, mB0, mB1, mY, prm);
  return launch_bn<kModeColumn>(c, tch.bn, mA, mB0, mB1, mY, prm);
}

tp_status launch_tc_column_multi(const LaunchCtx& c, const void* X, const void* const* W,
                                 void* const* Y, const int64_t* k, int nseg, int64_t T, int64_t d,
                                 int p, int* zero_cnt, int zero_n, bool* done) {
  *done = false;
  if (nseg < 1 || nseg > 3 || !pair_allowed()) return TP_OK;
  int64_t ktot = 0;
  for (int i = 0; i < nseg; ++i) {
    if (k[i] % p != 0 || (k[i] / p) % 32 != 0) return TP_OK;   // bulk stores per shard
    ktot += k[i];
  }
  const TileChoice tch = pick_tile(T, ktot, 1, ceil_div(d, BK), c.num_sms, false, true);
  if (!tch.pair) return TP_OK;
  CUtensorMap mA, mB[3], mC[3];
  if (!make_map_a(&mA, X, d, T, 1)) return TP_ERR_CUDA;
  for (int i = 0; i < nseg; ++i)
    if (!make_map_b(&mB[i], W[i], k[i], d) || !make_map_bf16_out(&mC[i], Y[i], k[i] / p, T, p))
      return TP_ERR_CUDA;
  TcParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.n_total = static_cast<int32_t>(k[0]);
  prm.s = static_cast<int32_t>(k[0] / p);
  prm.p = p;
  prm.batches = 1;
  prm.k_blocks = ceil_div(d, BK);
  prm.act = kActIdentity;
  prm.bias = nullptr;
  prm.out = Y[0];
  prm.bulk_out = 1;
  prm.zero_cnt = zero_cnt;
  prm.zero_n = zero_n;
  *done = true;
  return launch_tc_pair_column_multi(c, tch.bn, mA, mB, mC, k, nseg, prm);
}

// One int per region at most: regions are row tiles of 128 or 256 rows and
// 64 to 256 columns.
size_t region_counter_bytes(int64_t T, int64_t d) {
  const size_t n = static_cast<size_t>(ceil_div(T, BM)) * static_cast<size_t>(ceil_div(d, 64));
  return (n * sizeof(int) + 255) & ~size_t(255);
}

tp_status launch_tc_row(const LaunchCtx& c, const void* Y, const void* W2, float* P, int64_t T,
                        int64_t k, int64_t d, int p, int* region_cnt, RegionFold* rf) {
  const int64_t s = k / p;
  CUtensorMap mA, mB, mC;
  if (!make_map_a(&mA, Y, s, T, p) || !make_map_b(&mB, W2, d, k) ||
      !make_map_f32_out(&mC, P, d, T, p))
    return TP_ERR_CUDA;
  TcParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.n_total = static_cast<int32_t>(d);
  prm.s = static_cast<int32_t>(s);
  prm.p = p;
  prm.m_tiles = ceil_div(T, BM);
  prm.batches = p;
  prm.k_blocks = ceil_div(s, BK);
  prm.kb_per_shard = prm.k_blocks;
  prm.act = kActIdentity;
  prm.bias = nullptr;
  prm.out = P;
  const TileChoice tch = pick_tile(T, d, p, prm.k_blocks, c.num_sms, false, pair_allowed());
  if (rf != nullptr) *rf = RegionFold{};
  if (tch.pair) {
    if (region_cnt != nullptr && rf != nullptr) {
      // regions = the pair tiles (256 rows x bn columns); 8 epilogue warps
      // on each of the two CTAs count once per tile and shard
      prm.region_cnt = region_cnt;
      // Two halves of the m-tiles, all shards of the first half before the
      // second: the first half's regions complete mid-layer and are folded
      // while the tensor cores work on the second (each W2 panel is then
      // read once per half).
      const int32_t m_tiles = ceil_div(T, 2 * BM);
      prm.m_group = m_tiles >= 4 ? ceil_div(m_tiles, 2) : 0;
      *rf = RegionFold{region_cnt, 2 * BM, tch.bn, m_tiles, ceil_div(d, tch.bn),
                       2 * NUM_EPI_WARPS * p, prm.m_group};
    }
    return launch_tc_pair(c, kModeRowPartial, tch.bn, mA, mB, mB, mC, prm);
  }
  // Single-CTA row tiles (one wave on GPT-2, weight streaming on decode)
  // publish nothing: the fold beside them measured slower than the fold
  // after them.
  return launch_bn<kModeRowPartial>(c, tch.bn, mA, mB, mB, mC, prm);
}

tp_status launch_tc_row_chain(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                              const float* R, float* Z, int64_t T, int64_t k, int64_t d, int p,
                              int* region_cnt, bool* done) {
  *done = false;
  const int64_t s = k / p;
  TcParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.n_total = static_cast<int32_t>(d);
  prm.s = static_cast<int32_t>(s);
  prm.p = p;
  prm.m_tiles = ceil_div(T, BM);
  prm.batches = p;
  prm.k_blocks = ceil_div(s, BK);
  prm.kb_per_shard = prm.k_blocks;
  prm.act = kActIdentity;
  const TileChoice tch = pick_tile(T, d, p, prm.k_blocks, c.num_sms, false, pair_allowed());
  if (!tch.pair || region_cnt == nullptr) return TP_OK;   // the caller folds the partials
  CUtensorMap mA, mB, mZ, mR;
  if (!make_map_a(&mA, Y, s, T, p) || !make_map_b(&mB, W2, d, k) ||
      !make_map_f32_out(&mZ, Z, d, T, 1) ||
      (R != nullptr && !make_map_f32_out(&mR, const_cast<float*>(R), d, T, 1)))
    return TP_ERR_CUDA;
  prm.bias = b2;
  prm.out = Z;
  prm.resid = R != nullptr ? 1 : 0;
  prm.region_cnt = region_cnt;
  // Shards in order within each half of the m-tiles (as for the fold beside
  // the layer): a half's running sums, 128 T d bytes, are read and written
  // once per shard, so a half keeps them within reach of L2.
  const int32_t m_tiles = ceil_div(T, 2 * BM);
  prm.m_group = m_tiles >= 4 ? ceil_div(m_tiles, 2) : 0;
  const tp_status st = launch_tc_pair(c, kModeRowChain, tch.bn, mA, mB, mB, mZ, prm,
                                      R != nullptr ? &mR : nullptr);
  if (st == TP_ERR_UNSUPPORTED) return TP_OK;   // no cooperative launch of this grid here
  *done = st == TP_OK;
  return st;
}

tp_status launch_tc_row_splitk(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                               float* Z, int64_t T, int64_t k, int64_t d, int p) {
  const int64_t s = k / p;
  CUtensorMap mA, mB, mC;
  if (!make_map_a(&mA, Y, s, T, p) || !make_map_b(&mB, W2, d, k) ||
      !make_map_f32_out(&mC, Z, d, T, 1))
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
  const TileChoice tch = pick_tile(T, d, 1, prm.k_blocks, c.num_sms, false, pair_allowed());
  if (tch.pair) return launch_tc_pair(c, kModeRowSplitK, tch.bn, mA, mB, mB, mC, prm);
  return launch_bn<kModeRowSplitK>(c, tch.bn, mA, mB, mB, mC, prm);
}

}  // namespace tpk
