// Per-layer bf16 GEMM on CTA pairs (tcgen05 cta_group::2), sm_100a.
//
// Same layers and epilogues as tp_gemm_sm100.cu (column-parallel + bias +
// GELU/SwiGLU into the hidden shards, row-parallel fp32 partials, split-K
// over shards): a cluster of two CTAs computes a 256 x PBN tile (PBN 128 or
// 256).  Each CTA loads its own 128 rows of A and one half (PBN/2 columns) of
// B, and the even CTA's single MMA thread issues tcgen05.mma.cta_group::2
// M=256 N=PBN, which reads both CTAs' shared memory and writes each CTA's 128
// accumulator rows into that CTA's TMEM.  Per SM this halves the B operand
// bytes per MMA cycle (64 instead of 96 bytes per cycle at width 256).
//
// Synchronisation (all barrier waits bounded):
//   full[s]   on the even CTA: its expect_tx of both CTAs' bytes, completed by
//             both CTAs' TMA loads (cta_group::2 loads count on the even
//             CTA's barrier);
//   empty[s]  in each CTA: the MMA's commit multicast to both;
//   accf[b]   in each CTA: the MMA's commit multicast to both;
//   acce[b]   on the even CTA: one arrival per epilogue warp of both CTAs.
// No load uses cluster multicast: every CTA reads its own tiles.  Epilogues
// store through shared memory with TMA tensor stores, as in the single-CTA
// kernel.
//
// Launch-level options: a row layer of partials can publish per-tile
// completion counters for the fold that runs beside it (region_cnt, tiles
// taken in two halves of the m-tiles); a row layer can instead fold the
// shards itself (kModeRowChain: each shard's tile adds its partial to the
// running sum in Z once the counters show the previous shard's tile
// stored; a cooperative launch, so every pair it waits for is running);
// and a column layer can carry up to three weight/output segments of the
// same input (the attention block's Q, K and V in one launch; nseg).
#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <mutex>

#include "tp_gemm_parts.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

using namespace gemm;

constexpr int PBM = 2 * BM;  // rows of a pair tile

// Pair tile of PBN accumulator columns: each CTA holds PBN/2 columns of B.
template <int PBN, int EPI_BYTES_ = 0>
struct PCfg {
  static constexpr int EPI_BYTES = EPI_BYTES_;   // bulk-store staging (fp32 row layers)
  static constexpr int B_CHUNKS = PBN / 2 / B_BOX_COLS;
  static constexpr int STAGE_BYTES = A_BYTES + B_CHUNKS * B_CHUNK_BYTES;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - CTRL_BYTES - EPI_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + CTRL_BYTES;
  static constexpr int TMEM_COLS = 2 * PBN <= 256 ? 256 : 512;
  static constexpr uint32_t IDESC = idesc_bf16_f32(PBM, PBN, /*a_mn=*/0, /*b_mn=*/1);
  static_assert(PBN == 128 || PBN == 256, "pair tile width");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
  // barriers, TMEM slot + abort flag, then one barrier per epilogue warp (chain loads)
  static_assert(8 * (2 * STAGES + 5) + 16 + 8 * NUM_EPI_WARPS <= CTRL_BYTES, "control block");
};

// Loads of one slot for this CTA: A rows [m*256 + rank*128, +128), B columns
// [n*256 + rank*128, +128) of the layer's weight (SwiGLU: the even CTA loads
// the gate columns, the odd CTA the matching up columns).
template <int MODE, int PBN>
__device__ __forceinline__ void issue_slot_pair(const TcParams& P, const CUtensorMap* mA,
                                                const CUtensorMap* mB0, const CUtensorMap* mB1,
                                                const TileCoord& tc, int32_t kb, uint32_t rank,
                                                uint32_t sa, uint32_t sb, uint32_t bar) {
  constexpr int PB_CHUNKS = PCfg<PBN>::B_CHUNKS;
  const int32_t row0 = tc.m * PBM + static_cast<int32_t>(rank) * BM;
  if constexpr (MODE == kModeColumn) {
    tma_load_3d_pair(sa, mA, bar, kb * BK, row0, 0);
    const int32_t col0 = tc.n * PBN + static_cast<int32_t>(rank) * (PBN / 2);
#pragma unroll
    for (int c = 0; c < PB_CHUNKS; ++c)
      tma_load_2d_pair(sb + c * B_CHUNK_BYTES, mB0, bar, col0 + c * B_BOX_COLS, kb * BK);
  } else if constexpr (MODE == kModeColumnSwiglu) {
    tma_load_3d_pair(sa, mA, bar, kb * BK, row0, 0);
    const CUtensorMap* mB = rank == 0 ? mB0 : mB1;
    const int32_t col0 = tc.n * (PBN / 2);
#pragma unroll
    for (int c = 0; c < PB_CHUNKS; ++c)
      tma_load_2d_pair(sb + c * B_CHUNK_BYTES, mB, bar, col0 + c * B_BOX_COLS, kb * BK);
  } else if constexpr (MODE == kModeRowPartial || MODE == kModeRowChain) {
    tma_load_3d_pair(sa, mA, bar, kb * BK, row0, tc.batch);
    const int32_t col0 = tc.n * PBN + static_cast<int32_t>(rank) * (PBN / 2);
#pragma unroll
    for (int c = 0; c < PB_CHUNKS; ++c)
      tma_load_2d_pair(sb + c * B_CHUNK_BYTES, mB0, bar, col0 + c * B_BOX_COLS,
                       tc.batch * P.s + kb * BK);
  } else {
    const int32_t shard = kb / P.kb_per_shard;
    const int32_t kin = kb - shard * P.kb_per_shard;
    tma_load_3d_pair(sa, mA, bar, kin * BK, row0, shard);
    const int32_t col0 = tc.n * PBN + static_cast<int32_t>(rank) * (PBN / 2);
#pragma unroll
    for (int c = 0; c < PB_CHUNKS; ++c)
      tma_load_2d_pair(sb + c * B_CHUNK_BYTES, mB0, bar, col0 + c * B_BOX_COLS, kb * BK);
  }
}

template <int MODE>
constexpr bool kPairBulkOut = (MODE == kModeRowPartial || MODE == kModeRowSplitK);

// One lane waits until *cnt reaches target (acquire at GPU scope), bounded;
// false, with the CTA's abort flag and kErrWaitRegion set, when it does not.
__device__ __forceinline__ bool wait_count(const int* cnt, int target, volatile int* abort,
                                           const WaitCtl& w) {
  if (ld_acquire_gpu(cnt) >= target) return true;
  const uint64_t t0 = globaltimer_ns();
  while (true) {
    __nanosleep(200);
    if (ld_acquire_gpu(cnt) >= target) return true;
    if (*abort) return false;
    if (globaltimer_ns() - t0 > w.timeout_ns) {
      *abort = 1;
      atomicOr(w.err, kErrWaitRegion);
      return false;
    }
  }
}

// Chain fold of a row layer (kModeRowChain): the tile of shard s adds its
// partial to the running sum that shard s-1's tile of the same rows and
// columns left in Z, and the last shard adds b2 (then R with P.resid), so
// Z = (((P_0 + P_1) + ... + P_{p-1}) + b2) + R with one fp32 RNE addition
// per element in that order -- the fixed-order fold -- and no partials reach
// memory.  The warp waits (once per tile) for the region counter to show
// all earlier shards' tiles stored; then per 32 x 32 chunk the previous sum
// comes into the warp's staging tile by a TMA load (128-byte swizzle, the
// store's layout), each lane adds its row of the accumulator to its row of
// the chunk, and a TMA store writes the new sum back.  False if a wait gave
// up.
template <int PBN>
__device__ __forceinline__ bool epilogue_tile_chain(const TcParams& P, const TileCoord& tc,
                                                    uint32_t tacc, int32_t row0, int half,
                                                    uint32_t stage, uint32_t bar, uint32_t& ph,
                                                    const CUtensorMap* mapZ, const CUtensorMap* mapR,
                                                    volatile int* abort, int lane) {
  const float* __restrict__ b2 = static_cast<const float*>(P.bias);
  const bool first = tc.batch == 0;
  const bool last = tc.batch == P.p - 1;
  if (!first) {
    bool ok = true;
    if (lane == 0) {
      ok = wait_count(P.region_cnt + tc.n * P.m_tiles + tc.m, 2 * NUM_EPI_WARPS * tc.batch, abort,
                      P.wait);
      // the TMA loads below read, in the async proxy, what the acquire made visible
      fence_proxy_async_global();
    }
    if (!__shfl_sync(0xffffffffu, ok ? 1 : 0, 0)) return false;
  }
#pragma unroll 1
  for (int q = 0; q < PBN / 64; ++q) {
    const int c0 = half * (PBN / 2) + q * 32;
    const int32_t j0 = tc.n * PBN + c0;
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + c0, v);
    tmem_ld_wait();
    if (j0 >= P.n_total) continue;   // warp-uniform
    // the staging tile is free once the previous store has read it
    if (lane == 0) bulk_wait_read0();
    __syncwarp();
    if (!first) {
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, 32 * 32 * 4);
        tma_load_3d(stage, mapZ, bar, j0, row0, 0);
      }
      // not abortable: the load must land before the staging tile is reused
      if (!wait_teardown(bar, ph, P.wait)) return false;
      ph ^= 1u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t addr = stage + lane * 128 + ((c ^ (lane & 7)) << 4);
        uint32_t z0, z1, z2, z3;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(z0), "=r"(z1), "=r"(z2), "=r"(z3)
                     : "r"(addr)
                     : "memory");
        v[4 * c + 0] = __float_as_uint(__fadd_rn(__uint_as_float(z0), __uint_as_float(v[4 * c + 0])));
        v[4 * c + 1] = __float_as_uint(__fadd_rn(__uint_as_float(z1), __uint_as_float(v[4 * c + 1])));
        v[4 * c + 2] = __float_as_uint(__fadd_rn(__uint_as_float(z2), __uint_as_float(v[4 * c + 2])));
        v[4 * c + 3] = __float_as_uint(__fadd_rn(__uint_as_float(z3), __uint_as_float(v[4 * c + 3])));
      }
    }
    if (last && b2 != nullptr) {
#pragma unroll
      for (int e = 0; e < 32; ++e)
        v[e] = __float_as_uint(
            __fadd_rn(__uint_as_float(v[e]), j0 + e < P.n_total ? __ldg(b2 + j0 + e) : 0.0f));
    }
    if (last && P.resid) {
      __syncwarp();   // every lane has read the previous sum out of the staging tile
      if (lane == 0) {
        mbar_arrive_expect_tx(bar, 32 * 32 * 4);
        tma_load_3d(stage, mapR, bar, j0, row0, 0);
      }
      if (!wait_teardown(bar, ph, P.wait)) return false;
      ph ^= 1u;
#pragma unroll
      for (int c = 0; c < 8; ++c) {
        const uint32_t addr = stage + lane * 128 + ((c ^ (lane & 7)) << 4);
        uint32_t r0, r1, r2, r3;
        asm volatile("ld.shared.v4.b32 {%0, %1, %2, %3}, [%4];"
                     : "=r"(r0), "=r"(r1), "=r"(r2), "=r"(r3)
                     : "r"(addr)
                     : "memory");
        v[4 * c + 0] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * c + 0]), __uint_as_float(r0)));
        v[4 * c + 1] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * c + 1]), __uint_as_float(r1)));
        v[4 * c + 2] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * c + 2]), __uint_as_float(r2)));
        v[4 * c + 3] = __float_as_uint(__fadd_rn(__uint_as_float(v[4 * c + 3]), __uint_as_float(r3)));
      }
    }
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
      tma_store_3d(mapZ, stage, j0, row0, 0);
      bulk_commit();
    }
  }
  return true;
}

// Tile t of the launch and its segment (0 unless several column layers share
// the launch; within a segment m fastest, as decode_tile walks one layer).
__device__ __forceinline__ TileCoord decode_pair_tile(const TcParams& P, int32_t t, int& seg) {
  seg = 0;
  if (P.nseg <= 1) return decode_tile(P, t);
  while (seg + 1 < P.nseg && t >= P.seg_start[seg + 1]) ++seg;
  const int32_t r = t - P.seg_start[seg];
  TileCoord c;
  c.batch = 0;
  c.n = r / P.m_tiles;
  c.m = r - c.n * P.m_tiles;
  return c;
}

template <int MODE, int PBN>
using PKCfg = PCfg<PBN, EPI_STAGE_BYTES>;

template <int MODE, int PBN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_pair_kernel(const __grid_constant__ CUtensorMap mapA,
                        const __grid_constant__ CUtensorMap mapB0,
                        const __grid_constant__ CUtensorMap mapB1,
                        const __grid_constant__ CUtensorMap mapC, const TcParams P,
                        const __grid_constant__ CUtensorMap mapB2,
                        const __grid_constant__ CUtensorMap mapC1,
                        const __grid_constant__ CUtensorMap mapC2) {
  using C = PKCfg<MODE, PBN>;
  constexpr int PSTAGES = C::STAGES;
  constexpr int PSTAGE_BYTES = C::STAGE_BYTES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t epi_stage = base + PSTAGES * PSTAGE_BYTES;   // C::EPI_BYTES of staging
  uint8_t* const ctrl = smem_raw + (base - raw) + PSTAGES * PSTAGE_BYTES + C::EPI_BYTES;
  uint64_t* const bars = reinterpret_cast<uint64_t*>(ctrl);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (2 * PSTAGES + 5));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);
  uint64_t* const chain_bars = reinterpret_cast<uint64_t*>(ctrl + 8 * (2 * PSTAGES + 5) + 16);

  auto full_bar = [&](uint32_t s) { return smem_u32(&bars[s]); };
  auto empty_bar = [&](uint32_t s) { return smem_u32(&bars[PSTAGES + s]); };
  auto accf_bar = [&](uint32_t b) { return smem_u32(&bars[2 * PSTAGES + b]); };
  auto acce_bar = [&](uint32_t b) { return smem_u32(&bars[2 * PSTAGES + 2 + b]); };
  const uint32_t drain_bar = smem_u32(&bars[2 * PSTAGES + 4]);
  auto slot_a = [&](uint32_t s) { return base + s * PSTAGE_BYTES; };
  auto slot_b = [&](uint32_t s) { return base + s * PSTAGE_BYTES + A_BYTES; };

  const int warp = threadIdx.x / 32;
  const int lane = threadIdx.x % 32;
  const uint32_t rank = cluster_ctarank();
  const int32_t cluster = blockIdx.x / 2;
  const int32_t nclusters = gridDim.x / 2;

  if (threadIdx.x == 0) {
    for (int s = 0; s < PSTAGES; ++s) {
      mbar_init(full_bar(s), 1);
      mbar_init(empty_bar(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(accf_bar(b), 1);
      mbar_init(acce_bar(b), 2 * NUM_EPI_WARPS);
    }
    mbar_init(drain_bar, 1);
    for (int w = 0; w < NUM_EPI_WARPS; ++w) mbar_init(smem_u32(&chain_bars[w]), 1);
    *abort_flag = 0;
    fence_barrier_init();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapA);
    tma_prefetch_map(&mapB0);
    if (MODE == kModeColumnSwiglu) tma_prefetch_map(&mapB1);
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
  zero_counters(P, warp, lane);
  pdl_launch_dependents();

  if (warp == 0) {
    if (lane == 0) {
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int32_t t = cluster; ok && t < P.num_tiles; t += nclusters) {
        int seg;
        const TileCoord tc = decode_pair_tile(P, t, seg);
        // several column layers in one launch: segment seg's weight
        const CUtensorMap* mB0 = seg == 0 ? &mapB0 : (seg == 1 ? &mapB1 : &mapB2);
        for (int32_t kb = 0; kb < P.k_blocks; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, P.wait, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          // fault injection (tests of the bounded waits): the first pair only
          if (issued != P.debug_drop || cluster != 0) {
            if (rank == 0) mbar_arrive_expect_tx(full_bar(stage), 2 * PSTAGE_BYTES);
            issue_slot_pair<MODE, PBN>(P, &mapA, mB0, &mapB1, tc, kb, rank, slot_a(stage),
                                  slot_b(stage), mapa_shared(full_bar(stage), 0));
          }
          ++issued;
          if (++stage == PSTAGES) {
            stage = 0;
            phase ^= 1u;
          }
        }
      }
      // Teardown: our last loads must have landed before this CTA's shared
      // memory is released.  The even CTA sees that on its full barriers; the
      // odd CTA on its empty barriers (the MMA consumed the slot).
      const int64_t first = issued > PSTAGES ? issued - PSTAGES : 0;
      for (int64_t q = first; q < issued; ++q) {
        if (q == P.debug_drop && cluster == 0) continue;
        const uint32_t s = static_cast<uint32_t>(q % PSTAGES);
        const uint32_t ph = static_cast<uint32_t>((q / PSTAGES) & 1);
        wait_teardown(rank == 0 ? full_bar(s) : empty_bar(s), ph, P.wait);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0 && rank == 0) {
      // ---------------------------------------------------- MMA issuer (pair)
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
            const uint64_t adesc = smem_desc_sw128(sa + kk * UK * 2, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sb + kk * UK * 128, B_CHUNK_BYTES, 1024);
            tc_mma_f16_pair(d_tmem, adesc, bdesc, C::IDESC, (kb > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit_pair_mc(empty_bar(stage), 0x3);
          if (++stage == PSTAGES) {
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
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;
    uint32_t nchunk = 0;   // bf16 chunks this warp has staged (alternating halves)
    uint32_t chain_ph = 0;   // phase of this warp's chain-load barrier
    const uint32_t chain_bar = smem_u32(&chain_bars[warp - 4]);
    int32_t lt = 0;
    for (int32_t t = cluster; t < P.num_tiles; t += nclusters, ++lt) {
      const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
      int seg;
      const TileCoord tc = decode_pair_tile(P, t, seg);
      TcParams SP = P;   // the segment's width and shard width
      if (P.nseg > 1) {
        SP.n_total = P.seg_n[seg];
        SP.s = P.seg_s[seg];
      }
      const CUtensorMap* mC = seg == 0 ? &mapC : (seg == 1 ? &mapC1 : &mapC2);
      EpiBias<MODE, PBN> eb;
      load_epi_bias<MODE, PBN>(SP, tc, half, eb);
      bool ok = wait_bounded(accf_bar(b), ap, abort_flag, P.wait, kErrWaitAccFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * PBN;
      const int row0 = tc.m * PBM + static_cast<int>(rank) * BM + quad * 32;
      const uint32_t stage_w = epi_stage + (warp - 4) * EPI_WARP_STAGE_BYTES;
      if constexpr (MODE == kModeRowChain) {
        if (!epilogue_tile_chain<PBN>(P, tc, tacc, row0, half, stage_w, chain_bar, chain_ph,
                                      &mapC, &mapC1, abort_flag, lane))
          break;   // a wait gave up (error bit set); the MMA's waits end on the abort flag
      } else if constexpr (kPairBulkOut<MODE>) {
        epilogue_tile_bulk<MODE, PBN>(P, tc, tacc, row0, half, stage_w, &mapC, lane);
      } else {
        if (P.bulk_out)
          epilogue_tile_bulk_col<MODE, PBN>(SP, tc, tacc, row0, half, eb, stage_w, mC, lane,
                                            nchunk);
        else
          epilogue_tile<MODE, PBN>(SP, tc, tacc, row0 + lane, half, eb);
      }
      tc_fence_before();
      __syncwarp();
      if (lane == 0) mbar_arrive_cluster(mapa_shared(acce_bar(b), 0));
      if constexpr (MODE == kModeRowPartial || MODE == kModeRowChain) {
        if (P.region_cnt != nullptr) {
          // Publish this warp's part of the tile to the overlapped fold: its
          // bulk stores complete, are ordered for generic-proxy readers, and
          // one release increment counts them (16 per tile and shard).  The
          // accumulator was handed back above, so the wait delays no MMA.
          if (lane == 0) {
            bulk_wait_all0();
            fence_proxy_async_global();
            red_release_gpu_add(P.region_cnt + tc.n * P.m_tiles + tc.m, 1);
          }
          __syncwarp();
        }
      }
    }
    // the staging tiles must be read out before shared memory is released
    if (lane == 0) bulk_wait_all0();
  }

  tc_fence_before();
  cluster_sync();  // the pair's MMAs, commits and arrivals are done with both CTAs
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc_pair(tmem_base, C::TMEM_COLS);
  }
}

}  // namespace

template <int MODE, int PBN>
tp_status launch_pair_mode(const LaunchCtx& c, const CUtensorMap& a, const CUtensorMap& b0,
                           const CUtensorMap& b1, const CUtensorMap& cm, TcParams prm,
                           const CUtensorMap* b2 = nullptr, const CUtensorMap* c1 = nullptr,
                           const CUtensorMap* c2 = nullptr) {
  constexpr int PSMEM_BYTES = PKCfg<MODE, PBN>::SMEM_BYTES;
  // The chain row layer's tiles wait for other tiles of the same grid, so it
  // is launched cooperatively: all its CTAs are then resident together and
  // every such wait ends, whatever else runs on the GPU.  (Without
  // programmatic serialization: it starts after the layer before it ends.)
  const bool kCoop = (MODE == kModeRowChain) && coop_allowed();
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static int max_coop_clusters[64] = {};  // co-resident clusters of a cooperative launch
  static std::mutex mu;
  int clusters = c.num_sms / 2;
  if (clusters > prm.num_tiles) clusters = prm.num_tiles;
  cudaLaunchConfig_t cfg = {};
  cfg.gridDim = dim3(2 * clusters);
  cfg.blockDim = dim3(NUM_THREADS);
  cfg.dynamicSmemBytes = PSMEM_BYTES;
  cfg.stream = c.stream;
  cudaLaunchAttribute attr[2];
  attr[0].id = cudaLaunchAttributeClusterDimension;
  attr[0].val.clusterDim.x = 2;
  attr[0].val.clusterDim.y = 1;
  attr[0].val.clusterDim.z = 1;
  cfg.attrs = attr;
  cfg.numAttrs = 1;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_gemm_pair_kernel<MODE, PBN>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               PSMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      max_coop_clusters[dev] = 0;
      if (kCoop) {
        int coop = 0, n = 0;
        if (cudaDeviceGetAttribute(&coop, cudaDevAttrCooperativeLaunch, c.device) == cudaSuccess &&
            coop != 0 &&
            cudaOccupancyMaxActiveClusters(&n, tc_gemm_pair_kernel<MODE, PBN>, &cfg) == cudaSuccess)
          max_coop_clusters[dev] = n;
        (void)cudaGetLastError();
      }
      attr_epoch[dev] = c.epoch;
    }
    if (kCoop) {
      // as many clusters as can be resident together (the tiles are taken
      // round-robin by however many there are); none: nothing is enqueued
      // and the caller folds another way
      if (max_coop_clusters[dev] < 1) return TP_ERR_UNSUPPORTED;
      if (clusters > max_coop_clusters[dev]) clusters = max_coop_clusters[dev];
      cfg.gridDim = dim3(2 * clusters);
    }
  }
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  if (kCoop) {
    attr[1].id = cudaLaunchAttributeCooperative;
    attr[1].val.cooperative = 1;
    cfg.numAttrs = 2;
  } else if (pdl_allowed()) {
    attr[1].id = cudaLaunchAttributeProgrammaticStreamSerialization;
    attr[1].val.programmaticStreamSerializationAllowed = 1;
    cfg.numAttrs = 2;
  }
  const cudaError_t e = cudaLaunchKernelEx(&cfg, tc_gemm_pair_kernel<MODE, PBN>, a, b0, b1, cm, prm,
                                           b2 != nullptr ? *b2 : b0, c1 != nullptr ? *c1 : cm,
                                           c2 != nullptr ? *c2 : cm);
  if (kCoop && (e == cudaErrorCooperativeLaunchTooLarge || e == cudaErrorNotSupported)) {
    // refused before anything ran: no cooperative launches of this grid on
    // this context; the caller folds another way
    (void)cudaGetLastError();
    std::lock_guard<std::mutex> lk(mu);
    max_coop_clusters[c.device & 63] = 0;
    return TP_ERR_UNSUPPORTED;
  }
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("paired GEMM launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

// Tile space of the pair kernel for a layer: 256-row m-tiles, `pbn`-column
// (SwiGLU: pbn/2 output columns) n-tiles.
tp_status launch_tc_pair(const LaunchCtx& c, int mode, int pbn, const CUtensorMap& a,
                         const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& cm,
                         TcParams prm, const CUtensorMap* c1) {
  const int out_cols = mode == kModeColumnSwiglu ? pbn / 2 : pbn;
  prm.m_tiles = ceil_div(prm.T, PBM);
  prm.n_tiles = ceil_div(prm.n_total, out_cols);
  prm.num_tiles = prm.m_tiles * prm.n_tiles * prm.batches;
  if (pbn == 128) {
    switch (mode) {
      case kModeColumn: return launch_pair_mode<kModeColumn, 128>(c, a, b0, b1, cm, prm);
      case kModeColumnSwiglu: return launch_pair_mode<kModeColumnSwiglu, 128>(c, a, b0, b1, cm, prm);
      case kModeRowPartial: return launch_pair_mode<kModeRowPartial, 128>(c, a, b0, b1, cm, prm);
      case kModeRowChain:
        return launch_pair_mode<kModeRowChain, 128>(c, a, b0, b1, cm, prm, nullptr, c1);
      default: return launch_pair_mode<kModeRowSplitK, 128>(c, a, b0, b1, cm, prm);
    }
  }
  switch (mode) {
    case kModeColumn: return launch_pair_mode<kModeColumn, 256>(c, a, b0, b1, cm, prm);
    case kModeColumnSwiglu: return launch_pair_mode<kModeColumnSwiglu, 256>(c, a, b0, b1, cm, prm);
    case kModeRowPartial: return launch_pair_mode<kModeRowPartial, 256>(c, a, b0, b1, cm, prm);
    case kModeRowChain:
      return launch_pair_mode<kModeRowChain, 256>(c, a, b0, b1, cm, prm, nullptr, c1);
    default: return launch_pair_mode<kModeRowSplitK, 256>(c, a, b0, b1, cm, prm);
  }
}

// Several column layers (identity activation, no bias) of one input in one
// launch of 256 x 256 pair tiles: weight maps b[i], output maps cm[i], k[i]
// output columns on prm.p shards; the segments' tiles follow each other.
tp_status launch_tc_pair_column_multi(const LaunchCtx& c, int pbn, const CUtensorMap& a,
                                      const CUtensorMap* b, const CUtensorMap* cm,
                                      const int64_t* k, int nseg, TcParams prm) {
  prm.m_tiles = ceil_div(prm.T, PBM);
  int32_t start = 0;
  for (int i = 0; i < nseg; ++i) {
    prm.seg_start[i] = start;
    prm.seg_n[i] = static_cast<int32_t>(k[i]);
    prm.seg_s[i] = static_cast<int32_t>(k[i] / prm.p);
    start += prm.m_tiles * ceil_div(k[i], pbn);
  }
  prm.seg_start[nseg] = start;
  prm.nseg = nseg;
  prm.n_tiles = 0;   // per segment: (seg_start[i+1] - seg_start[i]) / m_tiles
  prm.num_tiles = start;
  const CUtensorMap& b1 = nseg > 1 ? b[1] : b[0];
  const CUtensorMap* b2 = nseg > 2 ? &b[2] : &b[0];
  const CUtensorMap* c1 = nseg > 1 ? &cm[1] : &cm[0];
  const CUtensorMap* c2 = nseg > 2 ? &cm[2] : &cm[0];
  if (pbn == 128) return launch_pair_mode<kModeColumn, 128>(c, a, b[0], b1, cm[0], prm, b2, c1, c2);
  return launch_pair_mode<kModeColumn, 256>(c, a, b[0], b1, cm[0], prm, b2, c1, c2);
}

}  // namespace tpk
