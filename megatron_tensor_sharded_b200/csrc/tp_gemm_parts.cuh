// Device-side pieces shared by the tensor-core kernels (the per-layer GEMM
// in tp_gemm_sm100.cu and the fused block in tp_block_sm100.cu): tile
// configuration, tile decoding, TMA slot issue and the epilogues.
#pragma once

#include <cuda.h>
#include <cuda_bf16.h>

#include <cstdint>
#include <cstring>

#include "tp_act.cuh"
#include "tp_device.cuh"
#include "tp_internal.h"

namespace tpk {
namespace gemm {

constexpr int BM = 128;                     // tile rows = UMMA M
constexpr int BK = 64;                      // k per slot: 64 bf16 = one 128-byte swizzle row
constexpr int UK = 16;                      // k per tcgen05.mma (16-bit inputs)
constexpr int A_BYTES = BM * BK * 2;        // 16 KiB
constexpr int B_BOX_COLS = 64;              // one swizzle atom wide
constexpr int B_CHUNK_BYTES = BK * B_BOX_COLS * 2;  // 8 KiB
constexpr int NUM_EPI_WARPS = 8;
constexpr int NUM_THREADS = 128 + 32 * NUM_EPI_WARPS;
constexpr int CTRL_BYTES = 256;
constexpr int SMEM_LIMIT = 232448;          // max dynamic shared memory per block

// Staging for the bulk-store epilogue of the fp32 row layers: one 32 x 32
// fp32 tile (4 KiB, a 128-byte swizzle pattern of 32 rows) per epilogue warp.
constexpr int EPI_WARP_STAGE_BYTES = 32 * 32 * 4;
constexpr int EPI_STAGE_BYTES = NUM_EPI_WARPS * EPI_WARP_STAGE_BYTES;

template <int BN_, int EPI_BYTES_ = 0>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr int EPI_BYTES = EPI_BYTES_;   // after the stages, before the control block
  static constexpr int B_CHUNKS = BN / B_BOX_COLS;
  static constexpr int B_BYTES = B_CHUNKS * B_CHUNK_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - CTRL_BYTES - EPI_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + EPI_BYTES + CTRL_BYTES;
  static constexpr uint32_t IDESC = idesc_bf16_f32(BM, BN, /*a_mn=*/0, /*b_mn=*/1);
  static_assert(BN % 64 == 0 && BN >= 64 && BN <= 256, "tile width");
  static_assert(SMEM_BYTES <= SMEM_LIMIT, "shared memory budget");
  static_assert(8 * (2 * STAGES + 5) + 16 <= CTRL_BYTES, "control block");
};

enum Mode : int { kModeColumn = 0, kModeColumnSwiglu = 1, kModeRowPartial = 2, kModeRowSplitK = 3 };

struct TcParams {
  int32_t T;             // tokens
  int32_t n_total;       // valid output columns: k (column) or d (row)
  int32_t s;             // shard width k/p
  int32_t p;
  int32_t m_tiles, n_tiles, batches, num_tiles;
  int32_t k_blocks;      // pipeline slots per tile
  int32_t kb_per_shard;  // split-K: slots per shard (s / 64)
  int32_t act;
  const void* bias;      // b1 (bf16, column) or b2 (fp32, split-K row); may be null
  void* out;             // Y bf16 [p][T][s] | P fp32 [p][T][d] | Z fp32 [T][d]
  int32_t bulk_out;      // column layers: 1 = bulk tensor stores through shared memory
  WaitCtl wait;
  int64_t debug_drop;    // slot (in issue order) whose load is skipped; -1 none
};

struct TileCoord {
  int32_t batch, m, n;
};

__device__ __forceinline__ TileCoord decode_tile(const TcParams& P, int32_t t) {
  const int32_t per_batch = P.m_tiles * P.n_tiles;
  TileCoord c;
  c.batch = t / per_batch;
  const int32_t r = t - c.batch * per_batch;
  c.n = r / P.m_tiles;   // m fastest: neighbouring CTAs share the weight panel
  c.m = r - c.n * P.m_tiles;
  return c;
}

template <int MODE, int BN>
__device__ __forceinline__ void issue_slot(const TcParams& P, const CUtensorMap* mA,
                                           const CUtensorMap* mB0, const CUtensorMap* mB1,
                                           const TileCoord& tc, int32_t kb, uint32_t sa,
                                           uint32_t sb, uint32_t bar) {
  constexpr int NCH = BN / B_BOX_COLS;
  const int32_t row0 = tc.m * BM;
  if constexpr (MODE == kModeColumn) {
    tma_load_3d(sa, mA, bar, kb * BK, row0, 0);
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      tma_load_2d(sb + c * B_CHUNK_BYTES, mB0, bar, tc.n * BN + c * B_BOX_COLS, kb * BK);
  } else if constexpr (MODE == kModeColumnSwiglu) {
    tma_load_3d(sa, mA, bar, kb * BK, row0, 0);
    const int32_t col0 = tc.n * (BN / 2);
#pragma unroll
    for (int c = 0; c < NCH / 2; ++c) {
      tma_load_2d(sb + c * B_CHUNK_BYTES, mB0, bar, col0 + c * B_BOX_COLS, kb * BK);
      tma_load_2d(sb + (c + NCH / 2) * B_CHUNK_BYTES, mB1, bar, col0 + c * B_BOX_COLS, kb * BK);
    }
  } else if constexpr (MODE == kModeRowPartial) {
    tma_load_3d(sa, mA, bar, kb * BK, row0, tc.batch);
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      tma_load_2d(sb + c * B_CHUNK_BYTES, mB0, bar, tc.n * BN + c * B_BOX_COLS,
                  tc.batch * P.s + kb * BK);
  } else {  // split-K over shards: slot kb covers hidden columns [kb*64, kb*64+64)
    const int32_t shard = kb / P.kb_per_shard;
    const int32_t kin = kb - shard * P.kb_per_shard;
    tma_load_3d(sa, mA, bar, kin * BK, row0, shard);
#pragma unroll
    for (int c = 0; c < NCH; ++c)
      tma_load_2d(sb + c * B_CHUNK_BYTES, mB0, bar, tc.n * BN + c * B_BOX_COLS, kb * BK);
  }
}

__device__ __forceinline__ float bf16_bits_to_float(uint16_t b) {
  return __uint_as_float(static_cast<uint32_t>(b) << 16);
}

__device__ __forceinline__ uint32_t pack_bf16x2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}

// 8 consecutive output columns j..j+7 of one row, bf16, into shard storage.
__device__ __forceinline__ void store_bf16x8(const TcParams& P, int row, int32_t j,
                                             const float (&y)[8]) {
  const int32_t shard = j / P.s;
  const int32_t jj = j - shard * P.s;
  const uint4 pk = make_uint4(pack_bf16x2(y[0], y[1]), pack_bf16x2(y[2], y[3]),
                              pack_bf16x2(y[4], y[5]), pack_bf16x2(y[6], y[7]));
  __nv_bfloat16* __restrict__ Y = static_cast<__nv_bfloat16*>(P.out);
  *reinterpret_cast<uint4*>(Y + (static_cast<int64_t>(shard) * P.T + row) * P.s + jj) = pk;
}

// 32-column chunks one epilogue warp handles per tile (it owns half of the
// accumulator's output columns).
template <int MODE, int BN>
struct EpiShape {
  static constexpr bool kColumn = (MODE == kModeColumn || MODE == kModeColumnSwiglu);
  static constexpr int kOutCols = (MODE == kModeColumnSwiglu) ? BN / 2 : BN;  // per tile
  static constexpr int kChunks = kOutCols / 64;                                // per warp
};

// The b1 values (bf16) a warp's column epilogue needs for one tile, loaded as
// 16-byte vectors before the accumulator is waited for, so the whole tile
// costs one memory latency, hidden behind the main loop.
template <int MODE, int BN>
struct EpiBias {
  static constexpr int N = EpiShape<MODE, BN>::kColumn ? EpiShape<MODE, BN>::kChunks * 4 : 1;
  uint4 v[N];
};

template <int MODE, int BN>
__device__ __forceinline__ void load_epi_bias(const TcParams& P, const TileCoord& tc, int half,
                                              EpiBias<MODE, BN>& eb) {
  using S = EpiShape<MODE, BN>;
  if constexpr (S::kColumn) {
    const uint16_t* __restrict__ bias = static_cast<const uint16_t*>(P.bias);
    if (bias == nullptr) return;
#pragma unroll
    for (int q = 0; q < S::kChunks; ++q) {
      const int32_t j0 = tc.n * S::kOutCols + half * (S::kOutCols / 2) + q * 32;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int32_t j = j0 + g * 8;
        eb.v[q * 4 + g] = j < P.n_total ? __ldg(reinterpret_cast<const uint4*>(bias + j))
                                        : make_uint4(0u, 0u, 0u, 0u);
      }
    }
  }
}

__device__ __forceinline__ void unpack_bf16x8(const uint4& u, float (&f)[8]) {
  const uint32_t w[4] = {u.x, u.y, u.z, u.w};
#pragma unroll
  for (int i = 0; i < 4; ++i) {
    f[2 * i] = __uint_as_float(w[i] << 16);
    f[2 * i + 1] = __uint_as_float(w[i] & 0xFFFF0000u);
  }
}

// Epilogue of one tile for one warp: TMEM lanes of `tacc`'s quadrant, the
// warp's half of the output columns.  `row` is this thread's output row.
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_tile(const TcParams& P, const TileCoord& tc,
                                              uint32_t tacc, int row, int half,
                                              const EpiBias<MODE, BN>& eb) {
  using S = EpiShape<MODE, BN>;
  const bool row_ok = row < P.T;
  if constexpr (MODE == kModeColumn) {
    const bool has_bias = P.bias != nullptr;
    // unrolled: the prefetched bias registers are indexed by chunk
#pragma unroll
    for (int q = 0; q < S::kChunks; ++q) {
      const int c0 = half * (BN / 2) + q * 32;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + c0, v);
      tmem_ld_wait();
      if (!row_ok) continue;
      const int32_t j0 = tc.n * BN + c0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int32_t j = j0 + g * 8;
        if (j >= P.n_total) break;
        float bv[8];
        unpack_bf16x8(eb.v[q * 4 + g], bv);
        float h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          h[e] = __uint_as_float(v[g * 8 + e]);
          if (has_bias) h[e] += bv[e];
          h[e] = act_unary_mufu(P.act, h[e]);
        }
        store_bf16x8(P, row, j, h);
      }
    }
  } else if constexpr (MODE == kModeColumnSwiglu) {
    const bool has_bias = P.bias != nullptr;
#pragma unroll
    for (int q = 0; q < S::kChunks; ++q) {
      const int c0 = half * (BN / 4) + q * 32;   // gate column inside the accumulator
      uint32_t g32[32], u32[32];
      tmem_ld_32x32b_x32(tacc + c0, g32);
      tmem_ld_32x32b_x32(tacc + BN / 2 + c0, u32);
      tmem_ld_wait();
      if (!row_ok) continue;
      const int32_t j0 = tc.n * (BN / 2) + c0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int32_t j = j0 + g * 8;
        if (j >= P.n_total) break;
        float bv[8];
        unpack_bf16x8(eb.v[q * 4 + g], bv);
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float gate = __uint_as_float(g32[g * 8 + e]);
          if (has_bias) gate += bv[e];
          y[e] = silu_mufu(gate) * __uint_as_float(u32[g * 8 + e]);
        }
        store_bf16x8(P, row, j, y);
      }
    }
  } else {
    const float* __restrict__ bias = static_cast<const float*>(P.bias);
    float* __restrict__ out = static_cast<float*>(P.out);
    const int64_t plane = (MODE == kModeRowPartial) ? static_cast<int64_t>(tc.batch) * P.T : 0;
#pragma unroll 1
    for (int q = 0; q < S::kChunks; ++q) {
      const int c0 = half * (BN / 2) + q * 32;
      const int32_t j0 = tc.n * BN + c0;
      // b2 (split-K): issue the loads before the TMEM load so the latencies overlap
      float bv[32];
      if (MODE == kModeRowSplitK && bias != nullptr) {
#pragma unroll
        for (int e = 0; e < 32; ++e) bv[e] = (j0 + e < P.n_total) ? __ldg(bias + j0 + e) : 0.0f;
      }
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + c0, v);
      tmem_ld_wait();
      if (!row_ok) continue;
      float* dst = out + (plane + row) * static_cast<int64_t>(P.n_total);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int32_t j = j0 + g * 4;
        if (j >= P.n_total) break;
        float4 o = make_float4(__uint_as_float(v[g * 4 + 0]), __uint_as_float(v[g * 4 + 1]),
                               __uint_as_float(v[g * 4 + 2]), __uint_as_float(v[g * 4 + 3]));
        if (MODE == kModeRowSplitK && bias != nullptr) {
          o.x = __fadd_rn(o.x, bv[g * 4 + 0]);
          o.y = __fadd_rn(o.y, bv[g * 4 + 1]);
          o.z = __fadd_rn(o.z, bv[g * 4 + 2]);
          o.w = __fadd_rn(o.w, bv[g * 4 + 3]);
        }
        *reinterpret_cast<float4*>(dst + j) = o;
      }
    }
  }
}

// Bulk-store epilogue of the fp32 row layers (partials [p][T][d], or split-K
// Z [T][d] + b2): for each 32-column chunk the warp moves its 32 rows from
// TMEM to registers, writes them into its 4 KiB staging tile in the 128-byte
// swizzled layout (16-byte chunk c of row r at c ^ (r % 8): no bank
// conflicts), and one lane issues a TMA tensor store of the 32 x 32 box.
// Whole cache lines leave the SM instead of 16-byte pieces of 32 rows per
// instruction.  The box is clipped at T and d by the tensor map.  `row0` is
// the warp's first output row; the caller waits for the last stores
// (bulk_wait_all0) before the CTA's shared memory is released.
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_tile_bulk(const TcParams& P, const TileCoord& tc,
                                                   uint32_t tacc, int32_t row0, int half,
                                                   uint32_t stage, const CUtensorMap* mapC,
                                                   int lane) {
  const float* __restrict__ bias = static_cast<const float*>(P.bias);
#pragma unroll 1
  for (int q = 0; q < BN / 64; ++q) {
    const int c0 = half * (BN / 2) + q * 32;
    const int32_t j0 = tc.n * BN + c0;
    float bv[32];
    if (MODE == kModeRowSplitK && bias != nullptr) {
#pragma unroll
      for (int e = 0; e < 32; ++e) bv[e] = (j0 + e < P.n_total) ? __ldg(bias + j0 + e) : 0.0f;
    }
    uint32_t v[32];
    tmem_ld_32x32b_x32(tacc + c0, v);
    tmem_ld_wait();
    if (j0 >= P.n_total) continue;   // warp-uniform
    if (MODE == kModeRowSplitK && bias != nullptr) {
#pragma unroll
      for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__fadd_rn(__uint_as_float(v[e]), bv[e]));
    }
    // the staging tile is free once the previous store has read it
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
      tma_store_3d(mapC, stage, j0, row0, MODE == kModeRowPartial ? tc.batch : 0);
      bulk_commit();
    }
  }
}

// Bulk-store epilogue of the column layers (bf16 Y [p][T][s], s % 32 == 0 so
// a 32-column chunk never straddles two shards): bias + activation as in
// epilogue_tile, then each warp writes its 32 rows x 32 columns (64 bytes a
// row) into its staging tile in the 64-byte swizzled layout (16-byte chunk c
// of row r at c ^ ((r / 2) % 4): conflict-free) and one lane issues a TMA
// tensor store, clipped at T by the tensor map.
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_tile_bulk_col(const TcParams& P, const TileCoord& tc,
                                                       uint32_t tacc, int32_t row0, int half,
                                                       const EpiBias<MODE, BN>& eb,
                                                       uint32_t stage, const CUtensorMap* mapY,
                                                       int lane) {
  using S = EpiShape<MODE, BN>;
  const bool has_bias = P.bias != nullptr;
#pragma unroll
  for (int q = 0; q < S::kChunks; ++q) {
    int32_t j0;
    float y[32];
    if constexpr (MODE == kModeColumn) {
      const int c0 = half * (BN / 2) + q * 32;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + c0, v);
      tmem_ld_wait();
      j0 = tc.n * BN + c0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float bv[8];
        unpack_bf16x8(eb.v[q * 4 + g], bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float h = __uint_as_float(v[g * 8 + e]);
          if (has_bias) h += bv[e];
          y[g * 8 + e] = act_unary_mufu(P.act, h);
        }
      }
    } else {
      const int c0 = half * (BN / 4) + q * 32;   // gate column inside the accumulator
      uint32_t g32[32], u32[32];
      tmem_ld_32x32b_x32(tacc + c0, g32);
      tmem_ld_32x32b_x32(tacc + BN / 2 + c0, u32);
      tmem_ld_wait();
      j0 = tc.n * (BN / 2) + c0;
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        float bv[8];
        unpack_bf16x8(eb.v[q * 4 + g], bv);
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float gate = __uint_as_float(g32[g * 8 + e]);
          if (has_bias) gate += bv[e];
          y[g * 8 + e] = silu_mufu(gate) * __uint_as_float(u32[g * 8 + e]);
        }
      }
    }
    if (j0 >= P.n_total) continue;   // warp-uniform
    if (lane == 0) bulk_wait_read0();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t addr = stage + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr),
                   "r"(pack_bf16x2(y[8 * c], y[8 * c + 1])), "r"(pack_bf16x2(y[8 * c + 2], y[8 * c + 3])),
                   "r"(pack_bf16x2(y[8 * c + 4], y[8 * c + 5])), "r"(pack_bf16x2(y[8 * c + 6], y[8 * c + 7]))
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int32_t shard = j0 / P.s;
      tma_store_3d(mapY, stage, j0 - shard * P.s, row0, shard);
      bulk_commit();
    }
  }
}

}  // namespace gemm

// Per-layer GEMM on CTA pairs (tp_gemm2_sm100.cu): 256 x pbn tiles (pbn 128
// or 256); `mode` is a gemm::Mode; prm's tile space is recomputed.
tp_status launch_tc_pair(const LaunchCtx& c, int mode, int pbn, const CUtensorMap& a,
                         const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& cm,
                         gemm::TcParams prm);

}  // namespace tpk
