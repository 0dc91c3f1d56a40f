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

// kModeRowChain (CTA pairs only): the row layer's tiles fold shard by shard
// into Z in the epilogue instead of writing partials.
enum Mode : int {
  kModeColumn = 0,
  kModeColumnSwiglu = 1,
  kModeRowPartial = 2,
  kModeRowSplitK = 3,
  kModeRowChain = 4
};

struct TcParams {
  int32_t T;             // tokens
  int32_t n_total;       // valid output columns: k (column) or d (row)
  int32_t s;             // shard width k/p
  int32_t p;
  int32_t m_tiles, n_tiles, batches, num_tiles;
  int32_t k_blocks;      // pipeline slots per tile
  int32_t kb_per_shard;  // split-K: slots per shard (s / 64)
  int32_t act;
  const void* bias;      // b1 (bf16, column) or b2 (fp32, split-K and chain row); may be null
  void* out;             // Y bf16 [p][T][s] | P fp32 [p][T][d] | Z fp32 [T][d]
  int32_t bulk_out;      // column layers: 1 = bulk tensor stores through shared memory
  int* region_cnt;       // row partials: per-tile completion counters read by the fold
                         // beside the layer ([n_tiles][m_tiles]); may be null.  Chain
                         // row layer: the same counters order the shards' tiles
  int* zero_cnt;         // column layers: counters this launch zeroes (after its wait for
  int32_t zero_n;        // the previous kernel) for the row layer that follows; may be null
  int32_t m_group;       // > 0: tiles walk groups of this many m-tiles, group slowest (all
                         // shards of one group before the next); 0: one group
  int32_t resid;         // chain row layer: 1 = the last shard also adds R (fp32 [T][d],
                         // the kernel's second output tensor map) after b2
  // Column layer on CTA pairs with several weights and outputs in one launch
  // (the Q, K, V projections): nseg > 1 segments, segment i owning tiles
  // [seg_start[i], seg_start[i + 1]), k = seg_n[i] output columns, shard
  // width seg_s[i]; weight i and output i come as the kernel's i-th B and C
  // tensor maps.
  int32_t nseg;
  int32_t seg_start[4];
  int32_t seg_n[3], seg_s[3];
  WaitCtl wait;
  int64_t debug_drop;    // slot (in issue order) whose load is skipped; -1 none
};

struct TileCoord {
  int32_t batch, m, n;
};

// Zeroes the counters the next row layer will count into: one warp of CTA 0,
// after griddepcontrol.wait (so no kernel before this one still reads them);
// the row layer waits for this grid to complete before it counts.
__device__ __forceinline__ void zero_counters(const TcParams& P, int warp, int lane) {
  if (P.zero_cnt != nullptr && blockIdx.x == 0 && warp == 3)
    for (int32_t i = lane; i < P.zero_n; i += 32) P.zero_cnt[i] = 0;
}

__device__ __forceinline__ TileCoord decode_tile(const TcParams& P, int32_t t) {
  // Within a group of m-tiles: shard slowest, then n, m fastest (neighbouring
  // CTAs share the weight panel).  Every group but the last is full.
  const int32_t mg_full = P.m_group > 0 ? P.m_group : P.m_tiles;
  const int32_t group_tiles = mg_full * P.n_tiles * P.batches;
  const int32_t g = t / group_tiles;
  const int32_t m0 = g * mg_full;
  const int32_t mg = P.m_tiles - m0 < mg_full ? P.m_tiles - m0 : mg_full;
  int32_t r = t - g * group_tiles;
  TileCoord c;
  c.batch = r / (mg * P.n_tiles);
  r -= c.batch * mg * P.n_tiles;
  c.n = r / mg;
  c.m = m0 + r - c.n * mg;
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

// 8 consecutive output columns j..j+7 of one row (4 bf16 pairs) into shard
// storage.
__device__ __forceinline__ void store_bf16x8(const TcParams& P, int row, int32_t j, uint4 pk) {
  const int32_t shard = j / P.s;
  const int32_t jj = j - shard * P.s;
  __nv_bfloat16* __restrict__ Y = static_cast<__nv_bfloat16*>(P.out);
  *reinterpret_cast<uint4*>(Y + (static_cast<int64_t>(shard) * P.T + row) * P.s + jj) = pk;
}

// ----------------------------------------------- column-layer activations
// Two adjacent hidden columns of one row at a time, as a packed fp32 pair:
// sm_100 issues one FFMA2 / FMUL2 / FADD2 for both, so the epilogue's
// arithmetic takes half the issue slots of the scalar form.  Results are
// rounded once to a bf16 pair (the stored Y).
//   GELU, tanh form:  h/2 + (h/2) tanh(u),  u = h (c1 + c3 h^2),
//                     c1 = sqrt(2/pi), c3 = 0.044715 c1;
//   SwiGLU:           a + a tanh(g/2),  a = (g/2) up  (= SiLU(g) up, since
//                     sigmoid(g) = (1 + tanh(g/2)) / 2).
// tanh is the MUFU approximation (relative error about 2^-11 of tanh): the
// GELU value then carries an absolute error of at most about 2^-11 |h| / 2,
// below its bf16 rounding wherever |GELU(h)| is not small; in the negative
// tail (h below about -2, where 1 + tanh(u) cancels) the relative error is
// larger but the value, and its absolute error, are tiny.

// Two bf16 bias values (one 32-bit word, lower column first) as a pair.
__device__ __forceinline__ uint64_t bf16_word_to_pair(uint32_t w) {
  return f2_pack(__uint_as_float(w << 16), __uint_as_float(w & 0xFFFF0000u));
}

__device__ __forceinline__ uint64_t tanh_pair(uint64_t x) {
  float a, b;
  f2_unpack(x, a, b);
  return f2_pack(tanh_mufu(a), tanh_mufu(b));
}

__device__ __forceinline__ uint32_t pair_to_bf16x2(uint64_t y) {
  float a, b;
  f2_unpack(y, a, b);
  return pack_bf16x2(a, b);
}

__device__ __forceinline__ uint32_t gelu_pair_bf16(uint64_t h) {
  const uint64_t c1 = f2_pack(0.7978845608028654f, 0.7978845608028654f);
  const uint64_t c3 = f2_pack(0.035677408136300125f, 0.035677408136300125f);
  const uint64_t half = f2_pack(0.5f, 0.5f);
  const uint64_t u = f2_mul(h, f2_fma(f2_mul(h, h), c3, c1));
  const uint64_t hh = f2_mul(h, half);
  return pair_to_bf16x2(f2_fma(hh, tanh_pair(u), hh));
}

__device__ __forceinline__ uint32_t swiglu_pair_bf16(uint64_t gate, uint64_t up) {
  const uint64_t hg = f2_mul(gate, f2_pack(0.5f, 0.5f));
  const uint64_t a = f2_mul(hg, up);
  return pair_to_bf16x2(f2_fma(a, tanh_pair(hg), a));
}

// Identity / ReLU (the exact-integer test activations): scalar.
__device__ __forceinline__ uint32_t plain_pair_bf16(int act, uint64_t h) {
  float a, b;
  f2_unpack(h, a, b);
  return pack_bf16x2(act_unary_mufu(act, a), act_unary_mufu(act, b));
}

__device__ __forceinline__ uint32_t word_of(const uint4& u, int k) {
  return k == 0 ? u.x : (k == 1 ? u.y : (k == 2 ? u.z : u.w));
}

// One row's 32-column chunk of the column layer: the accumulator words `a`
// (gate for SwiGLU, with `up` the matching up-projection words), the bias
// (4 vectors of 8 bf16, or none) and the activation, into 16 bf16 pairs.
template <bool kSwiglu>
__device__ __forceinline__ void act_chunk_bf16(int act, bool has_bias, const uint32_t (&a)[32],
                                               const uint32_t (&up)[32], const uint4* bias,
                                               uint32_t (&out)[16]) {
  if (kSwiglu) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      uint64_t g = f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
      if (has_bias) g = f2_add(g, bf16_word_to_pair(word_of(bias[i / 4], i % 4)));
      out[i] = swiglu_pair_bf16(g, f2_pack(__uint_as_float(up[2 * i]),
                                           __uint_as_float(up[2 * i + 1])));
    }
  } else if (act == kActGeluTanh) {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      uint64_t h = f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
      if (has_bias) h = f2_add(h, bf16_word_to_pair(word_of(bias[i / 4], i % 4)));
      out[i] = gelu_pair_bf16(h);
    }
  } else {
#pragma unroll
    for (int i = 0; i < 16; ++i) {
      uint64_t h = f2_pack(__uint_as_float(a[2 * i]), __uint_as_float(a[2 * i + 1]));
      if (has_bias) h = f2_add(h, bf16_word_to_pair(word_of(bias[i / 4], i % 4)));
      out[i] = plain_pair_bf16(act, h);
    }
  }
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
  if constexpr (S::kColumn) {
    constexpr bool kSwiglu = (MODE == kModeColumnSwiglu);
    const bool has_bias = P.bias != nullptr;
    // unrolled: the prefetched bias registers are indexed by chunk
#pragma unroll
    for (int q = 0; q < S::kChunks; ++q) {
      // gate (or hidden) column inside the accumulator; SwiGLU's up columns
      // sit BN/2 further
      const int c0 = half * (S::kOutCols / 2) + q * 32;
      uint32_t v[32], u[32];
      tmem_ld_32x32b_x32(tacc + c0, v);
      if (kSwiglu) tmem_ld_32x32b_x32(tacc + BN / 2 + c0, u);
      tmem_ld_wait();
      if (!row_ok) continue;
      const int32_t j0 = tc.n * S::kOutCols + c0;
      uint32_t y[16];
      act_chunk_bf16<kSwiglu>(P.act, has_bias, v, u, &eb.v[q * 4], y);
#pragma unroll
      for (int g = 0; g < 4; ++g) {
        const int32_t j = j0 + g * 8;
        if (j >= P.n_total) break;
        store_bf16x8(P, row, j, make_uint4(y[4 * g], y[4 * g + 1], y[4 * g + 2], y[4 * g + 3]));
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
// a 32-column chunk never straddles two shards): bias + activation on packed
// pairs, then each warp writes its 32 rows x 32 columns (64 bytes a row) into
// one half of its staging tile in the 64-byte swizzled layout (16-byte chunk
// c of row r at c ^ ((r / 2) % 4): conflict-free) and one lane issues a TMA
// tensor store, clipped at T by the tensor map.  The two halves alternate
// (`nchunk` counts the warp's chunks across tiles), so a chunk waits only
// for the store before last to have read its half, not for the previous one.
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_tile_bulk_col(const TcParams& P, const TileCoord& tc,
                                                       uint32_t tacc, int32_t row0, int half,
                                                       const EpiBias<MODE, BN>& eb,
                                                       uint32_t stage, const CUtensorMap* mapY,
                                                       int lane, uint32_t& nchunk) {
  using S = EpiShape<MODE, BN>;
  constexpr bool kSwiglu = (MODE == kModeColumnSwiglu);
  constexpr uint32_t kChunkBytes = 32 * 64;
  static_assert(2 * kChunkBytes <= EPI_WARP_STAGE_BYTES, "two bf16 chunks per staging tile");
  const bool has_bias = P.bias != nullptr;
#pragma unroll
  for (int q = 0; q < S::kChunks; ++q) {
    const int c0 = half * (S::kOutCols / 2) + q * 32;
    const int32_t j0 = tc.n * S::kOutCols + c0;
    if (j0 >= P.n_total) break;   // warp-uniform; later chunks are further right
    uint32_t v[32], u[32];
    tmem_ld_32x32b_x32(tacc + c0, v);
    if (kSwiglu) tmem_ld_32x32b_x32(tacc + BN / 2 + c0, u);
    tmem_ld_wait();
    uint32_t y[16];
    act_chunk_bf16<kSwiglu>(P.act, has_bias, v, u, &eb.v[q * 4], y);
    const uint32_t buf = stage + (nchunk & 1u) * kChunkBytes;
    // the half is free once the store issued two chunks ago has read it
    if (lane == 0) bulk_wait_read1();
    __syncwarp();
#pragma unroll
    for (int c = 0; c < 4; ++c) {
      const uint32_t addr = buf + lane * 64 + ((c ^ ((lane >> 1) & 3)) << 4);
      asm volatile("st.shared.v4.b32 [%0], {%1, %2, %3, %4};" ::"r"(addr), "r"(y[4 * c]),
                   "r"(y[4 * c + 1]), "r"(y[4 * c + 2]), "r"(y[4 * c + 3])
                   : "memory");
    }
    fence_proxy_async_smem();
    __syncwarp();
    if (lane == 0) {
      const int32_t shard = j0 / P.s;
      tma_store_3d(mapY, buf, j0 - shard * P.s, row0, shard);
      bulk_commit();
    }
    ++nchunk;
  }
}

}  // namespace gemm

// Per-layer GEMM on CTA pairs (tp_gemm2_sm100.cu): 256 x pbn tiles (pbn 128
// or 256); `mode` is a gemm::Mode; prm's tile space is recomputed.
// (chain row layer: `c1` is the map of R when prm.resid is set)
tp_status launch_tc_pair(const LaunchCtx& c, int mode, int pbn, const CUtensorMap& a,
                         const CUtensorMap& b0, const CUtensorMap& b1, const CUtensorMap& cm,
                         gemm::TcParams prm, const CUtensorMap* c1 = nullptr);
// Up to three identity column layers of one input in one launch of 256 x pbn
// pair tiles, pbn 128 or 256 (tp_gemm2_sm100.cu).
tp_status launch_tc_pair_column_multi(const LaunchCtx& c, int pbn, const CUtensorMap& a,
                                      const CUtensorMap* b, const CUtensorMap* cm,
                                      const int64_t* k, int nseg, gemm::TcParams prm);

}  // namespace tpk
