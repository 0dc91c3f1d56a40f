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
//                  bias + activation (or none), convert, store.
// Tile width BN (64..256) is picked per problem so that the tiles of a small
// problem still cover the SMs.  Every barrier wait is bounded.  Launches use
// programmatic dependent launch: the prologue overlaps the previous kernel,
// and every global access comes after griddepcontrol.wait.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cstdint>
#include <cstdlib>
#include <cstring>
#include <mutex>

#include "tp_act.cuh"
#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

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

template <int BN_>
struct Cfg {
  static constexpr int BN = BN_;
  static constexpr int B_CHUNKS = BN / B_BOX_COLS;
  static constexpr int B_BYTES = B_CHUNKS * B_CHUNK_BYTES;
  static constexpr int STAGE_BYTES = A_BYTES + B_BYTES;
  static constexpr int STAGES_FIT = (SMEM_LIMIT - 1024 - CTRL_BYTES) / STAGE_BYTES;
  static constexpr int STAGES = STAGES_FIT > 8 ? 8 : STAGES_FIT;
  static constexpr int TMEM_COLS = 2 * BN <= 128 ? 128 : (2 * BN <= 256 ? 256 : 512);
  static constexpr int SMEM_BYTES = 1024 + STAGES * STAGE_BYTES + CTRL_BYTES;
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
  __nv_bfloat16* Y = static_cast<__nv_bfloat16*>(P.out);
  *reinterpret_cast<uint4*>(Y + (static_cast<int64_t>(shard) * P.T + row) * P.s + jj) = pk;
}

// Epilogue of one tile for one warp: TMEM lanes tacc's quadrant, accumulator
// columns [c0, c0 + ncols) (ncols a multiple of 32).
template <int MODE, int BN>
__device__ __forceinline__ void epilogue_tile(const TcParams& P, const TileCoord& tc,
                                              uint32_t tacc, int row, int half) {
  const bool row_ok = row < P.T;
  if constexpr (MODE == kModeColumn) {
    const uint16_t* bias = static_cast<const uint16_t*>(P.bias);
    constexpr int NQ = BN / 64;  // 32-column chunks per half
#pragma unroll 1
    for (int q = 0; q < NQ; ++q) {
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
        float h[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          h[e] = __uint_as_float(v[g * 8 + e]);
          if (bias != nullptr) h[e] += bf16_bits_to_float(__ldg(bias + j + e));
          h[e] = act_unary_mufu(P.act, h[e]);
        }
        store_bf16x8(P, row, j, h);
      }
    }
  } else if constexpr (MODE == kModeColumnSwiglu) {
    const uint16_t* bias = static_cast<const uint16_t*>(P.bias);
    constexpr int NQ = BN / 128;  // 32-column output chunks per half
#pragma unroll 1
    for (int q = 0; q < NQ; ++q) {
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
        float y[8];
#pragma unroll
        for (int e = 0; e < 8; ++e) {
          float gate = __uint_as_float(g32[g * 8 + e]);
          if (bias != nullptr) gate += bf16_bits_to_float(__ldg(bias + j + e));
          y[e] = silu_mufu(gate) * __uint_as_float(u32[g * 8 + e]);
        }
        store_bf16x8(P, row, j, y);
      }
    }
  } else {
    const float* bias = static_cast<const float*>(P.bias);
    float* out = static_cast<float*>(P.out);
    const int64_t plane = (MODE == kModeRowPartial) ? static_cast<int64_t>(tc.batch) * P.T : 0;
    constexpr int NQ = BN / 64;
#pragma unroll 1
    for (int q = 0; q < NQ; ++q) {
      const int c0 = half * (BN / 2) + q * 32;
      uint32_t v[32];
      tmem_ld_32x32b_x32(tacc + c0, v);
      tmem_ld_wait();
      if (!row_ok) continue;
      const int32_t j0 = tc.n * BN + c0;
      float* dst = out + (plane + row) * static_cast<int64_t>(P.n_total);
#pragma unroll
      for (int g = 0; g < 8; ++g) {
        const int32_t j = j0 + g * 4;
        if (j >= P.n_total) break;
        float4 o = make_float4(__uint_as_float(v[g * 4 + 0]), __uint_as_float(v[g * 4 + 1]),
                               __uint_as_float(v[g * 4 + 2]), __uint_as_float(v[g * 4 + 3]));
        if (MODE == kModeRowSplitK && bias != nullptr) {
          o.x = __fadd_rn(o.x, bias[j + 0]);
          o.y = __fadd_rn(o.y, bias[j + 1]);
          o.z = __fadd_rn(o.z, bias[j + 2]);
          o.w = __fadd_rn(o.w, bias[j + 3]);
        }
        *reinterpret_cast<float4*>(dst + j) = o;
      }
    }
  }
}

template <int MODE, int BN>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_gemm_kernel(const __grid_constant__ CUtensorMap mapA, const __grid_constant__ CUtensorMap mapB0,
                   const __grid_constant__ CUtensorMap mapB1, const TcParams P) {
  using C = Cfg<BN>;
  constexpr int STAGES = C::STAGES;
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;  // swizzle atoms need 1024-byte alignment
  uint8_t* const ctrl = smem_raw + (base - raw) + STAGES * C::STAGE_BYTES;
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
    int32_t lt = 0;
    for (int32_t t = blockIdx.x; t < P.num_tiles; t += gridDim.x, ++lt) {
      const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
      bool ok = wait_bounded(accf_bar(b), ap, abort_flag, P.wait, kErrWaitAccFull);
      ok = __all_sync(0xffffffffu, ok);
      if (!ok) break;
      tc_fence_after();
      const TileCoord tc = decode_tile(P, t);
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * BN;
      epilogue_tile<MODE, BN>(P, tc, tacc, tc.m * BM + quad * 32 + lane, half);
      tc_fence_before();
      mbar_arrive(acce_bar(b));
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

PFN_cuTensorMapEncodeTiled_v12000 encode_fn() {
  static PFN_cuTensorMapEncodeTiled_v12000 fn = nullptr;
  static std::once_flag once;
  std::call_once(once, [] {
    void* p = nullptr;
    cudaDriverEntryPointQueryResult q;
    if (cudaGetDriverEntryPoint("cuTensorMapEncodeTiled", &p, cudaEnableDefault, &q) ==
            cudaSuccess &&
        q == cudaDriverEntryPointSuccess)
      fn = reinterpret_cast<PFN_cuTensorMapEncodeTiled_v12000>(p);
  });
  return fn;
}

// Small cache of encoded tensor maps: the same buffers are used call after
// call, and an encode is pure host work.
struct MapKey {
  const void* g;
  uint64_t dims[3], strides[2];
  uint32_t box[3];
  int rank;
  bool operator==(const MapKey& o) const { return memcmp(this, &o, sizeof(MapKey)) == 0; }
};
struct MapEntry {
  MapKey key;
  CUtensorMap map;
  bool used;
};
constexpr int kMapCache = 32;
MapEntry g_maps[kMapCache];
int g_map_next = 0;
std::mutex g_map_mu;

// bf16 tensor map, 128-byte swizzle, zero fill outside the tensor.
bool make_map(CUtensorMap* m, const void* gaddr, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.g = gaddr;
  key.rank = rank;
  for (int i = 0; i < rank; ++i) {
    key.dims[i] = dims[i];
    key.box[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) key.strides[i] = strides_bytes[i];
  {
    std::lock_guard<std::mutex> lk(g_map_mu);
    for (auto& e : g_maps)
      if (e.used && e.key == key) {
        *m = e.map;
        return true;
      }
  }
  auto fn = encode_fn();
  if (fn == nullptr) {
    set_error_detail("cuTensorMapEncodeTiled unavailable");
    return false;
  }
  cuuint64_t d[3], st[2];
  cuuint32_t bx[3], es[3] = {1, 1, 1};
  for (int i = 0; i < rank; ++i) {
    d[i] = dims[i];
    bx[i] = box[i];
  }
  for (int i = 0; i < rank - 1; ++i) st[i] = strides_bytes[i];
  const CUresult r =
      fn(m, CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
         const_cast<void*>(gaddr), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
         CU_TENSOR_MAP_SWIZZLE_128B, CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
         CU_TENSOR_MAP_FLOAT_OOB_FILL_NONE);
  if (r != CUDA_SUCCESS) {
    set_error_detail("cuTensorMapEncodeTiled failed (%d)", static_cast<int>(r));
    return false;
  }
  std::lock_guard<std::mutex> lk(g_map_mu);
  MapEntry& e = g_maps[g_map_next];
  g_map_next = (g_map_next + 1) % kMapCache;
  e.key = key;
  e.map = *m;
  e.used = true;
  return true;
}

// [rows][inner] bf16 matrices stacked `batches` times, boxes of 128 x 64.
bool make_map_a(CUtensorMap* m, const void* g, int64_t inner, int64_t rows, int64_t batches) {
  const uint64_t dims[3] = {static_cast<uint64_t>(inner), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batches)};
  const uint64_t strides[2] = {static_cast<uint64_t>(inner) * 2,
                               static_cast<uint64_t>(inner) * rows * 2};
  const uint32_t box[3] = {BK, BM, 1};
  return make_map(m, g, 3, dims, strides, box);
}

// [rows = k][cols = n] bf16 weight, N-contiguous, boxes of 64 k-rows x 64 cols.
bool make_map_b(CUtensorMap* m, const void* g, int64_t cols, int64_t rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(cols) * 2};
  const uint32_t box[2] = {B_BOX_COLS, BK};
  return make_map(m, g, 2, dims, strides, box);
}

template <int MODE, int BN>
tp_status launch_mode(const LaunchCtx& c, const CUtensorMap& a, const CUtensorMap& b0,
                      const CUtensorMap& b1, TcParams prm) {
  using Cf = Cfg<BN>;
  static bool attr_done[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(tc_gemm_kernel<MODE, BN>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_done[dev] = true;
    }
  }
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  const int grid = prm.num_tiles < c.num_sms ? prm.num_tiles : c.num_sms;
  const cudaError_t e = launch_pdl(tc_gemm_kernel<MODE, BN>, dim3(grid), dim3(NUM_THREADS),
                                   Cf::SMEM_BYTES, c.stream, a, b0, b1, prm);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("tensor-core GEMM launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

int32_t ceil_div(int64_t a, int64_t b) { return static_cast<int32_t>((a + b - 1) / b); }

// Tile width: minimise (waves of tiles over the SMs) x (per-tile cost), the
// per-tile cost taken as BN plus a fixed 64-column overhead (pipeline fill,
// epilogue).  Wide problems keep BN = 256, the most efficient per FLOP.
int pick_bn(int64_t m_tiles, int64_t n_total, int64_t batches, int num_sms, bool swiglu) {
  static const int cand_all[4] = {256, 192, 128, 64};
  static const int cand_swiglu[2] = {256, 128};
  const int* cand = swiglu ? cand_swiglu : cand_all;
  const int n = swiglu ? 2 : 4;
  int best = 256;
  int64_t best_cost = INT64_MAX;
  for (int i = 0; i < n; ++i) {
    const int bn = cand[i];
    const int64_t out_cols = swiglu ? bn / 2 : bn;
    const int64_t tiles = m_tiles * ((n_total + out_cols - 1) / out_cols) * batches;
    const int64_t waves = (tiles + num_sms - 1) / num_sms;
    const int64_t cost = waves * (bn + 64);
    if (cost < best_cost) {
      best_cost = cost;
      best = bn;
    }
  }
  return best;
}

template <int MODE>
tp_status launch_bn(const LaunchCtx& c, int bn, const CUtensorMap& a, const CUtensorMap& b0,
                    const CUtensorMap& b1, TcParams prm) {
  const int out_cols = MODE == kModeColumnSwiglu ? bn / 2 : bn;
  prm.n_tiles = ceil_div(prm.n_total, out_cols);
  prm.num_tiles = prm.m_tiles * prm.n_tiles * prm.batches;
  switch (bn) {
    case 256: return launch_mode<MODE, 256>(c, a, b0, b1, prm);
    case 128: return launch_mode<MODE, 128>(c, a, b0, b1, prm);
    default: break;
  }
  if constexpr (MODE != kModeColumnSwiglu) {
    if (bn == 192) return launch_mode<MODE, 192>(c, a, b0, b1, prm);
    if (bn == 64) return launch_mode<MODE, 64>(c, a, b0, b1, prm);
  }
  set_error_detail("no tile width %d", bn);
  return TP_ERR_UNSUPPORTED;
}

}  // namespace

tp_status launch_tc_column(const LaunchCtx& c, const void* X, const void* W1, const void* Wup,
                           const void* b1, void* Y, int64_t T, int64_t d, int64_t k, int p,
                           int act) {
  CUtensorMap mA, mB0, mB1;
  if (!make_map_a(&mA, X, d, T, 1) || !make_map_b(&mB0, W1, k, d)) return TP_ERR_CUDA;
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
  const int bn = pick_bn(prm.m_tiles, k, 1, c.num_sms, swiglu);
  if (swiglu) return launch_bn<kModeColumnSwiglu>(c, bn, mA, mB0, mB1, prm);
  return launch_bn<kModeColumn>(c, bn, mA, mB0, mB1, prm);
}

tp_status launch_tc_row(const LaunchCtx& c, const void* Y, const void* W2, float* P, int64_t T,
                        int64_t k, int64_t d, int p) {
  const int64_t s = k / p;
  CUtensorMap mA, mB;
  if (!make_map_a(&mA, Y, s, T, p) || !make_map_b(&mB, W2, d, k)) return TP_ERR_CUDA;
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
  const int bn = pick_bn(prm.m_tiles, d, p, c.num_sms, false);
  return launch_bn<kModeRowPartial>(c, bn, mA, mB, mB, prm);
}

tp_status launch_tc_row_splitk(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                               float* Z, int64_t T, int64_t k, int64_t d, int p) {
  const int64_t s = k / p;
  CUtensorMap mA, mB;
  if (!make_map_a(&mA, Y, s, T, p) || !make_map_b(&mB, W2, d, k)) return TP_ERR_CUDA;
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
  const int bn = pick_bn(prm.m_tiles, d, 1, c.num_sms, false);
  return launch_bn<kModeRowSplitK>(c, bn, mA, mB, mB, prm);
}

}  // namespace tpk
