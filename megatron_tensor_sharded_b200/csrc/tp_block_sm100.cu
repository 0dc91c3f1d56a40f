// Both GEMM layers of the sharded MLP block in one persistent tensor-core
// launch (sm_100a).
//
// Tiles of both layers share one static schedule: first every column-parallel
// tile (Y_i = act(X W1_i + b1_i), all shards), then every row-parallel tile
// (partials P_i = Y_i W2_i, shard by shard as the separate row kernel runs
// them, or split-K over shards straight into Z).  A row tile of m-tile m
// needs the hidden rows of that m-tile from every column tile: column tiles
// publish completion through a per-m-tile counter (release), and the
// producer of a row tile waits on it (acquire, bounded) before its TMA reads
// the hidden shards.  The schedule cannot deadlock: column tiles never wait,
// and every CTA runs all of its column tiles before any of its row tiles,
// so each column tile a row tile waits for belongs to a CTA that is running
// or has not started yet and needs nothing to make progress.  The grid is
// at most one CTA per SM, so normally every CTA is resident from the start;
// when other work holds SMs (other streams, processes, MPS), a CTA whose
// column tiles have not been scheduled yet delays the row tiles waiting on
// them, and under heavy contention that delay can run past the bounded wait
// (TP_ERR_DEVICE_TIMEOUT, reported by the call's status word).  The row
// layer thus starts without a kernel boundary, on SMs the column layer has
// left idle.
//
// The arithmetic of every output element is that of the separate kernels
// (same MMA k order, same epilogues), so Y and the partials are bit-identical
// to tp_column_linear -> tp_row_linear.
#include <cuda.h>
#include <cuda_runtime.h>

#include <climits>
#include <cstdint>
#include <mutex>

#include "tp_gemm_parts.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

using namespace gemm;

constexpr unsigned kErrWaitDep = 1u << 5;  // a row tile's hidden rows never completed

struct BlockParams {
  TcParams col;         // column phase: out = Y (bf16), bias = b1
  TcParams row;         // row phase: out = P (partials) or Z (split-K)
  int32_t n_col_tiles;  // the schedule's first n_col_tiles tiles are column tiles
  int32_t num_tiles;
  int32_t dep_target;   // column tiles per m-tile
  int* dep_cnt;         // [m_tiles] column tiles finished
};

// Barrier 1 among the epilogue warps only (warps 4..11).
__device__ __forceinline__ void epi_sync() {
  asm volatile("bar.sync 1, %0;" ::"n"(NUM_EPI_WARPS * 32) : "memory");
}

// Same barrier, and AND of a predicate over all epilogue threads.
__device__ __forceinline__ bool epi_all(bool v) {
  uint32_t r;
  asm volatile(
      "{\n\t.reg .pred p, q;\n\t"
      "setp.ne.u32 q, %1, 0;\n\t"
      "bar.red.and.pred p, 1, %2, q;\n\t"
      "selp.u32 %0, 1, 0, p;\n\t}"
      : "=r"(r)
      : "r"(static_cast<uint32_t>(v)), "n"(NUM_EPI_WARPS * 32)
      : "memory");
  return r != 0;
}

// Bounded wait (acquire) until `*cnt >= target`, then order the async proxy
// (TMA) after it.
__device__ __forceinline__ bool wait_counter(const int* cnt, int target, volatile int* abort,
                                             const WaitCtl& w) {
  if (ld_acquire_gpu(cnt) < target) {
    const uint64_t t0 = globaltimer_ns();
    while (ld_acquire_gpu(cnt) < target) {
      if (*abort) return false;
      if (globaltimer_ns() - t0 > w.timeout_ns) {
        *abort = 1;
        atomicOr(w.err, kErrWaitDep);
        return false;
      }
      __nanosleep(64);
    }
  }
  fence_proxy_async_global();
  return true;
}

template <bool SWIGLU, bool SPLITK, int BNC, int BNR>
__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_block_kernel(const __grid_constant__ CUtensorMap mapX, const __grid_constant__ CUtensorMap mapW1,
                    const __grid_constant__ CUtensorMap mapWu, const __grid_constant__ CUtensorMap mapY,
                    const __grid_constant__ CUtensorMap mapW2, const BlockParams B) {
  constexpr int MODE_C = SWIGLU ? kModeColumnSwiglu : kModeColumn;
  constexpr int MODE_R = SPLITK ? kModeRowSplitK : kModeRowPartial;
  constexpr int BNMAX = BNC > BNR ? BNC : BNR;
  using C = Cfg<BNMAX>;  // slots and TMEM sized for the wider tile
  constexpr int STAGES = C::STAGES;
  constexpr uint32_t IDESC_C = idesc_bf16_f32(BM, BNC, 0, 1);
  constexpr uint32_t IDESC_R = idesc_bf16_f32(BM, BNR, 0, 1);
  constexpr uint32_t TX_C = A_BYTES + (BNC / B_BOX_COLS) * B_CHUNK_BYTES;
  constexpr uint32_t TX_R = A_BYTES + (BNR / B_BOX_COLS) * B_CHUNK_BYTES;

  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
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
  const WaitCtl& W = B.col.wait;

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
    tma_prefetch_map(&mapX);
    tma_prefetch_map(&mapW1);
    if (SWIGLU) tma_prefetch_map(&mapWu);
    tma_prefetch_map(&mapY);
    tma_prefetch_map(&mapW2);
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
      // ------------------------------------------------------------ producer
      uint32_t stage = 0, phase = 0;
      int64_t issued = 0;
      bool ok = true;
      for (int32_t t = blockIdx.x; ok && t < B.num_tiles; t += gridDim.x) {
        const bool is_col = t < B.n_col_tiles;
        TileCoord tc;
        if (is_col) {
          tc = decode_tile(B.col, t);
        } else {
          tc = decode_tile(B.row, t - B.n_col_tiles);
          if (!wait_counter(B.dep_cnt + tc.m, B.dep_target, abort_flag, W)) break;
        }
        const int32_t kblocks = is_col ? B.col.k_blocks : B.row.k_blocks;
        for (int32_t kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(empty_bar(stage), phase ^ 1u, abort_flag, W, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (issued != B.col.debug_drop) {
            if (is_col) {
              mbar_arrive_expect_tx(full_bar(stage), TX_C);
              issue_slot<MODE_C, BNC>(B.col, &mapX, &mapW1, &mapWu, tc, kb, slot_a(stage),
                                      slot_b(stage), full_bar(stage));
            } else {
              mbar_arrive_expect_tx(full_bar(stage), TX_R);
              issue_slot<MODE_R, BNR>(B.row, &mapY, &mapW2, &mapW2, tc, kb, slot_a(stage),
                                      slot_b(stage), full_bar(stage));
            }
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
        if (q == B.col.debug_drop) continue;
        wait_teardown(full_bar(static_cast<uint32_t>(q % STAGES)),
                      static_cast<uint32_t>((q / STAGES) & 1), W);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      uint32_t stage = 0, phase = 0;
      bool ok = true;
      int32_t lt = 0;
      for (int32_t t = blockIdx.x; ok && t < B.num_tiles; t += gridDim.x, ++lt) {
        const bool is_col = t < B.n_col_tiles;
        const int32_t kblocks = is_col ? B.col.k_blocks : B.row.k_blocks;
        const uint32_t idesc = is_col ? IDESC_C : IDESC_R;
        const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
        if (!wait_bounded(acce_bar(b), ap ^ 1u, abort_flag, W, kErrWaitAccEmpty)) {
          ok = false;
          break;
        }
        tc_fence_after();
        const uint32_t d_tmem = tmem_base + b * BNMAX;
        for (int32_t kb = 0; kb < kblocks; ++kb) {
          if (!wait_bounded(full_bar(stage), phase, abort_flag, W, kErrWaitFull)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t sa = slot_a(stage), sb = slot_b(stage);
#pragma unroll
          for (int kk = 0; kk < BK / UK; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sa + kk * UK * 2, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sb + kk * UK * 128, B_CHUNK_BYTES, 1024);
            tc_mma_f16(d_tmem, adesc, bdesc, idesc, (kb > 0 || kk > 0) ? 1u : 0u);
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
      wait_teardown(drain_bar, 0, W);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // -------------------------------------------------------------- epilogue
    const int quad = warp & 3;
    const int half = (warp - 4) >> 2;
    const int etid = threadIdx.x - 128;   // 0..255 among the epilogue threads
    int32_t lt = 0;
    for (int32_t t = blockIdx.x; t < B.num_tiles; t += gridDim.x, ++lt) {
      const uint32_t b = lt & 1, ap = (lt >> 1) & 1;
      const bool is_col = t < B.n_col_tiles;
      const TileCoord tc = is_col ? decode_tile(B.col, t) : decode_tile(B.row, t - B.n_col_tiles);
      EpiBias<MODE_C, BNC> eb;
      if (is_col) load_epi_bias<MODE_C, BNC>(B.col, tc, half, eb);
      bool ok = wait_bounded(accf_bar(b), ap, abort_flag, W, kErrWaitAccFull);
      // all epilogue warps take the same decision (they meet at barrier 1 below)
      if (!epi_all(ok)) break;
      tc_fence_after();
      const uint32_t tacc = tmem_base + (static_cast<uint32_t>(quad * 32) << 16) + b * BNMAX;
      const int row = tc.m * BM + quad * 32 + lane;
      if (is_col) {
        epilogue_tile<MODE_C, BNC>(B.col, tc, tacc, row, half, eb);
        tc_fence_before();
        mbar_arrive(acce_bar(b));
        // Publish the hidden rows to the other CTAs' TMA (async proxy):
        // every writer orders its stores for the async proxy, the barrier
        // gathers them, one thread releases the count.
        fence_proxy_async_global();
        epi_sync();
        if (etid == 0) {
          __threadfence();
          atomicAdd(B.dep_cnt + tc.m, 1);
        }
      } else {
        const EpiBias<MODE_R, BNR> none{};
        epilogue_tile<MODE_R, BNR>(B.row, tc, tacc, row, half, none);
        tc_fence_before();
        mbar_arrive(acce_bar(b));
      }
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, C::TMEM_COLS);
  }
}

// ------------------------------------------------------------------ host side

template <bool SWIGLU, bool SPLITK, int BNC, int BNR>
tp_status launch_cfg(const LaunchCtx& c, const CUtensorMap& mX, const CUtensorMap& mW1,
                     const CUtensorMap& mWu, const CUtensorMap& mY, const CUtensorMap& mW2,
                     BlockParams B) {
  constexpr int BNMAX = BNC > BNR ? BNC : BNR;
  using Cf = Cfg<BNMAX>;
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_block_kernel<SWIGLU, SPLITK, BNC, BNR>,
                               cudaFuncAttributeMaxDynamicSharedMemorySize,
                               Cf::SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  const int grid = B.num_tiles < c.num_sms ? B.num_tiles : c.num_sms;
  const cudaError_t e = launch_pdl(tc_block_kernel<SWIGLU, SPLITK, BNC, BNR>, dim3(grid),
                                   dim3(NUM_THREADS), Cf::SMEM_BYTES, c.stream, mX, mW1, mWu, mY,
                                   mW2, B);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("fused block launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

// Critical-path estimate of a (column, row) tile-width pair: waves of each
// phase times per-tile cost (width + 64) times k slots.
int64_t estimate(int64_t m_tiles, int64_t k, int64_t d, int p, bool swiglu, bool splitk,
                 int64_t kb_col, int64_t kb_row, int num_sms, int bnc, int bnr) {
  const int64_t col_out = swiglu ? bnc / 2 : bnc;
  const int64_t col_tiles = m_tiles * ((k + col_out - 1) / col_out);
  const int64_t row_tiles = m_tiles * ((d + bnr - 1) / bnr) * (splitk ? 1 : p);
  const int64_t wc = (col_tiles + num_sms - 1) / num_sms;
  const int64_t wr = (row_tiles + num_sms - 1) / num_sms;
  return wc * (bnc + 64) * kb_col + wr * (bnr + 64) * kb_row;
}

template <bool SWIGLU, bool SPLITK>
tp_status launch_pair(const LaunchCtx& c, int bnc, int bnr, const CUtensorMap& mX,
                      const CUtensorMap& mW1, const CUtensorMap& mWu, const CUtensorMap& mY,
                      const CUtensorMap& mW2, BlockParams B) {
  if (bnc == 256 && bnr == 256) return launch_cfg<SWIGLU, SPLITK, 256, 256>(c, mX, mW1, mWu, mY, mW2, B);
  if (bnc == 128 && bnr == 128) return launch_cfg<SWIGLU, SPLITK, 128, 128>(c, mX, mW1, mWu, mY, mW2, B);
  if constexpr (!SWIGLU) {
    if (bnc == 192 && bnr == 128) return launch_cfg<SWIGLU, SPLITK, 192, 128>(c, mX, mW1, mWu, mY, mW2, B);
  }
  set_error_detail("no fused tile pair %d/%d", bnc, bnr);
  return TP_ERR_UNSUPPORTED;
}

}  // namespace

size_t block_counter_bytes(int64_t T, int64_t d) {
  (void)d;
  const int64_t m_tiles = (T + 127) / 128;
  const size_t bytes = static_cast<size_t>(m_tiles) * sizeof(int);
  return (bytes + 255) & ~size_t(255);
}

tp_status launch_tc_block(const LaunchCtx& c, const void* X, const void* W1, const void* Wup,
                          const void* b1, const void* W2, const float* b2, void* Y, float* P,
                          float* Z, int* counters, int64_t T, int64_t d, int64_t k, int p, int act,
                          bool splitk) {
  const int64_t s = k / p;
  const bool swiglu = (act == kActSwiglu);
  CUtensorMap mX, mW1, mWu, mY, mW2;
  if (!make_map_a(&mX, X, d, T, 1) || !make_map_b(&mW1, W1, k, d) ||
      !make_map_a(&mY, Y, s, T, p) || !make_map_b(&mW2, W2, d, k))
    return TP_ERR_CUDA;
  if (swiglu) {
    if (!make_map_b(&mWu, Wup, k, d)) return TP_ERR_CUDA;
  } else {
    mWu = mW1;
  }
  const int32_t m_tiles = ceil_div(T, BM);
  const int64_t kb_col = ceil_div(d, BK);
  const int64_t kb_row = splitk ? (s / BK) * p : ceil_div(s, BK);

  static const int pairs_all[3][2] = {{256, 256}, {192, 128}, {128, 128}};
  static const int pairs_swiglu[2][2] = {{256, 256}, {128, 128}};
  const int npairs = swiglu ? 2 : 3;
  int bnc = 256, bnr = 256;
  int64_t best = INT64_MAX;
  for (int i = 0; i < npairs; ++i) {
    const int* pr = swiglu ? pairs_swiglu[i] : pairs_all[i];
    const int64_t e = estimate(m_tiles, k, d, p, swiglu, splitk, kb_col, kb_row, c.num_sms, pr[0], pr[1]);
    if (e < best) {
      best = e;
      bnc = pr[0];
      bnr = pr[1];
    }
  }

  BlockParams B{};
  TcParams& C = B.col;
  C.T = static_cast<int32_t>(T);
  C.n_total = static_cast<int32_t>(k);
  C.s = static_cast<int32_t>(s);
  C.p = p;
  C.m_tiles = m_tiles;
  C.n_tiles = ceil_div(k, swiglu ? bnc / 2 : bnc);
  C.batches = 1;
  C.num_tiles = C.m_tiles * C.n_tiles;
  C.k_blocks = static_cast<int32_t>(kb_col);
  C.act = act;
  C.bias = b1;
  C.out = Y;
  C.wait.err = c.err_word;
  C.wait.timeout_ns = c.timeout_ns;
  C.debug_drop = c.debug_drop;

  TcParams& R = B.row;
  R.T = static_cast<int32_t>(T);
  R.n_total = static_cast<int32_t>(d);
  R.s = static_cast<int32_t>(s);
  R.p = p;
  R.m_tiles = m_tiles;
  R.n_tiles = ceil_div(d, bnr);
  R.batches = splitk ? 1 : p;
  R.num_tiles = R.m_tiles * R.n_tiles * R.batches;
  R.k_blocks = static_cast<int32_t>(kb_row);
  R.kb_per_shard = static_cast<int32_t>(splitk ? s / BK : kb_row);
  R.act = kActIdentity;
  R.bias = splitk ? static_cast<const void*>(b2) : nullptr;
  R.out = splitk ? static_cast<void*>(Z) : static_cast<void*>(P);
  R.wait = C.wait;
  R.debug_drop = -1;

  B.n_col_tiles = C.num_tiles;
  B.num_tiles = C.num_tiles + R.num_tiles;
  B.dep_target = C.n_tiles;
  B.dep_cnt = counters;

  if (swiglu) {
    return splitk ? launch_pair<true, true>(c, bnc, bnr, mX, mW1, mWu, mY, mW2, B)
                  : launch_pair<true, false>(c, bnc, bnr, mX, mW1, mWu, mY, mW2, B);
  }
  return splitk ? launch_pair<false, true>(c, bnc, bnr, mX, mW1, mWu, mY, mW2, B)
                : launch_pair<false, false>(c, bnc, bnr, mX, mW1, mWu, mY, mW2, B);
}

}  // namespace tpk
