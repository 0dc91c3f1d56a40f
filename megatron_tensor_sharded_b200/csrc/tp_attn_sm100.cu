// Attention of every shard's own heads, one persistent tcgen05 launch (sm_100a).
//
// The tensor-parallel attention block gives each shard h/p query heads (and
// h_kv/p key/value heads) through column-parallel Q, K, V projections; the
// attention itself then runs on each shard's heads with no communication
// (day-41 post, "Attention heads: naturally parallel"; "Tensor parallel
// math", "Attention: parallel across heads": softmax(Q K^T / sqrt(d_k)) V per
// head).  This kernel computes it for all shards and heads at once.
//
// Work unit: (shard, query head, block of 128 queries); key/value blocks of
// 128.  Roles (256 threads):
//   warp 0 lane 0  TMA: the unit's Q tile [128 x 128] once, then K_j, V_j per
//                  key block through a 2-slot ring (128-byte swizzle);
//   warp 1 lane 0  MMA: S_j = Q K_j^T into one of two TMEM score buffers
//                  (128 x 128 fp32), O += P_j V_j into a TMEM accumulator;
//                  S_{j+1} is issued before O += P_j V_j so the tensor core
//                  works while the softmax of block j runs;
//   warp 2         TMEM allocation;
//   warps 4..7     online softmax: thread = query row (its TMEM lane), so
//                  the row maximum and sum never leave the thread; scores
//                  in the log2 domain with ex2.approx; when the row maximum
//                  grows, the thread rescales its O row in TMEM before the
//                  next O += P V; P is written as bf16 into shared memory in
//                  the MMA's K-major 128-byte-swizzled layout; at the end O
//                  is divided by the row sum, converted to bf16 and stored.
// Keys beyond T and (causal) keys after the query are masked.  Every
// barrier wait is bounded.
#include <cuda.h>
#include <cuda_bf16.h>
#include <cuda_runtime.h>

#include <cmath>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "tp_device.cuh"
#include "tp_internal.h"
#include "tp_launch.cuh"

namespace tpk {
namespace {

constexpr int DH = 128;                 // head dimension
constexpr int BQ = 128;                 // queries per unit (TMEM lanes)
constexpr int BKV = 128;                // keys per block
constexpr int NST = 2;                  // K/V ring slots
constexpr int TILE_BYTES = 128 * 128 * 2;   // one 128 x 128 bf16 tile (two 64-column boxes)
constexpr int HALF_BYTES = TILE_BYTES / 2;  // one box: 128 rows x 64 columns
constexpr int SMEM_BYTES = 1024 + 2 * TILE_BYTES /* Q, P */ + NST * 2 * TILE_BYTES /* K, V */ + 256;
constexpr int NUM_THREADS = 256;
constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, /*a_mn=*/0, /*b_mn=*/0);  // Q K^T
constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, DH, /*a_mn=*/0, /*b_mn=*/1);   // P V
constexpr uint32_t S_COL0 = 0, O_COL = 2 * BKV, TMEM_COLS = 512;
constexpr unsigned kErrWaitAttn = 1u << 6;

struct AttnParams {
  int32_t T, p, hq, hkv, group, q_blocks, num_units, causal;
  float scale_log2;          // log2(e) / sqrt(DH)
  __nv_bfloat16* O;          // [p][T][hq*DH]
  WaitCtl wait;
  int64_t debug_drop;
};

struct Unit {
  int32_t shard, head, qb, kvh, nkb;
};

__device__ __forceinline__ Unit decode_unit(const AttnParams& P, int32_t u) {
  Unit x;
  x.qb = u % P.q_blocks;          // query blocks fastest: neighbours share K, V
  const int32_t r = u / P.q_blocks;
  x.head = r % P.hq;
  x.shard = r / P.hq;
  x.kvh = x.head / P.group;
  const int32_t all = (P.T + BKV - 1) / BKV;
  x.nkb = P.causal ? (x.qb + 1 < all ? x.qb + 1 : all) : all;
  return x;
}

__device__ __forceinline__ float ex2(float x) {
  float y;
  asm("ex2.approx.ftz.f32 %0, %1;" : "=f"(y) : "f"(x));
  return y;
}

__device__ __forceinline__ uint32_t pack2(float lo, float hi) {
  __nv_bfloat162 v = __floats2bfloat162_rn(lo, hi);
  uint32_t u;
  memcpy(&u, &v, 4);
  return u;
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  const uint32_t sQ = base, sP = base + TILE_BYTES;
  auto sK = [&](uint32_t st) { return base + 2 * TILE_BYTES + st * 2 * TILE_BYTES; };
  auto sV = [&](uint32_t st) { return base + 2 * TILE_BYTES + st * 2 * TILE_BYTES + TILE_BYTES; };
  uint8_t* const ctrl = smem_raw + (base - raw) + 2 * TILE_BYTES + NST * 2 * TILE_BYTES;
  uint8_t* const sP_ptr = smem_raw + (base - raw) + TILE_BYTES;
  uint64_t* const bars = reinterpret_cast<uint64_t*>(ctrl);
  // barrier slots
  const uint32_t q_full = smem_u32(&bars[0]), q_empty = smem_u32(&bars[1]);
  auto kv_full = [&](uint32_t s) { return smem_u32(&bars[2 + s]); };
  auto kv_empty = [&](uint32_t s) { return smem_u32(&bars[2 + NST + s]); };
  auto s_full = [&](uint32_t b) { return smem_u32(&bars[2 + 2 * NST + b]); };
  auto s_empty = [&](uint32_t b) { return smem_u32(&bars[4 + 2 * NST + b]); };
  const uint32_t p_full = smem_u32(&bars[6 + 2 * NST]);
  const uint32_t o_done = smem_u32(&bars[7 + 2 * NST]);
  const uint32_t o_empty = smem_u32(&bars[8 + 2 * NST]);
  const uint32_t drain = smem_u32(&bars[9 + 2 * NST]);
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * (10 + 2 * NST));
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int b = 0; b < 2; ++b) {
      mbar_init(s_full(b), 1);
      mbar_init(s_empty(b), 128);
    }
    mbar_init(p_full, 128);
    mbar_init(o_done, 1);
    mbar_init(o_empty, 128);
    mbar_init(drain, 1);
    *abort_flag = 0;
    fence_barrier_init();
    fence_proxy_async_smem();
  }
  if (warp == 0 && lane == 0) {
    tma_prefetch_map(&mapQ);
    tma_prefetch_map(&mapK);
    tma_prefetch_map(&mapV);
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
      uint32_t st = 0, ph = 0;
      int64_t issued = 0, last_q = -1;
      int32_t lu = 0;
      bool ok = true;
      for (int32_t u = blockIdx.x; ok && u < P.num_units; u += gridDim.x, ++lu) {
        const Unit x = decode_unit(P, u);
        if (!wait_bounded(q_empty, (lu & 1) ^ 1u, abort_flag, P.wait, kErrWaitAttn)) break;
        mbar_arrive_expect_tx(q_full, TILE_BYTES);
        for (int c = 0; c < 2; ++c)
          tma_load_3d(sQ + c * HALF_BYTES, &mapQ, q_full, x.head * DH + c * 64, x.qb * BQ, x.shard);
        last_q = lu;
        for (int32_t j = 0; j < x.nkb; ++j) {
          if (!wait_bounded(kv_empty(st), ph ^ 1u, abort_flag, P.wait, kErrWaitEmpty)) {
            ok = false;
            break;
          }
          if (issued != P.debug_drop) {
            mbar_arrive_expect_tx(kv_full(st), 2 * TILE_BYTES);
            for (int c = 0; c < 2; ++c) {
              tma_load_3d(sK(st) + c * HALF_BYTES, &mapK, kv_full(st), x.kvh * DH + c * 64, j * BKV,
                          x.shard);
              tma_load_3d(sV(st) + c * HALF_BYTES, &mapV, kv_full(st), x.kvh * DH + c * 64, j * BKV,
                          x.shard);
            }
          }
          ++issued;
          if (++st == NST) {
            st = 0;
            ph ^= 1u;
          }
        }
      }
      // Teardown: let the last loads land before shared memory is released.
      if (last_q >= 0) wait_teardown(q_full, static_cast<uint32_t>(last_q & 1), P.wait);
      const int64_t first = issued > NST ? issued - NST : 0;
      for (int64_t q = first; q < issued; ++q) {
        if (q == P.debug_drop) continue;
        wait_teardown(kv_full(static_cast<uint32_t>(q % NST)), static_cast<uint32_t>((q / NST) & 1),
                      P.wait);
      }
    }
    __syncwarp();
  } else if (warp == 1) {
    if (lane == 0) {
      // ---------------------------------------------------------- MMA issuer
      // K/V blocks are consumed in the producer's order: block n of the whole
      // sequence sits in ring slot n % NST, phase (n / NST) & 1.
      uint32_t kv_n = 0;         // K/V blocks taken by S MMAs so far
      uint32_t gs = 0;           // S buffers used so far
      uint32_t gb = 0;           // P V products issued so far
      int32_t lu = 0;
      bool ok = true;
      auto issue_s = [&](uint32_t kst) {
        const uint32_t b = gs & 1;
        const uint32_t d = tmem_base + S_COL0 + b * BKV;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          tc_mma_f16(d, smem_desc_sw128(sQ + off, 16, 1024), smem_desc_sw128(sK(kst) + off, 16, 1024),
                     IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full(b));
        ++gs;
      };
      // wait for K/V block n and a free S buffer, then issue S = Q K_n^T
      auto next_s = [&](uint32_t n) -> bool {
        if (!wait_bounded(kv_full(n % NST), (n / NST) & 1, abort_flag, P.wait, kErrWaitFull) ||
            !wait_bounded(s_empty(gs & 1), ((gs >> 1) & 1) ^ 1u, abort_flag, P.wait, kErrWaitAttn))
          return false;
        tc_fence_after();
        issue_s(n % NST);
        return true;
      };
      for (int32_t u = blockIdx.x; ok && u < P.num_units; u += gridDim.x, ++lu) {
        const Unit x = decode_unit(P, u);
        if (!wait_bounded(q_full, lu & 1, abort_flag, P.wait, kErrWaitAttn)) break;
        const uint32_t n0 = kv_n;
        if (!next_s(n0)) break;
        for (int32_t j = 0; j < x.nkb; ++j) {
          if (j + 1 < x.nkb && !next_s(n0 + j + 1)) {
            ok = false;
            break;
          }
          if (j == 0 && lu > 0 &&
              !wait_bounded(o_empty, (lu - 1) & 1, abort_flag, P.wait, kErrWaitAttn)) {
            ok = false;
            break;
          }
          if (!wait_bounded(p_full, gb & 1, abort_flag, P.wait, kErrWaitAttn)) {
            ok = false;
            break;
          }
          tc_fence_after();
          const uint32_t vst = (n0 + j) % NST;
#pragma unroll
          for (int kk = 0; kk < BKV / 16; ++kk) {
            const uint64_t adesc = smem_desc_sw128(sP + (kk >> 2) * HALF_BYTES + (kk & 3) * 32, 16, 1024);
            const uint64_t bdesc = smem_desc_sw128(sV(vst) + kk * 16 * 128, HALF_BYTES, 1024);
            tc_mma_f16(tmem_base + O_COL, adesc, bdesc, IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
          }
          tc_commit(o_done);
          tc_commit(kv_empty(vst));
          ++gb;
        }
        if (!ok) break;
        kv_n = n0 + x.nkb;
        tc_commit(q_empty);
      }
      tc_commit(drain);
      wait_teardown(drain, 0, P.wait);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------- softmax / output
    const int quad = warp & 3;
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    uint32_t gs = 0, gb = 0;
    int32_t lu = 0;
    for (int32_t u = blockIdx.x; u < P.num_units; u += gridDim.x, ++lu) {
      const Unit x = decode_unit(P, u);
      const int32_t q = x.qb * BQ + quad * 32 + lane;
      float m = -INFINITY, l = 0.0f;
      bool ok = true;
      for (int32_t j = 0; j < x.nkb; ++j) {
        const uint32_t b = gs & 1;
        ok = wait_bounded(s_full(b), (gs >> 1) & 1, abort_flag, P.wait, kErrWaitAttn);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const uint32_t tS = tmem_base + lane_off + S_COL0 + b * BKV;
        const int32_t key0 = j * BKV;
        // pass 1: row maximum (log2 domain)
        float mx = -INFINITY;
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tS + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; ++e) {
            const int32_t key = key0 + c * 32 + e;
            const bool valid = key < P.T && (!P.causal || key <= q);
            const float xv = valid ? __uint_as_float(v[e]) * P.scale_log2 : -INFINITY;
            mx = fmaxf(mx, xv);
          }
        }
        const float m_new = fmaxf(m, mx);
        // pass 2: probabilities (bf16, packed) and their sum
        uint32_t pk[BKV / 2];
        float sum = 0.0f;
#pragma unroll
        for (int c = 0; c < BKV / 32; ++c) {
          uint32_t v[32];
          tmem_ld_32x32b_x32(tS + c * 32, v);
          tmem_ld_wait();
#pragma unroll
          for (int e = 0; e < 32; e += 2) {
            float pr[2];
#pragma unroll
            for (int t = 0; t < 2; ++t) {
              const int32_t key = key0 + c * 32 + e + t;
              const bool valid = key < P.T && (!P.causal || key <= q);
              pr[t] = valid ? ex2(__uint_as_float(v[e + t]) * P.scale_log2 - m_new) : 0.0f;
              sum += pr[t];
            }
            pk[(c * 32 + e) / 2] = pack2(pr[0], pr[1]);
          }
        }
        tc_fence_before();
        mbar_arrive(s_empty(b));
        ++gs;
        const float alpha = ex2(m - m_new);   // 0 for the first block (m = -inf)
        l = l * alpha + sum;
        m = m_new;
        // P's buffer and O are busy until the previous O += P V has finished
        if (gb > 0) {
          ok = wait_bounded(o_done, (gb - 1) & 1, abort_flag, P.wait, kErrWaitAttn);
          ok = __all_sync(0xffffffffu, ok);
          if (!ok) break;
          tc_fence_after();
        }
        if (j > 0 && __any_sync(0xffffffffu, alpha < 1.0f)) {
          const uint32_t tO = tmem_base + lane_off + O_COL;
#pragma unroll
          for (int c = 0; c < DH / 32; ++c) {
            uint32_t v[32];
            tmem_ld_32x32b_x32(tO + c * 32, v);
            tmem_ld_wait();
#pragma unroll
            for (int e = 0; e < 32; ++e) v[e] = __float_as_uint(__uint_as_float(v[e]) * alpha);
            tmem_st_32x32b_x32(tO + c * 32, v);
          }
          tmem_st_wait();
        }
        // P row -> shared memory, K-major with 128-byte swizzle
        const int r = quad * 32 + lane;
#pragma unroll
        for (int c = 0; c < 2; ++c) {
#pragma unroll
          for (int un = 0; un < 8; ++un) {
            const uint32_t off = c * HALF_BYTES + r * 128 + ((un ^ (r & 7)) * 16);
            const int w0 = c * 32 + un * 4;
            *reinterpret_cast<uint4*>(sP_ptr + off) = make_uint4(pk[w0], pk[w0 + 1], pk[w0 + 2], pk[w0 + 3]);
          }
        }
        fence_proxy_async_smem();
        tc_fence_before();
        mbar_arrive(p_full);
        ++gb;
      }
      if (!ok) break;
      // the unit's last O += P V
      bool ok2 = wait_bounded(o_done, (gb - 1) & 1, abort_flag, P.wait, kErrWaitAttn);
      ok2 = __all_sync(0xffffffffu, ok2);
      if (!ok2) break;
      tc_fence_after();
      const float inv_l = 1.0f / l;
      const uint32_t tO = tmem_base + lane_off + O_COL;
      __nv_bfloat16* dst = P.O + ((static_cast<int64_t>(x.shard) * P.T + q) * P.hq + x.head) * DH;
#pragma unroll
      for (int c = 0; c < DH / 32; ++c) {
        uint32_t v[32];
        tmem_ld_32x32b_x32(tO + c * 32, v);
        tmem_ld_wait();
        if (q < P.T) {
#pragma unroll
          for (int g = 0; g < 4; ++g) {
            const uint4 o4 = make_uint4(
                pack2(__uint_as_float(v[g * 8 + 0]) * inv_l, __uint_as_float(v[g * 8 + 1]) * inv_l),
                pack2(__uint_as_float(v[g * 8 + 2]) * inv_l, __uint_as_float(v[g * 8 + 3]) * inv_l),
                pack2(__uint_as_float(v[g * 8 + 4]) * inv_l, __uint_as_float(v[g * 8 + 5]) * inv_l),
                pack2(__uint_as_float(v[g * 8 + 6]) * inv_l, __uint_as_float(v[g * 8 + 7]) * inv_l));
            *reinterpret_cast<uint4*>(dst + c * 32 + g * 8) = o4;
          }
        }
      }
      tc_fence_before();
      mbar_arrive(o_empty);
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

}  // namespace

tp_status launch_tc_attention(const LaunchCtx& c, const void* Q, const void* K, const void* V,
                              void* O, int64_t T, int p, int hq, int hkv, int causal) {
  CUtensorMap mQ, mK, mV;
  if (!make_map_a(&mQ, Q, static_cast<int64_t>(hq) * DH, T, p) ||
      !make_map_a(&mK, K, static_cast<int64_t>(hkv) * DH, T, p) ||
      !make_map_a(&mV, V, static_cast<int64_t>(hkv) * DH, T, p))
    return TP_ERR_CUDA;
  static bool attr_done[64] = {};
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (!attr_done[dev]) {
      if (cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_done[dev] = true;
    }
  }
  AttnParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.p = p;
  prm.hq = hq;
  prm.hkv = hkv;
  prm.group = hq / hkv;
  prm.q_blocks = ceil_div(T, BQ);
  prm.num_units = p * hq * prm.q_blocks;
  prm.causal = causal ? 1 : 0;
  prm.scale_log2 = static_cast<float>(1.4426950408889634 / std::sqrt(static_cast<double>(DH)));
  prm.O = static_cast<__nv_bfloat16*>(O);
  prm.wait.err = c.err_word;
  prm.wait.timeout_ns = c.timeout_ns;
  prm.debug_drop = c.debug_drop;
  const int grid = prm.num_units < c.num_sms ? prm.num_units : c.num_sms;
  const cudaError_t e = launch_pdl(tc_attn_kernel, dim3(grid), dim3(NUM_THREADS), SMEM_BYTES,
                                   c.stream, mQ, mK, mV, prm);
  note_launch();
  if (e != cudaSuccess) {
    set_error_detail("attention launch failed: %s", cudaGetErrorString(e));
    return TP_ERR_CUDA;
  }
  return TP_OK;
}

}  // namespace tpk
