// Attention of every shard's own heads, one persistent tcgen05 launch (sm_100a).
//
// The tensor-parallel attention block gives each shard h/p query heads (and
// h_kv/p key/value heads) through column-parallel Q, K, V projections; the
// attention itself then runs on each shard's heads with no communication
// (day-41 post, "Attention heads: naturally parallel"; "Tensor parallel
// math", "Attention: parallel across heads": softmax(Q K^T / sqrt(d_k)) V per
// head).  This kernel computes it for all shards and heads at once.
//
// Work unit: (shard, query head, pair of 128-query tiles); the two tiles share
// every K/V block load.  Key/value blocks of 128.  Roles (384 threads):
//   warp 0 lane 0  TMA: the unit's two Q tiles once, then K_j and V_j per key
//                  block through a 2-slot ring (128-byte swizzle);
//   warp 1 lane 0  MMA: S_t = Q_t K_j^T into tile t's TMEM score buffer
//                  (128 x 128 fp32); O_t += P_t V_j with P_t read from TMEM,
//                  where the softmax left it (bf16, over the first 64 columns
//                  of the score buffer).  Issue order per block:
//                  PV_0 -> S_0(next) -> PV_1 -> S_1(next), so the tensor core
//                  runs one tile's products while the other tile's softmax
//                  runs.  Only the Q K^T products read the Q tiles, so they
//                  are handed back to the producer as soon as the unit's last
//                  one completes: the next unit's Q load overlaps this unit's
//                  last softmax and P V products;
//   warp 2         TMEM allocation;
//   warps 4..7     online softmax of tile 0, warps 8..11 of tile 1: thread =
//                  query row (its TMEM lane), one round trip to TMEM per
//                  block (all 128 scores loaded at once); scores in the log2
//                  domain; the row max in registers (3-input max, four
//                  independent chains); exponent arguments, sums in packed
//                  fp32 pairs; exp2 by MUFU (ex2.approx) for 3/4 of the
//                  elements and by a polynomial on the FMA pipe for 1/4, so
//                  the MUFU unit (16 per clock per SM) is not the only one.
//                  The running maximum is only moved when it grows by more
//                  than 2^8 (the stale maximum is exact once the sum and O
//                  share it), so O is rarely rescaled; when it is, the thread
//                  scales its O row in TMEM -- safe without a wait, because
//                  the score block it just read was committed after the
//                  previous O += P V.  At the end O is divided by the row
//                  sum, converted to bf16 and stored.
// Keys beyond T and (causal) keys after the query are masked, on the blocks
// that hold any.  Causal units are taken longest first.  Every barrier wait
// is bounded.
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
constexpr int BQ = 128;                 // queries per tile (TMEM lanes)
constexpr int BKV = 128;                // keys per block
constexpr int NQT = 2;                  // query tiles per unit
constexpr int NST = 2;                  // K/V ring slots
constexpr int TILE_BYTES = 128 * 128 * 2;   // one 128 x 128 bf16 tile (two 64-column boxes)
constexpr int HALF_BYTES = TILE_BYTES / 2;  // one box: 128 rows x 64 columns
constexpr int SMEM_BYTES = 1024 + NQT * TILE_BYTES + NST * 2 * TILE_BYTES + 256;
constexpr int NUM_THREADS = 384;
constexpr uint32_t IDESC_S = idesc_bf16_f32(BQ, BKV, /*a_mn=*/0, /*b_mn=*/0);  // Q K^T
constexpr uint32_t IDESC_O = idesc_bf16_f32(BQ, DH, /*a_mn=*/0, /*b_mn=*/1);   // P V
constexpr uint32_t O_COL0 = NQT * BKV, TMEM_COLS = 512;   // S_t at t*128, O_t at 256 + t*128
constexpr float RESCALE_LOG2 = 8.0f;
constexpr int POLY_PAIRS = 2;           // of every 8 probability pairs, this many use the
                                        // polynomial exp2 on the FMA pipe, the rest MUFU    // move the running maximum only past this growth
constexpr unsigned kErrWaitAttn = 1u << 6;

struct AttnParams {
  int32_t T, p, hq, hkv, group, q_blocks, q_pairs, num_units, causal;
  float scale_log2;          // log2(e) / sqrt(DH)
  __nv_bfloat16* O;          // [p][T][hq*DH]
  WaitCtl wait;
  int64_t debug_drop;
};

struct Unit {
  int32_t shard, head, kvh, qb0, nkb0, nkb1, nmax;
  // key blocks of query tile t (0 when the tile lies beyond T)
  __device__ __forceinline__ int32_t nkb(int t) const { return t == 0 ? nkb0 : nkb1; }
};

__device__ __forceinline__ Unit decode_unit(const AttnParams& P, int32_t u) {
  Unit x;
  const int32_t heads = P.p * P.hq;
  const int32_t level = u / heads;
  const int32_t hh = u % heads;
  // causal: the longest query pairs first
  const int32_t qp = P.causal ? P.q_pairs - 1 - level : level;
  x.shard = hh / P.hq;
  x.head = hh % P.hq;
  x.kvh = x.head / P.group;
  x.qb0 = qp * NQT;
  const int32_t all = (P.T + BKV - 1) / BKV;
  auto blocks = [&](int32_t qb) {
    return qb >= P.q_blocks ? 0 : (P.causal ? (qb + 1 < all ? qb + 1 : all) : all);
  };
  x.nkb0 = blocks(x.qb0);
  x.nkb1 = blocks(x.qb0 + 1);
  x.nmax = x.nkb0 > x.nkb1 ? x.nkb0 : x.nkb1;   // causal: tile 1 never has fewer
  return x;
}

// The CTA's r-th unit: rounds of gridDim.x units, alternately walked
// forwards and backwards across the CTAs ("snake" order), so that with the
// longest causal units first every CTA gets a similar total (the plain
// round-robin left one CTA with 1.3x the average on the 4-shard shape).
__device__ __forceinline__ int32_t unit_of(int32_t r) {
  const int32_t g = static_cast<int32_t>(gridDim.x), b = static_cast<int32_t>(blockIdx.x);
  return r * g + ((r & 1) ? g - 1 - b : b);
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

// The softmax's hot loop uses the packed fp32 pair helpers f2_* of
// tp_device.cuh (sm_100 FFMA2 / FADD2: two lanes per instruction).
__device__ __forceinline__ float max3(float a, float b, float c) {
  float d;
  asm("max.f32 %0, %1, %2, %3;" : "=f"(d) : "f"(a), "f"(b), "f"(c));
  return d;
}

// 2^x on the FMA pipe, for part of the probabilities so that the MUFU unit
// (16 exp2 per clock per SM) is not the only one computing them: range
// reduction to the nearest integer n (x = n + f, |f| <= 1/2, by the
// 1.5 * 2^23 rounding constant), a degree-4 polynomial for 2^f whose
// coefficients were fitted to minimise the relative error on [-1/2, 1/2]
// (iteratively reweighted least squares; max relative error of the fit
// 2.6e-6, of the fp32 evaluation below at most 2.7e-6 on [-126, 0]), and n
// added to the exponent field.  x is clamped to >= -126 (the probabilities
// are bf16, so 2^-126 and 0 are the same to them).  Two lanes per call.
__device__ __forceinline__ uint64_t exp2_poly2(uint64_t x2) {
  float x0, x1;
  f2_unpack(x2, x0, x1);
  x2 = f2_pack(fmaxf(x0, -126.0f), fmaxf(x1, -126.0f));
  const uint64_t magic = f2_pack(12582912.0f, 12582912.0f);
  const uint64_t t = f2_add(x2, magic);
  const uint64_t n = f2_add(t, f2_pack(-12582912.0f, -12582912.0f));
  const uint64_t f = f2_fma(n, f2_pack(-1.0f, -1.0f), x2);
  uint64_t p = f2_fma(f2_pack(0.009570101276040077f, 0.009570101276040077f), f,
                      f2_pack(0.05591785907745361f, 0.05591785907745361f));
  p = f2_fma(p, f, f2_pack(0.240247443318367f, 0.240247443318367f));
  p = f2_fma(p, f, f2_pack(0.6931217908859253f, 0.6931217908859253f));
  p = f2_fma(p, f, f2_pack(0.9999992847442627f, 0.9999992847442627f));
  float p0, p1, t0, t1;
  f2_unpack(p, p0, p1);
  f2_unpack(t, t0, t1);
  return f2_pack(__int_as_float(__float_as_int(p0) + (__float_as_int(t0) << 23)),
                 __int_as_float(__float_as_int(p1) + (__float_as_int(t1) << 23)));
}

// One softmax step of a thread's row over a 128-key block in TMEM columns
// [tS, tS+128), with a single round trip to tensor memory: all 128 scores
// are loaded at once (one wait), the maximum is taken in registers, the
// running maximum updated (moved only past RESCALE_LOG2 growth), and the
// probabilities written back as bf16 pairs into columns [tS, tS+64).
// Returns the block's probability sum; m and alpha are updated in place.
template <bool MASK>
__device__ __forceinline__ float softmax_one_pass(uint32_t tS, float scale, float& m, float& alpha,
                                                  bool& grow, int32_t key0, int32_t T,
                                                  int32_t causal, int32_t q) {
  uint32_t v[128];
#pragma unroll
  for (int c = 0; c < 4; ++c)
    tmem_ld_32x32b_x32(tS + c * 32, *reinterpret_cast<uint32_t(*)[32]>(&v[c * 32]));
  tmem_ld_wait();
  if (MASK) {
#pragma unroll
    for (int e = 0; e < 128; ++e) {
      const int32_t key = key0 + e;
      if (key >= T || (causal && key > q)) v[e] = __float_as_uint(-INFINITY);
    }
  }
  float acc[4] = {-INFINITY, -INFINITY, -INFINITY, -INFINITY};
#pragma unroll
  for (int e = 0; e < 128; e += 8) {
    const int a = (e / 8) & 3;
    acc[a] = max3(acc[a], __uint_as_float(v[e]), __uint_as_float(v[e + 1]));
    acc[a] = max3(acc[a], __uint_as_float(v[e + 2]), __uint_as_float(v[e + 3]));
    acc[a] = max3(acc[a], __uint_as_float(v[e + 4]), __uint_as_float(v[e + 5]));
    acc[a] = max3(acc[a], __uint_as_float(v[e + 6]), __uint_as_float(v[e + 7]));
  }
  const float m_cand = max3(acc[0], acc[1], fmaxf(acc[2], acc[3])) * scale;
  grow = m_cand > m + RESCALE_LOG2;
  alpha = grow ? ex2(m - m_cand) : 1.0f;
  if (grow) m = m_cand;
  const uint64_t sc2 = f2_pack(scale, scale);
  const uint64_t nm2 = f2_pack(-m, -m);
  uint64_t sum2[2] = {f2_pack(0.0f, 0.0f), f2_pack(0.0f, 0.0f)};
#pragma unroll
  for (int c = 0; c < 4; ++c) {
    uint32_t pk[16];
#pragma unroll
    for (int e = 0; e < 32; e += 2) {
      const int i = c * 32 + e;
      const uint64_t xa = f2_fma(f2_pack(__uint_as_float(v[i]), __uint_as_float(v[i + 1])), sc2, nm2);
      float a0, a1;
      if ((e / 2) % 8 < POLY_PAIRS) {
        f2_unpack(exp2_poly2(xa), a0, a1);
      } else {
        float x0, x1;
        f2_unpack(xa, x0, x1);
        a0 = ex2(x0);
        a1 = ex2(x1);
      }
      sum2[(e / 2) & 1] = f2_add(sum2[(e / 2) & 1], f2_pack(a0, a1));
      pk[e / 2] = pack2(a0, a1);
    }
    tmem_st_32x32b_x16(tS + c * 16, pk);
  }
  tmem_st_wait();
  float s0, s1, s2, s3;
  f2_unpack(sum2[0], s0, s1);
  f2_unpack(sum2[1], s2, s3);
  return (s0 + s1) + (s2 + s3);
}

__global__ void __launch_bounds__(NUM_THREADS, 1)
    tc_attn_kernel(const __grid_constant__ CUtensorMap mapQ, const __grid_constant__ CUtensorMap mapK,
                   const __grid_constant__ CUtensorMap mapV, const AttnParams P) {
  extern __shared__ uint8_t smem_raw[];
  const uint32_t raw = smem_u32(smem_raw);
  const uint32_t base = (raw + 1023u) & ~1023u;
  auto sQ = [&](uint32_t t) { return base + t * TILE_BYTES; };
  auto sK = [&](uint32_t st) { return base + NQT * TILE_BYTES + st * 2 * TILE_BYTES; };
  auto sV = [&](uint32_t st) { return base + NQT * TILE_BYTES + st * 2 * TILE_BYTES + TILE_BYTES; };
  uint8_t* const ctrl = smem_raw + (base - raw) + NQT * TILE_BYTES + NST * 2 * TILE_BYTES;
  uint64_t* const bars = reinterpret_cast<uint64_t*>(ctrl);
  // barrier slots
  const uint32_t q_full = smem_u32(&bars[0]), q_empty = smem_u32(&bars[1]);
  auto kv_full = [&](uint32_t s) { return smem_u32(&bars[2 + s]); };
  auto kv_empty = [&](uint32_t s) { return smem_u32(&bars[2 + NST + s]); };
  auto s_full = [&](uint32_t t) { return smem_u32(&bars[2 + 2 * NST + t]); };
  auto p_full = [&](uint32_t t) { return smem_u32(&bars[2 + 2 * NST + NQT + t]); };
  auto o_full = [&](uint32_t t) { return smem_u32(&bars[2 + 2 * NST + 2 * NQT + t]); };
  auto o_empty = [&](uint32_t t) { return smem_u32(&bars[2 + 2 * NST + 3 * NQT + t]); };
  const uint32_t drain = smem_u32(&bars[2 + 2 * NST + 4 * NQT]);
  constexpr int NBARS = 3 + 2 * NST + 4 * NQT;
  uint32_t* const tmem_slot = reinterpret_cast<uint32_t*>(ctrl + 8 * NBARS);
  volatile int* const abort_flag = reinterpret_cast<volatile int*>(tmem_slot + 1);

  const int warp = threadIdx.x / 32, lane = threadIdx.x % 32;
  if (threadIdx.x == 0) {
    mbar_init(q_full, 1);
    mbar_init(q_empty, 1);
    for (int s = 0; s < NST; ++s) {
      mbar_init(kv_full(s), 1);
      mbar_init(kv_empty(s), 1);
    }
    for (int t = 0; t < NQT; ++t) {
      mbar_init(s_full(t), 1);
      mbar_init(p_full(t), 128);
      mbar_init(o_full(t), 1);
      mbar_init(o_empty(t), 128);
    }
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
      for (int32_t u = unit_of(0); ok && u < P.num_units; u = unit_of(++lu)) {
        const Unit x = decode_unit(P, u);
        if (!wait_bounded(q_empty, (lu & 1) ^ 1u, abort_flag, P.wait, kErrWaitAttn)) break;
        const int ntiles = x.nkb1 > 0 ? 2 : 1;
        mbar_arrive_expect_tx(q_full, ntiles * TILE_BYTES);
        for (int t = 0; t < ntiles; ++t)
          for (int c = 0; c < 2; ++c)
            tma_load_3d(sQ(t) + c * HALF_BYTES, &mapQ, q_full, x.head * DH + c * 64,
                        (x.qb0 + t) * BQ, x.shard);
        last_q = lu;
        for (int32_t j = 0; j < x.nmax; ++j) {
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
      // K/V blocks arrive in the producer's order: block n of the whole
      // sequence sits in ring slot n % NST, phase (n / NST) & 1.
      uint32_t kv_n = 0;             // K/V blocks of finished units
      uint32_t pv[NQT] = {0, 0};     // O += P V products per tile (p_full phases)
      uint32_t ou[NQT] = {0, 0};     // units per tile with an output (o_empty phases)
      int32_t lu = 0;
      bool ok = true;
      auto wait_kv = [&](uint32_t n) {
        return wait_bounded(kv_full(n % NST), (n / NST) & 1, abort_flag, P.wait, kErrWaitFull);
      };
      auto issue_s = [&](uint32_t t, uint32_t n) {
        const uint32_t kst = n % NST;
#pragma unroll
        for (int kk = 0; kk < DH / 16; ++kk) {
          const uint32_t off = (kk >> 2) * HALF_BYTES + (kk & 3) * 32;
          tc_mma_f16(tmem_base + t * BKV, smem_desc_sw128(sQ(t) + off, 16, 1024),
                     smem_desc_sw128(sK(kst) + off, 16, 1024), IDESC_S, kk > 0 ? 1u : 0u);
        }
        tc_commit(s_full(t));
      };
      for (int32_t u = unit_of(0); ok && u < P.num_units; u = unit_of(++lu)) {
        const Unit x = decode_unit(P, u);
        if (!wait_bounded(q_full, lu & 1, abort_flag, P.wait, kErrWaitAttn)) break;
        const uint32_t n0 = kv_n;
        if (!wait_kv(n0)) break;
        tc_fence_after();
#pragma unroll
        for (int t = 0; t < NQT; ++t)
          if (x.nkb(t) > 0) issue_s(t, n0);
        // Q is read only by the Q K^T products: once the unit's last one is
        // issued, a commit hands the Q tiles back to the producer, which
        // loads the next unit's while this unit's last softmax and P V run.
        int s_pending = 0;   // tiles whose last Q K^T product is still to be issued
#pragma unroll
        for (int t = 0; t < NQT; ++t)
          if (x.nkb(t) > 1) ++s_pending;
        if (s_pending == 0) tc_commit(q_empty);
        for (int32_t j = 0; ok && j < x.nmax; ++j) {
          const uint32_t vst = (n0 + j) % NST;
#pragma unroll
          for (int t = 0; t < NQT; ++t) {
            if (j >= x.nkb(t)) continue;
            if (j == 0 && ou[t] > 0 &&
                !wait_bounded(o_empty(t), (ou[t] - 1) & 1, abort_flag, P.wait, kErrWaitAttn)) {
              ok = false;
              break;
            }
            if (!wait_bounded(p_full(t), pv[t] & 1, abort_flag, P.wait, kErrWaitAttn)) {
              ok = false;
              break;
            }
            tc_fence_after();
#pragma unroll
            for (int kk = 0; kk < BKV / 16; ++kk) {
              const uint64_t bdesc = smem_desc_sw128(sV(vst) + kk * 16 * 128, HALF_BYTES, 1024);
              tc_mma_f16_ts(tmem_base + O_COL0 + t * DH, tmem_base + t * BKV + kk * 8, bdesc,
                            IDESC_O, (j > 0 || kk > 0) ? 1u : 0u);
            }
            ++pv[t];
            // the last tile that uses block j releases its ring slot
            const bool last_user = (t == NQT - 1) || (j >= x.nkb1);
            if (last_user) tc_commit(kv_empty(vst));
            if (j + 1 < x.nkb(t)) {
              if (!wait_kv(n0 + j + 1)) {
                ok = false;
                break;
              }
              tc_fence_after();
              issue_s(t, n0 + j + 1);
              if (j + 2 == x.nkb(t) && --s_pending == 0) tc_commit(q_empty);
            } else {
              tc_commit(o_full(t));
            }
          }
        }
        if (!ok) break;
#pragma unroll
        for (int t = 0; t < NQT; ++t)
          if (x.nkb(t) > 0) ++ou[t];
        kv_n = n0 + x.nmax;
      }
      tc_commit(drain);
      wait_teardown(drain, 0, P.wait);
    }
    __syncwarp();
  } else if (warp >= 4) {
    // ------------------------------------------------------- softmax / output
    const int t = (warp - 4) / 4;          // query tile of this warpgroup
    const int quad = warp & 3;             // TMEM lane quarter this warp may access
    const uint32_t lane_off = static_cast<uint32_t>(quad * 32) << 16;
    const uint32_t tS = tmem_base + lane_off + t * BKV;
    const uint32_t tO = tmem_base + lane_off + O_COL0 + t * DH;
    const float scale = P.scale_log2;
    uint32_t sc = 0, uc = 0;
    int32_t ru = 0;
    for (int32_t u = unit_of(0); u < P.num_units; u = unit_of(++ru)) {
      const Unit x = decode_unit(P, u);
      const int32_t nkb = x.nkb(t);
      if (nkb == 0) continue;
      const int32_t q0 = (x.qb0 + t) * BQ;
      const int32_t q = q0 + quad * 32 + lane;
      float m = -INFINITY, l = 0.0f;
      bool ok = true;
      for (int32_t j = 0; j < nkb; ++j) {
        ok = wait_bounded(s_full(t), sc & 1, abort_flag, P.wait, kErrWaitAttn);
        ok = __all_sync(0xffffffffu, ok);
        if (!ok) break;
        tc_fence_after();
        const int32_t key0 = j * BKV;
        const bool masked = (key0 + BKV > P.T) || (P.causal && key0 + BKV - 1 > q0);
        float alpha;
        bool grow;
        const float sum = masked
            ? softmax_one_pass<true>(tS, scale, m, alpha, grow, key0, P.T, P.causal, q)
            : softmax_one_pass<false>(tS, scale, m, alpha, grow, key0, P.T, P.causal, q);
        if (j > 0 && __any_sync(0xffffffffu, grow)) {
          // O += P V of the previous block has completed (it was issued
          // before this score block, whose commit we waited for)
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
        l = l * alpha + sum;
        tc_fence_before();
        mbar_arrive(p_full(t));
        ++sc;
      }
      if (!ok) break;
      // the tile's last O += P V
      bool ok2 = wait_bounded(o_full(t), uc & 1, abort_flag, P.wait, kErrWaitAttn);
      ok2 = __all_sync(0xffffffffu, ok2);
      if (!ok2) break;
      tc_fence_after();
      const float inv_l = 1.0f / l;
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
      mbar_arrive(o_empty(t));
      ++uc;
    }
  }

  __syncthreads();
  if (warp == 2) {
    tc_fence_after();
    tmem_dealloc(tmem_base, TMEM_COLS);
  }
}

// Test hook: y[i] = exp2_poly2(x[i]) for i < n, two elements per thread
// (an odd tail pairs the last element with a dummy lane).
__global__ void exp2_poly_probe_kernel(const float* __restrict__ x, float* __restrict__ y,
                                       int64_t n) {
  const int64_t i = 2 * (static_cast<int64_t>(blockIdx.x) * blockDim.x + threadIdx.x);
  if (i >= n) return;
  const float x0 = x[i];
  const float x1 = i + 1 < n ? x[i + 1] : 0.0f;
  float y0, y1;
  f2_unpack(exp2_poly2(f2_pack(x0, x1)), y0, y1);
  y[i] = y0;
  if (i + 1 < n) y[i + 1] = y1;
}

}  // namespace

cudaError_t launch_exp2_poly_probe(const LaunchCtx& c, const float* x, float* y, int64_t n) {
  if (n == 0) return cudaSuccess;
  const int threads = 256;
  const int64_t blocks = (n + 2 * threads - 1) / (2 * threads);
  exp2_poly_probe_kernel<<<static_cast<unsigned>(blocks), threads, 0, c.stream>>>(x, y, n);
  note_launch();
  return cudaGetLastError();
}

tp_status launch_tc_attention(const LaunchCtx& c, const void* Q, const void* K, const void* V,
                              void* O, int64_t T, int p, int hq, int hkv, int causal) {
  CUtensorMap mQ, mK, mV;
  if (!make_map_a(&mQ, Q, static_cast<int64_t>(hq) * DH, T, p) ||
      !make_map_a(&mK, K, static_cast<int64_t>(hkv) * DH, T, p) ||
      !make_map_a(&mV, V, static_cast<int64_t>(hkv) * DH, T, p))
    return TP_ERR_CUDA;
  static uint64_t attr_epoch[64] = {};   // context epoch the attribute was set under
  static std::mutex mu;
  {
    std::lock_guard<std::mutex> lk(mu);
    const int dev = c.device & 63;
    if (attr_epoch[dev] != c.epoch) {
      if (cudaFuncSetAttribute(tc_attn_kernel, cudaFuncAttributeMaxDynamicSharedMemorySize,
                               SMEM_BYTES) != cudaSuccess) {
        set_error_detail("cudaFuncSetAttribute failed: %s", cudaGetErrorString(cudaGetLastError()));
        return TP_ERR_CUDA;
      }
      attr_epoch[dev] = c.epoch;
    }
  }
  AttnParams prm{};
  prm.T = static_cast<int32_t>(T);
  prm.p = p;
  prm.hq = hq;
  prm.hkv = hkv;
  prm.group = hq / hkv;
  prm.q_blocks = ceil_div(T, BQ);
  prm.q_pairs = ceil_div(prm.q_blocks, NQT);
  prm.num_units = p * hq * prm.q_pairs;
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
