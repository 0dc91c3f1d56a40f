// Internal launchers shared by the C ABI translation unit and the kernel
// translation units.  Not part of the public interface.
#pragma once

#include <cuda.h>
#include <cuda_runtime.h>

#include <cstdint>

#include "tp_mlp.h"

namespace tpk {

struct LaunchCtx {
  cudaStream_t stream;
  int device;
  int num_sms;
  unsigned* err_word;    // device address of the per-device status word
  uint64_t timeout_ns;   // limit of each bounded device wait
  int64_t debug_drop;    // fault injection: pipeline slot whose load is skipped (-1: none)
  uint64_t epoch;        // changes whenever the device gets a new CUDA context: per-device
                         // caches (function attributes, streams, symbol addresses) compare it
};

// The current device and its context epoch (see LaunchCtx::epoch).
tp_status current_device(int* dev, uint64_t* epoch);

// Counts one kernel launch (process-wide, thread-safe).
void note_launch();

// ---- fixed-order partial-sum reduction (tp_reduce.cu)
cudaError_t launch_reduce(const LaunchCtx& c, const float* P, const float* b2, float* Z, int64_t T,
                          int64_t d, int p);

// ---- fp32 path, plain FMA, no TF32 (tp_simt_f32.cu)
cudaError_t launch_simt_column(const LaunchCtx& c, const float* X, const float* W1,
                               const float* Wup, const float* b1, float* Y, int64_t T, int64_t d,
                               int64_t k, int p, int act);
cudaError_t launch_simt_row(const LaunchCtx& c, const float* Y, const float* W2, float* P,
                            int64_t T, int64_t k, int64_t d, int p);
cudaError_t launch_simt_row_splitk(const LaunchCtx& c, const float* Y, const float* W2,
                                   const float* b2, float* Z, int64_t T, int64_t k, int64_t d,
                                   int p);

// ---- bf16 tensor-core path, tcgen05 + TMEM + TMA (tp_gemm_sm100.cu)
// Column layer; with `zero_cnt` it also zeroes zero_n counters for the row
// layer that follows (region_counter_bytes()).
tp_status launch_tc_column(const LaunchCtx& c, const void* X, const void* W1, const void* Wup,
                           const void* b1, void* Y, int64_t T, int64_t d, int64_t k, int p,
                           int act, int* zero_cnt = nullptr, int zero_n = 0);
// Regions of the partials whose p shard tiles the row layer counts as done
// (row layers on CTA-pair tiles only): region (m, n) covers rows
// [m*rows, +rows) and columns [n*cols, +cols); counter n*m_regions + m
// reaches `target` once every shard's tile of it is in memory.
struct RegionFold {
  int* cnt;   // null: the row layer publishes nothing, fold after it
  int rows, cols, m_regions, n_regions, target;
  int m_group;   // regions complete group by group of this many m (0: one group)
};
// Up to three identity column layers of the same X in one launch of
// CTA-pair tiles (the attention block's Q, K, V projections): *done = false
// (nothing launched) when the combined layer would not take pair tiles or a
// shard width is not a multiple of 32, and the caller launches them one by
// one.
tp_status launch_tc_column_multi(const LaunchCtx& c, const void* X, const void* const* W,
                                 void* const* Y, const int64_t* k, int nseg, int64_t T, int64_t d,
                                 int p, int* zero_cnt, int zero_n, bool* done);
// Row layer; with `region_cnt` (zeroed, region_counter_bytes()) it also
// publishes per-tile completion when it runs on CTA-pair tiles and
// describes the regions in *rf (rf->cnt stays null otherwise).
tp_status launch_tc_row(const LaunchCtx& c, const void* Y, const void* W2, float* P, int64_t T,
                        int64_t k, int64_t d, int p, int* region_cnt = nullptr,
                        RegionFold* rf = nullptr);
size_t region_counter_bytes(int64_t T, int64_t d);
// Row layer and the fixed-order fold in one launch, where it runs on CTA-pair
// tiles: shard by shard each tile adds its partial to the running sum in Z,
// the last shard adds b2, then R (fp32 [T][d], 16-byte aligned; may be null);
// region_cnt (zeroed, region_counter_bytes()) orders the shards.  *done =
// false (nothing launched) where the layer would not run on pairs: the
// caller then folds the partials itself.
tp_status launch_tc_row_chain(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                              const float* R, float* Z, int64_t T, int64_t k, int64_t d, int p,
                              int* region_cnt, bool* done);
tp_status launch_tc_row_splitk(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                               float* Z, int64_t T, int64_t k, int64_t d, int p);

// ---- tensor-core path host helpers (tp_tmap.cu)
// bf16 tensor map with 128-byte swizzle and zero fill outside the tensor
// (cached by address, sizes and box).
bool make_map(CUtensorMap* m, const void* gaddr, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box);
// [batches][rows][inner] bf16, boxes of 128 rows x 64 inner elements (K-major A tiles).
bool make_map_a(CUtensorMap* m, const void* g, int64_t inner, int64_t rows, int64_t batches);
bool make_map_f32_out(CUtensorMap* m, void* g, int64_t cols, int64_t rows, int64_t batches);
bool make_map_bf16_out(CUtensorMap* m, void* g, int64_t cols, int64_t rows, int64_t batches);
bool make_map_f32_strided(CUtensorMap* m, void* g, int64_t cols, int64_t rows, int64_t batches,
                          int64_t row_stride, int64_t batch_stride);
// [rows][cols] bf16 weight, N-contiguous, boxes of 64 rows x 64 columns (N-major B tiles).
bool make_map_b(CUtensorMap* m, const void* g, int64_t cols, int64_t rows);
// Tile width (accumulator columns) and whether to use CTA-pair tiles
// (256 rows on two SMs) for one GEMM layer of T rows, n_total output
// columns, `batches` shards and k_blocks 64-deep k slots per tile.
struct TileChoice {
  int bn;
  bool pair;
};
TileChoice pick_tile(int64_t T, int64_t n_total, int64_t batches, int64_t k_blocks, int num_sms,
                     bool swiglu, bool allow_pair, bool allow_192 = true);

inline int32_t ceil_div(int64_t a, int64_t b) { return static_cast<int32_t>((a + b - 1) / b); }

// ---- fused block (tp_block_sm100.cu): column GEMM + row GEMM (+ fixed-order
// fold of the partials, or split-K over shards) in one persistent launch.
// `counters` is zeroed device scratch of block_counter_bytes() bytes.
size_t block_counter_bytes(int64_t T, int64_t d);
tp_status launch_tc_block(const LaunchCtx& c, const void* X, const void* W1, const void* Wup,
                          const void* b1, const void* W2, const float* b2, void* Y, float* P,
                          float* Z, int* counters, int64_t T, int64_t d, int64_t k, int p, int act,
                          bool splitk);

// ---- row layer with the fixed-order fold in its epilogue (tp_gemm_fold_sm100.cu)
tp_status launch_tc_row_fold(const LaunchCtx& c, const void* Y, const void* W2, const float* b2,
                             float* Z, int64_t T, int64_t k, int64_t d, int p);

// ---- fixed-order fold overlapped with the row layer (tp_reduce.cu): the
// same additions as launch_reduce (then + R, as the row-wise fold with
// residual adds it), region by region as the counters of `rf` complete;
// launched right behind the row layer.
cudaError_t launch_fold_regions(const LaunchCtx& c, const float* P, const float* b2, float* Z,
                                int64_t T, int64_t d, int p, const RegionFold& rf,
                                const float* R = nullptr);

// ---- row-wise fold (+ bias, + residual) and LayerNorm (tp_rowops.cu)
cudaError_t launch_row_fold_ln(const LaunchCtx& c, const float* P, int p, const float* bias,
                               const float* R, float* H, const float* gamma, const float* beta,
                               void* Y, int64_t T, int64_t d, float eps);

cudaError_t launch_colsum(const LaunchCtx& c, const void* A, float* out, float* scratch,
                          int64_t batches, int64_t R, int64_t n, int64_t out_batch_stride);

// ---- backward pass of the MLP block (tp_gemm_bwd_sm100.cu)
tp_status launch_bwd_act_grad(const LaunchCtx& c, const void* dZ, const void* W2, const void* H,
                              const void* Hup, void* dH, void* dU, int64_t T, int64_t d, int64_t k,
                              int p, int act);
// dX partials; with `region_cnt` (zeroed, region_counter_bytes()) it also
// publishes per-tile completion when it runs on CTA pairs and says so in *rf.
tp_status launch_bwd_dx_partials(const LaunchCtx& c, const void* dH, const void* dU,
                                 const void* W1, const void* Wup, float* P, int64_t T, int64_t d,
                                 int64_t k, int p, int* region_cnt = nullptr,
                                 RegionFold* rf = nullptr);
// Whether the dX partials run on CTA-pair tiles (k_eff: k, or 2k for SwiGLU).
bool bwd_dx_on_pairs(const LaunchCtx& c, int64_t T, int64_t k_eff, int64_t d, int p);
tp_status launch_bwd_dw1(const LaunchCtx& c, const void* X, const void* dH, const void* dU,
                         float* dW1, float* dWup, int64_t T, int64_t d, int64_t k, int p);
tp_status launch_bwd_dw2(const LaunchCtx& c, const void* Y, const void* dZ, float* dW2, int64_t T,
                         int64_t d, int64_t k, int p);

// ---- attention of every shard's heads (tp_attn_sm100.cu), head_dim 128, bf16
tp_status launch_tc_attention(const LaunchCtx& c, const void* Q, const void* K, const void* V,
                              void* O, int64_t T, int p, int hq, int hkv, int causal);

// ---- the all-reduce of partials held on p GPUs (tp_allreduce.cu)
// Z_q[rows of the slab] = fixed-order fold of parts[0..p) (+ b2), for q < n_out.
cudaError_t launch_gather_fold(const LaunchCtx& c, const float* const* parts, int p,
                               const float* b2, float* const* outs, int n_out, int64_t row0,
                               int64_t rows, int64_t d);
tp_status ipc_export(const void* ptr, tp_ipc_handle* h);
tp_status ipc_import(const tp_ipc_handle* h, void** ptr);
tp_status ipc_release(const tp_ipc_handle* h);

// Test hook: the attention softmax's 2^x polynomial applied to x[0..n).
cudaError_t launch_exp2_poly_probe(const LaunchCtx& c, const float* x, float* y, int64_t n);

// Records a human-readable detail for tp_last_error_detail().
void set_error_detail(const char* fmt, ...);

}  // namespace tpk
