// Host-side helpers of the tensor-core path: TMA tensor maps (with a small
// cache, since the same buffers come back call after call) and the choice of
// tile width.
#include <cuda.h>
#include <cudaTypedefs.h>
#include <cuda_runtime.h>

#include <algorithm>
#include <climits>
#include <cstdint>
#include <cstring>
#include <mutex>

#include "tp_internal.h"

namespace tpk {
namespace {

constexpr uint32_t kBoxK = 64;      // k per pipeline slot (one 128-byte swizzle row of bf16)
constexpr uint32_t kBoxRows = 128;  // A-tile rows
constexpr uint32_t kBoxCols = 64;   // B box width (one swizzle atom)

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
  int dtype;
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

}  // namespace

// bf16 tensor map, 128-byte swizzle, zero fill outside the tensor.
bool make_map_typed(CUtensorMap* m, const void* gaddr, int rank, const uint64_t* dims,
                    const uint64_t* strides_bytes, const uint32_t* box, bool f32,
                    bool swizzle64 = false) {
  MapKey key;
  memset(&key, 0, sizeof(key));
  key.g = gaddr;
  key.dtype = (f32 ? 1 : 0) | (swizzle64 ? 2 : 0);
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
      fn(m, f32 ? CU_TENSOR_MAP_DATA_TYPE_FLOAT32 : CU_TENSOR_MAP_DATA_TYPE_BFLOAT16, static_cast<cuuint32_t>(rank),
         const_cast<void*>(gaddr), d, st, bx, es, CU_TENSOR_MAP_INTERLEAVE_NONE,
         swizzle64 ? CU_TENSOR_MAP_SWIZZLE_64B : CU_TENSOR_MAP_SWIZZLE_128B,
         CU_TENSOR_MAP_L2_PROMOTION_L2_256B,
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

bool make_map(CUtensorMap* m, const void* gaddr, int rank, const uint64_t* dims,
              const uint64_t* strides_bytes, const uint32_t* box) {
  return make_map_typed(m, gaddr, rank, dims, strides_bytes, box, false);
}

// fp32 output [batches][rows][cols] for bulk tensor stores of 32 x 32 boxes
// (one 128-byte swizzle row of fp32 per box row).
bool make_map_f32_out(CUtensorMap* m, void* g, int64_t cols, int64_t rows, int64_t batches) {
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batches)};
  const uint64_t strides[2] = {static_cast<uint64_t>(cols) * 4,
                               static_cast<uint64_t>(cols) * rows * 4};
  const uint32_t box[3] = {32, 32, 1};
  return make_map_typed(m, g, 3, dims, strides, box, true);
}

// fp32 output with explicit row and batch strides (elements), boxes 32 x 32
// (a shard's column block inside a wider matrix: batch stride = the block's
// width); false if the driver does not accept the layout.
bool make_map_f32_strided(CUtensorMap* m, void* g, int64_t cols, int64_t rows, int64_t batches,
                          int64_t row_stride, int64_t batch_stride) {
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batches)};
  const uint64_t strides[2] = {static_cast<uint64_t>(row_stride) * 4,
                               static_cast<uint64_t>(batch_stride) * 4};
  const uint32_t box[3] = {32, 32, 1};
  return make_map_typed(m, g, 3, dims, strides, box, true);
}

// bf16 output [batches][rows][cols] for bulk tensor stores of 32 x 32 boxes
// (64-byte rows, 64-byte swizzle).
bool make_map_bf16_out(CUtensorMap* m, void* g, int64_t cols, int64_t rows, int64_t batches) {
  const uint64_t dims[3] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batches)};
  const uint64_t strides[2] = {static_cast<uint64_t>(cols) * 2,
                               static_cast<uint64_t>(cols) * rows * 2};
  const uint32_t box[3] = {32, 32, 1};
  return make_map_typed(m, g, 3, dims, strides, box, false, true);
}

// [rows][inner] bf16 matrices stacked `batches` times, boxes of 128 x 64.
bool make_map_a(CUtensorMap* m, const void* g, int64_t inner, int64_t rows, int64_t batches) {
  const uint64_t dims[3] = {static_cast<uint64_t>(inner), static_cast<uint64_t>(rows),
                            static_cast<uint64_t>(batches)};
  const uint64_t strides[2] = {static_cast<uint64_t>(inner) * 2,
                               static_cast<uint64_t>(inner) * rows * 2};
  const uint32_t box[3] = {kBoxK, kBoxRows, 1};
  return make_map(m, g, 3, dims, strides, box);
}

// [rows = k][cols = n] bf16 weight, N-contiguous, boxes of 64 k-rows x 64 cols.
bool make_map_b(CUtensorMap* m, const void* g, int64_t cols, int64_t rows) {
  const uint64_t dims[2] = {static_cast<uint64_t>(cols), static_cast<uint64_t>(rows)};
  const uint64_t strides[1] = {static_cast<uint64_t>(cols) * 2};
  const uint32_t box[2] = {kBoxCols, kBoxK};
  return make_map(m, g, 2, dims, strides, box);
}


// Tile choice for one GEMM layer.  Per tile: k slots x max(MMA cycles,
// operand bytes / ingest rate) + a fixed cost (pipeline fill, epilogue);
// waves = tiles over the SMs (single-CTA tiles) or SM pairs (pair tiles);
// minimise waves x per-tile cost.  Per 64-deep k slot, a single-CTA tile of
// width BN issues 2*BN MMA cycles and loads 16 KiB of A + 128*BN bytes of B;
// a pair tile of width PBN loads 16 KiB + 64*PBN bytes per CTA for 2*PBN
// cycles.  Ingest is taken as 80 bytes per SM cycle and the fixed cost as
// 2000 cycles (both from the measured kernels).  Pair tiles need at least
// 256 rows and are considered only when single-CTA tiles need more than one
// wave.  Ties keep the earlier (wider, single-CTA) choice.
TileChoice pick_tile(int64_t T, int64_t n_total, int64_t batches, int64_t k_blocks, int num_sms,
                     bool swiglu, bool allow_pair, bool allow_192) {
  constexpr double kIngest = 80.0, kFixed = 2000.0;
  TileChoice best{256, false};
  double best_cost = 1e300;
  int64_t best_tiles = 0;
  auto consider = [&](int bn, bool pair) {
    const int64_t out_cols = swiglu ? bn / 2 : bn;
    const int64_t rows = pair ? 256 : 128;
    const int64_t tiles = ((T + rows - 1) / rows) * ((n_total + out_cols - 1) / out_cols) * batches;
    const int64_t slots = pair ? num_sms / 2 : num_sms;
    const double waves = static_cast<double>((tiles + slots - 1) / slots);
    const double b_bytes = pair ? 64.0 * bn : 128.0 * bn;
    const double kb = std::max(2.0 * bn, (16384.0 + b_bytes) / kIngest);
    const double cost = waves * (static_cast<double>(k_blocks) * kb + kFixed);
    if (cost < best_cost * (1.0 - 1e-9)) {
      best_cost = cost;
      best = TileChoice{bn, pair};
      best_tiles = tiles;
    }
  };
  consider(256, false);
  if (!swiglu && allow_192) consider(192, false);
  consider(128, false);
  if (!swiglu) consider(64, false);
  // Pair tiles only pay once the layer takes more than one wave of
  // single-CTA tiles (measured: they slowed the one-wave GPT-2 layers).
  if (allow_pair && T >= 256 && best_tiles > num_sms) {
    consider(256, true);
    consider(128, true);
  }
  return best;
}

}  // namespace tpk
