/*
 * tp_mlp.h -- C ABI of libtpmlp: the Megatron tensor-parallel MLP block run
 * as p simulated shards on one NVIDIA B200 (sm_100a).
 *
 * The method (column-parallel first layer, per-shard activation, row-parallel
 * second layer, one sum of partials) is the one set out on the pages:
 *   - "Simulating column parallel linear", "Simulating row parallel linear"
 *     and "Pairing them: the Megatron-LM MLP" (skandtandon.pages.dev, day-41
 *     post on tensor parallelism);
 *   - "Column-parallel: split the weight by output columns", "Row-parallel:
 *     split the weight by input rows", "The MLP block: column then row, one
 *     all-reduce" (aicassindra.com, "Tensor parallel math");
 *   - sections 1.A, 1.B and 2.B of "Tensor Parallelism Explained: Splitting
 *     Attention and FFN Weights Across GPUs" (initnode.dev), 2.B being the
 *     SwiGLU variant.
 *
 * Notation: T tokens, d model width, k FFN width, p shards, s = k/p.
 * All matrices are dense and row-major.  Weights are stored [in, out]
 * (Y = X W), as on the day-41 post and "Tensor parallel math".
 *
 * Conventions shared by every call:
 *   - Every pointer is a DEVICE pointer owned by the caller, unless a call
 *     says otherwise (the host-buffer block, the pointer tables of the
 *     p-GPU fold and the IPC handles are host memory).  The library never
 *     allocates device memory and never frees caller memory.
 *   - Calls are asynchronous on `stream` (a cudaStream_t; NULL = the legacy
 *     default stream).  Argument errors are returned synchronously before
 *     anything is launched; a CUDA launch error returns TP_ERR_CUDA.
 *   - Every wait inside the tensor-core kernels is bounded (default 2 s,
 *     see tp_set_wait_timeout_ns).  A wait that runs out makes the kernel
 *     record TP_ERR_DEVICE_TIMEOUT in a per-device status word and return;
 *     tp_sync_status() reports and clears it.  Nothing traps or spins forever.
 *   - dtype TP_BF16: X, weights, b1 and the hidden shards are bf16; products
 *     accumulate in fp32 (tcgen05 tensor cores, TMEM accumulators); partials,
 *     b2 and Z are fp32.  Requires d % 8 == 0, s % 8 == 0 and 16-byte aligned
 *     X, W1, W_up, Y, W2, partials and Z (TMA row pitches), else
 *     TP_ERR_ALIGNMENT.
 *   - dtype TP_F32: everything fp32, plain fp32 FMA (no TF32); any sizes,
 *     4-byte alignment.
 *   - T == 0 (no tokens) is valid: nothing is launched, TP_OK is returned.
 */
#ifndef TP_MLP_H
#define TP_MLP_H

#include <stddef.h>
#include <stdint.h>

#ifdef __cplusplus
extern "C" {
#endif

typedef enum {
  TP_OK = 0,
  TP_ERR_INVALID_ARG = 1,     /* null pointer, p < 1, negative size, bad enum   */
  TP_ERR_INDIVISIBLE = 2,     /* k % p != 0: the walkthrough asserts
                                 out_features % num_gpus == 0 before slicing
                                 ("Simulating column parallel linear") and
                                 in_features % num_gpus == 0 for the row split */
  TP_ERR_ALIGNMENT = 3,       /* bf16 path: pitch or pointer not 16-byte aligned */
  TP_ERR_UNSUPPORTED = 4,     /* combination not provided (see each call)       */
  TP_ERR_CUDA = 5,            /* a CUDA runtime call failed                      */
  TP_ERR_DEVICE_TIMEOUT = 6,  /* a bounded device-side wait gave up              */
  TP_ERR_WORKSPACE = 7        /* tp_mlp_block: workspace missing or too small    */
} tp_status;

typedef enum { TP_F32 = 0, TP_BF16 = 1 } tp_dtype;

typedef enum {
  TP_ACT_GELU_TANH = 0,  /* 0.5 h (1 + tanh(sqrt(2/pi) (h + 0.044715 h^3)))     */
  TP_ACT_SWIGLU = 1,     /* SiLU(X W_gate,i) * (X W_up,i), "Tensor Parallelism
                            Explained" 2.B; SiLU(h) = h / (1 + e^-h)            */
  TP_ACT_IDENTITY = 2,   /* h (exact-arithmetic tests)                          */
  TP_ACT_RELU = 3        /* max(0, h), the day-41 walkthrough's activation      */
} tp_act;

/* tp_mlp_block flags */
#define TP_FLAG_NONE 0
/* Accumulate all p shards of the row-parallel layer in one tensor-core
 * accumulator (split-K over shards) and write Z once, instead of writing p
 * partials and folding them.  Same result up to fp32 summation order (not
 * bit-identical to the fixed-order fold).  bf16 requires s % 64 == 0. */
#define TP_FLAG_SPLITK_FUSED 1
/* bf16: run both GEMM layers in one persistent launch (row-parallel tiles
 * start as soon as the hidden rows they read are complete) instead of one
 * launch per layer.  Same bits either way; the default per-layer launches
 * were faster on every measured shape (they use CTA-pair tiles). */
#define TP_FLAG_FUSED_LAUNCH 2
/* bf16: the row-parallel layer computes the p partials of each output tile
 * one after another in tensor memory and folds them in its epilogue in shard
 * order (then + b2), so the partials never reach HBM and no separate
 * reduction runs.  Bit-identical to the default (partials + fixed-order
 * fold).  Needs s % 64 == 0; combines with no other flag; the workspace
 * holds only the hidden shards (no p * T * d * 4 bytes of partials).  Slower
 * than the default on every measured shape: its 128-column single-CTA tiles
 * (the accumulator ring and the running sum share TMEM) read twice the
 * operand bytes per FLOP of the default row layer's CTA-pair tiles. */
#define TP_FLAG_ROW_FOLD 4

/*
 * Column-parallel linear + activation, all p shards in one launch.
 *   Y_i = act(X W1_i + b1_i),  W1_i = W1[:, i*s:(i+1)*s],  i = 0..p-1
 * ("Simulating column parallel linear"; "Column-parallel: split the weight
 * by output columns").  The activation is applied on each shard alone, which
 * the pairing allows because it is element-wise ("The MLP block").
 *
 *   X     [T][d]        dtype
 *   W1    [d][k]        dtype   (W_gate for SwiGLU)
 *   W_up  [d][k]        dtype   SwiGLU only (must be non-NULL), else ignored
 *   b1    [k]           dtype   nullable (no bias); with SwiGLU, b1 is added
 *                               to the gate pre-activation; bf16: 16-byte
 *                               aligned (read as 8-element vectors), else
 *                               TP_ERR_ALIGNMENT
 *   Y     [p][T][s]     dtype   output: shard i is a dense [T][s] matrix
 *   returns TP_ERR_INDIVISIBLE when k % p != 0.
 */
tp_status tp_column_linear(const void* X, const void* W1, const void* W_up, const void* b1,
                           void* Y, int64_t T, int64_t d, int64_t k, int p,
                           tp_dtype dtype, tp_act act, void* stream);

/*
 * Row-parallel linear: full-shape partials, one per shard.
 *   P_i = Y_i W2_i,  W2_i = W2[i*s:(i+1)*s, :]
 * ("Simulating row parallel linear"; "Row-parallel: split the weight by
 * input rows": every shard emits a [T, d] partial whose sum is the answer).
 *
 *   Y        [p][T][s]  dtype
 *   W2       [k][d]     dtype
 *   partials [p][T][d]  fp32 output
 */
tp_status tp_row_linear(const void* Y, const void* W2, float* partials,
                        int64_t T, int64_t k, int64_t d, int p,
                        tp_dtype dtype, void* stream);

/*
 * The sum that replaces the all-reduce, in a fixed order:
 *   Z = ((P_0 + P_1) + ...) + P_{p-1}  [+ b2]
 * every addition one fp32 round-to-nearest-even operation, shard index
 * ascending, the output bias added once after the sum (day-41 post:
 * sum(partial_sums) + bias).  Bit-reproducible: the same inputs always give
 * the same bits, on any grid.
 *
 *   partials [p][T][d]  fp32
 *   b2       [d]        fp32, nullable
 *   Z        [T][d]     fp32 output (must not alias partials)
 */
tp_status tp_reduce_partials(const float* partials, const float* b2, float* Z,
                             int64_t T, int64_t d, int p, void* stream);

/*
 * The all-reduce of the partials when the p shards live on p GPUs, one
 * process per GPU ("Simulating row parallel linear": the sum of partials is
 * the all-reduce over NVLink; "Building GPT from Scratch -- Part 9",
 * "Implementation Sketch": RowParallelLinear.forward all-reduces the
 * partial outputs, then adds the bias).  GPU r owns the token-row slab
 * [row0, row0 + rows) of Z.  This call folds that slab of the p partials in
 * shard order, exactly as tp_reduce_partials does (bit-identical on the same
 * values: P_0 first, one fp32 round-to-nearest-even add per shard, b2
 * last), and writes the folded slab to every destination in `outs` -- the
 * caller's own Z and, through peer mappings, the other GPUs' Z, so one pass
 * is both halves of the all-reduce (reduce-scatter and all-gather).
 *
 *   partials  HOST array of p device pointers, shard order; partials[j] is
 *             P_j, a [T][d] fp32 row-major buffer on this GPU or a peer
 *             mapping of another GPU's buffer (tp_ipc_import).  Only rows
 *             [row0, row0 + rows) are read.
 *   b2        [d] fp32 device pointer or NULL.
 *   outs      HOST array of n_out device pointers, each a [T][d] fp32
 *             buffer (local or peer-mapped); only the slab's rows are
 *             written, the same values to each.
 *   1 <= p <= TP_GATHER_MAX, 1 <= n_out <= TP_GATHER_MAX, 0 <= row0,
 *   0 <= rows, d >= 1.  Pointers 4-byte aligned (16-byte aligned with
 *   d % 4 == 0 takes 128-bit loads and stores).  No destination slab may
 *   overlap a partial's slab.
 * The kernel does not wait on other GPUs: order it after every GPU's P_j is
 * complete and before any GPU reads its Z (for instance a one-element
 * all-reduce on the stream before and after it).  Peer memory is read and
 * written with plain loads and stores only.  Errors: TP_ERR_INVALID_ARG for
 * bad counts, sizes, NULL or overlapping pointers, TP_ERR_ALIGNMENT,
 * TP_ERR_CUDA.  rows == 0 is a no-op.
 */
#define TP_GATHER_MAX 16
tp_status tp_reduce_partials_gather(const float* const* partials, int p, const float* b2,
                                    float* const* outs, int n_out, int64_t row0, int64_t rows,
                                    int64_t d, void* stream);

/*
 * Sharing device buffers between the processes of a p-GPU run (CUDA IPC),
 * so that each rank can map its peers' partials and outputs.
 *   tp_ipc_export   fills `handle` for the device buffer starting at `ptr`
 *                   (which must lie in a cudaMalloc allocation: PyTorch's
 *                   default allocator qualifies, its expandable segments do
 *                   not).  TP_ERR_INVALID_ARG if `ptr` is not device memory,
 *                   TP_ERR_CUDA if the allocation cannot be exported.
 *   tp_ipc_import   maps the buffer of a handle exported by ANOTHER process
 *                   and returns its address in this process (`*ptr`);
 *                   importing the same allocation again reuses the mapping.
 *   tp_ipc_release  drops one import; the mapping is closed with the last.
 * A handle is plain bytes and may be sent through any channel.
 */
typedef struct {
  unsigned char bytes[64];   /* cudaIpcMemHandle_t of the allocation        */
  uint64_t offset;           /* ptr - allocation base                        */
  uint64_t size;             /* allocation size in bytes                     */
} tp_ipc_handle;
tp_status tp_ipc_export(const void* ptr, tp_ipc_handle* handle);
tp_status tp_ipc_import(const tp_ipc_handle* handle, void** ptr);
tp_status tp_ipc_release(const tp_ipc_handle* handle);

/*
 * The whole block, Z = sum_i act(X W1_i + b1_i) W2_i  [+ b2]
 * ("Pairing them: the Megatron-LM MLP"; "The MLP block: column then row,
 * one all-reduce").  Computes exactly what tp_column_linear ->
 * tp_row_linear -> tp_reduce_partials compute (bit for bit), with the hidden
 * shards and the partials in the caller's workspace; the kernels are chained
 * with programmatic dependent launch.  Where the row layer runs on CTA-pair
 * tiles (bf16, b2 NULL or 16-byte aligned), it does the fold itself: shard
 * by shard, each tile adds its partial to the running sum that the previous
 * shard's tile left in Z, and the last shard adds b2 (same additions, same
 * order, same bits; no partials are written).  That layer is a cooperative
 * launch, so all its CTAs are resident together.  Z must not overlap the
 * workspace.  With TP_FLAG_SPLITK_FUSED the second layer accumulates over
 * all shards and writes Z directly (no partials).
 *
 *   workspace        device memory of at least
 *                    tp_mlp_block_workspace_size(...) bytes, 256-byte aligned;
 *                    contents on return: hidden shards [p][T][s] at offset 0,
 *                    then (default mode) room for the partials [p][T][d]
 *                    fp32 at the next 256-byte boundary (written only where
 *                    the row layer does not fold itself), then counters at
 *                    the end (reset on every call that uses them): one int32
 *                    per 128-row m-tile for TP_FLAG_FUSED_LAUNCH, or one per
 *                    256-row region of the row layer (column-major order,
 *                    each counted to 16 p, which orders the shards of the
 *                    fold; the area has room for ceil(T/128) * ceil(d/64) of
 *                    them).
 *   other arguments  as for the three calls above.
 */
tp_status tp_mlp_block(const void* X, const void* W1, const void* W_up, const void* b1,
                       const void* W2, const float* b2, float* Z,
                       void* workspace, size_t workspace_bytes,
                       int64_t T, int64_t d, int64_t k, int p,
                       tp_dtype dtype, tp_act act, int flags, void* stream);

/*
 * tp_mlp_block without a caller workspace, for callers that cannot allocate
 * device memory (a plugin inside a host framework that owns the whole device
 * memory pool, or a latency-critical loop that cannot afford cudaMalloc's
 * implicit device synchronisation).  The pages have no counterpart: this is
 * a deployment convenience, not part of the method.
 *
 * Same arguments and result as tp_mlp_block, minus the workspace: the hidden
 * shards and the partials live in one 16 MiB array of device memory inside
 * the library (held by every GPU that loads the library until the process
 * exits).  Nothing is allocated by the call.
 *   - Problems whose scratch, tp_mlp_block_workspace_size(...), exceeds
 *     16 MiB are rejected with TP_ERR_WORKSPACE.
 *   - All calls share that array.  Calls whose kernels overlap on one GPU
 *     (different streams or host threads) overwrite each other's scratch:
 *     issue them on one stream, one after another.
 *   - The first call on each device looks up the array's device address;
 *     make that first call before any stream capture begins.
 */
tp_status tp_mlp_block_noalloc(const void* X, const void* W1, const void* W_up, const void* b1,
                               const void* W2, const float* b2, float* Z,
                               int64_t T, int64_t d, int64_t k, int p,
                               tp_dtype dtype, tp_act act, int flags, void* stream);

/* Workspace bytes tp_mlp_block needs for these arguments (0 if invalid). */
size_t tp_mlp_block_workspace_size(int64_t T, int64_t d, int64_t k, int p,
                                   tp_dtype dtype, tp_act act, int flags);

/*
 * tp_mlp_block with the activations in HOST memory: X is read from, and Z
 * written to, host buffers; the weights and biases are device buffers (they
 * stay resident between calls).  The block is row-wise (row t of Z depends
 * only on row t of X: "Tensor parallel math", "The MLP block: column then
 * row, one all-reduce"), so the call cuts the T token rows into up to eight
 * chunks (multiples of 128 rows, at least 256 each) and pipelines them: the
 * copy of chunk c+1 into the device, the block on chunk c and the copy of
 * chunk c-1 back to the host overlap on the GPU's two copy engines and its
 * SMs.  Z has exactly the bits of copying X in, calling tp_mlp_block on all
 * rows and copying Z out.
 *
 *   X_host     [T][d] host memory (bf16 or fp32 per dtype).  Pinned
 *              (page-locked) memory lets the copies overlap the compute;
 *              pageable memory works but copies synchronously.
 *   Z_host     [T][d] fp32 host memory.
 *   workspace  device memory of at least tp_mlp_block_host_workspace_size()
 *              bytes, 256-byte aligned: device copies of X and Z, then the
 *              block's workspace for one chunk (for two when T spans more
 *              than one chunk: consecutive chunks run on two streams).
 *   others     as for tp_mlp_block.
 *
 * Stream semantics: everything is ordered on `stream`.  The call forks three
 * library-owned helper streams (one per copy direction and a second compute
 * stream, created on the first call on each device and kept for the
 * process) from `stream` with an event and joins them back before it
 * returns, so Z_host is complete once `stream` has reached the point of the
 * call (cudaStreamSynchronize).  Even chunks run on `stream`, odd chunks on
 * the second compute stream, so one chunk's kernels can fill the SMs the
 * other's last wave of tiles leaves idle; Z has the same bits either way.  The call can be
 * captured into a CUDA graph from `stream` when both host buffers are pinned
 * and the device has had one uncaptured call first.  Calls on one device
 * enqueue under a lock (the helper events are shared).
 *
 * Errors: argument errors return before anything is enqueued; a CUDA error
 * after the fork returns TP_ERR_CUDA with the helper streams still joined
 * into `stream`.
 */
tp_status tp_mlp_block_host(const void* X_host, const void* W1, const void* W_up,
                            const void* b1, const void* W2, const float* b2, float* Z_host,
                            void* workspace, size_t workspace_bytes,
                            int64_t T, int64_t d, int64_t k, int p,
                            tp_dtype dtype, tp_act act, int flags, void* stream);

/* Workspace bytes tp_mlp_block_host needs (0 if the arguments are invalid
 * or T == 0). */
size_t tp_mlp_block_host_workspace_size(int64_t T, int64_t d, int64_t k, int p,
                                        tp_dtype dtype, tp_act act, int flags);

/*
 * Attention of every shard's own heads (the local step of the
 * tensor-parallel attention block: each shard holds h/p query heads and
 * h_kv/p key/value heads and attends with no communication; day-41 post,
 * "Attention heads: naturally parallel"; "Tensor parallel math", "Attention:
 * parallel across heads").  Per head: O = softmax(Q K^T / sqrt(head_dim)) V,
 * query head j of a shard using key/value head j / (n_heads / n_kv_heads).
 *
 *   Q  [p][T][(n_heads/p) * head_dim]     bf16 (the column-parallel layout)
 *   K  [p][T][(n_kv_heads/p) * head_dim]  bf16
 *   V  [p][T][(n_kv_heads/p) * head_dim]  bf16
 *   O  [p][T][(n_heads/p) * head_dim]     bf16 output, the input of the
 *                                         row-parallel output projection
 *   causal  nonzero: query t attends to keys 0..t only
 * head_dim must be 128 (else TP_ERR_UNSUPPORTED); n_heads and n_kv_heads
 * must be divisible by p (else TP_ERR_INDIVISIBLE -- "Tensor Parallelism
 * Explained", section 4) and n_heads by n_kv_heads.
 */
tp_status tp_attention_heads(const void* Q, const void* K, const void* V, void* O, int64_t T,
                             int p, int n_heads, int n_kv_heads, int head_dim, int causal,
                             void* stream);

/*
 * The tensor-parallel attention block, Z = sum_i Attn_i(X) Wo_i [+ bo]:
 * column-parallel Q, K, V projections by heads (tp_column_linear, identity),
 * tp_attention_heads, row-parallel output projection (tp_row_linear) and the
 * fixed-order fold (tp_reduce_partials) -- one reduction per block ("Tensor
 * parallel math", "Attention: parallel across heads"; "Tensor Parallelism
 * Explained", section 2.A).  As in tp_mlp_block, the output projection
 * folds the shards itself where it runs on CTA-pair tiles (bo NULL or
 * 16-byte aligned); same bits.  Z must not overlap the workspace.
 *
 *   X [T][d]; Wq [d][n_heads*head_dim]; Wk, Wv [d][n_kv_heads*head_dim];
 *   Wo [n_heads*head_dim][d]  (all bf16, [in, out]);  bo [d] fp32 nullable;
 *   Z [T][d] fp32.
 *   workspace: tp_attn_block_workspace_size(...) bytes, 256-byte aligned
 *   (Q, K, V, O shards, then room for the fp32 partials, then the region
 *   counters).
 */
tp_status tp_attn_block(const void* X, const void* Wq, const void* Wk, const void* Wv,
                        const void* Wo, const float* bo, float* Z,
                        void* workspace, size_t workspace_bytes,
                        int64_t T, int64_t d, int n_heads, int n_kv_heads, int head_dim, int p,
                        int causal, void* stream);

/* Workspace bytes tp_attn_block needs (0 if the arguments are invalid). */
size_t tp_attn_block_workspace_size(int64_t T, int64_t d, int n_heads, int n_kv_heads,
                                    int head_dim, int p);

/*
 * LayerNorm of every row ("Building GPT from Scratch -- Part 9",
 * "Communication Pattern per Transformer Block": LayerNorm, replicated, no
 * communication): Y = (x - mean) / sqrt(var + eps) * gamma + beta with the
 * biased variance, computed in fp32, Y rounded to bf16 (the input of the
 * next block's column-parallel GEMMs).
 *
 *   X [T][d] fp32, gamma [d], beta [d] fp32, Y [T][d] bf16 (all 16-byte
 *   aligned); d % 4 == 0 and d <= 16384 (else TP_ERR_UNSUPPORTED); eps > 0.
 */
tp_status tp_layer_norm(const float* X, const float* gamma, const float* beta, void* Y, int64_t T,
                        int64_t d, float eps, void* stream);

/*
 * The reduction that ends a transformer sub-block, with the residual
 * connection folded in: Z = ((P_0 + ... + P_{p-1}) + bias) + residual, each
 * addition one fp32 round-to-nearest-even operation in that order
 * (bit-reproducible).  ("Building GPT from Scratch -- Part 9",
 * "Communication Pattern per Transformer Block": all-reduce after the
 * output projection / W2, then the element-wise residual add.)
 *
 *   partials [p][T][d] fp32, bias [d] fp32 or NULL, residual [T][d] fp32 or
 *   NULL (may equal Z; no other overlap), Z [T][d] fp32; 16-byte aligned;
 *   d % 4 == 0 and d <= 16384.
 */
tp_status tp_reduce_partials_residual(const float* partials, const float* bias,
                                      const float* residual, float* Z, int64_t T, int64_t d, int p,
                                      void* stream);

/* Weights of one transformer block (bf16 matrices [in, out], fp32 vectors;
 * bo, W_up, b1, b2 may be NULL; W_up is required for TP_ACT_SWIGLU, b1 is bf16
 * like the column-parallel layer's bias). */
typedef struct tp_block_params {
  const float* ln1_gamma;
  const float* ln1_beta;
  const void* Wq;   /* [d][n_heads * head_dim]    */
  const void* Wk;   /* [d][n_kv_heads * head_dim] */
  const void* Wv;   /* [d][n_kv_heads * head_dim] */
  const void* Wo;   /* [n_heads * head_dim][d]    */
  const float* bo;  /* [d]                        */
  const float* ln2_gamma;
  const float* ln2_beta;
  const void* W1;   /* [d][k] (W_gate for SwiGLU) */
  const void* W_up; /* [d][k]                     */
  const void* b1;   /* [k] bf16                   */
  const void* W2;   /* [k][d]                     */
  const float* b2;  /* [d]                        */
} tp_block_params;

/*
 * One pre-norm tensor-parallel transformer block on p simulated shards
 * ("Building GPT from Scratch -- Part 9", "Communication Pattern per
 * Transformer Block"; "Tensor parallel math", "Counting all-reduces": two
 * reductions per layer):
 *
 *   H   = X + tp_attn_block(LayerNorm(X; ln1))        (reduction #1 + residual)
 *   out = H + tp_mlp_block(LayerNorm(H; ln2))          (reduction #2 + residual)
 *
 * Each reduction adds, per element, the p partials in shard order, then the
 * bias, then the residual.  Reduction #2 runs in the MLP's row layer, which
 * adds b2 and then the residual after the last shard, where that layer runs
 * on CTA-pair tiles (b2 NULL or 16-byte aligned), as in tp_mlp_block; same
 * bits.  out must not overlap the workspace.
 *
 * X, out [T][d] fp32 (out may equal X); every GEMM reads bf16 and
 * accumulates fp32; head_dim 128; d % 8 == 0 and d <= 16384.  workspace:
 * tp_transformer_block_workspace_size(...) bytes, 256-byte aligned.
 */
tp_status tp_transformer_block(const float* X, const tp_block_params* params, float* out,
                               void* workspace, size_t workspace_bytes, int64_t T, int64_t d,
                               int n_heads, int n_kv_heads, int head_dim, int64_t k, int p,
                               int act, int causal, float eps, void* stream);

/* Workspace bytes tp_transformer_block needs (0 if the arguments are invalid). */
size_t tp_transformer_block_workspace_size(int64_t T, int64_t d, int n_heads, int n_kv_heads,
                                           int head_dim, int64_t k, int p);

/*
 * Backward pass of the MLP block through the f / g conjugate operators
 * ("Tensor parallel math", "The f and g conjugate operators": f is the
 * identity forward and an all-reduce backward, g the reverse; "Counting
 * all-reduces": one all-reduce per block in the backward pass).  g's
 * identity backward hands every shard the whole dZ; shard i then computes
 * locally
 *     dY_i = dZ W2_i^T,  dH_i = dY_i * act'(H_i)   (SwiGLU: dG_i, dU_i),
 *     dW2_i = Y_i^T dZ,  dW1_i = X^T dH_i,  db1_i = sum_t dH_i,
 * and f's all-reduce becomes the fixed-order fold of the p full-shape
 * partials dX = sum_i dH_i W1_i^T (+ dU_i Wup_i^T).  db2 = sum_t dZ.
 *
 *   X [T][d], W1 / W_up [d][k], W2 [k][d]   bf16, as in the forward call
 *   H     [p][T][k/p] bf16 pre-activation X W1_i + b1_i (SwiGLU: the gate),
 *         e.g. from tp_column_linear with TP_ACT_IDENTITY
 *   H_up  [p][T][k/p] bf16 up projection X Wup_i (SwiGLU only, else NULL)
 *   Y     [p][T][k/p] bf16 activation output (tp_column_linear's Y)
 *   dZ    [T][d] bf16 upstream gradient
 * Outputs (fp32, each may be NULL to skip it): dX [T][d]; dW1, dW_up
 * [d][k] (column blocks per shard); db1 [k]; dW2 [k][d] (row blocks);
 * db2 [d].  workspace: tp_mlp_block_backward_workspace_size(...) bytes,
 * 256-byte aligned.  k/p must be a multiple of 64 (else
 * TP_ERR_UNSUPPORTED).  Bias gradients are summed over tokens in a fixed
 * order (reproducible).
 */
tp_status tp_mlp_block_backward(const void* X, const void* W1, const void* W_up, const void* W2,
                                const void* H, const void* H_up, const void* Y, const void* dZ,
                                float* dX, float* dW1, float* dW_up, float* db1, float* dW2,
                                float* db2, void* workspace, size_t workspace_bytes, int64_t T,
                                int64_t d, int64_t k, int p, int act, void* stream);

/* Workspace bytes tp_mlp_block_backward needs (0 if the arguments are invalid). */
size_t tp_mlp_block_backward_workspace_size(int64_t T, int64_t d, int64_t k, int p, int act);

/*
 * The same backward pass from the forward inputs alone (activation
 * recomputation): the column-parallel layer is run again to rebuild the
 * pre-activations H (and the up projection) and the activations Y in the
 * workspace, then tp_mlp_block_backward runs on them.  Same results as
 * calling tp_column_linear (identity, then act) and tp_mlp_block_backward.
 *   b1 [k] bf16 or NULL (the forward's bias); other arguments as in
 *   tp_mlp_block_backward.  workspace:
 *   tp_mlp_block_backward_recompute_workspace_size(...) bytes, 256-aligned.
 */
tp_status tp_mlp_block_backward_recompute(const void* X, const void* W1, const void* W_up,
                                          const void* b1, const void* W2, const void* dZ,
                                          float* dX, float* dW1, float* dW_up, float* db1,
                                          float* dW2, float* db2, void* workspace,
                                          size_t workspace_bytes, int64_t T, int64_t d, int64_t k,
                                          int p, int act, void* stream);

size_t tp_mlp_block_backward_recompute_workspace_size(int64_t T, int64_t d, int64_t k, int p,
                                                      int act);

/* Synchronise `stream`, then report (and clear) the device status word of
 * the current device: TP_ERR_DEVICE_TIMEOUT if a bounded wait ran out since
 * the last call, TP_ERR_CUDA if the stream reported an error, else TP_OK. */
tp_status tp_sync_status(void* stream);

/* Limit for every bounded device-side wait, in nanoseconds (default 2e9).
 * Applies to launches made after the call. 0 restores the default. */
void tp_set_wait_timeout_ns(uint64_t ns);

/* Fault injection for tests of the bounded waits: when `stage_index` >= 0,
 * the next tensor-core launch's producer skips the load of that pipeline
 * slot (counted from 0 in issue order), so its consumer's wait must run
 * out.  In a launch of CTA-pair tiles only the first pair skips it (the
 * other pairs' waits on that pair's tiles then run out too); in other
 * launches every CTA does.  -1 (default) disables it.  Applies to the next
 * launch only. */
void tp_debug_drop_load(int64_t stage_index);
/* The same, for the tensor-core launch that follows `launches_to_skip`
 * others (0: the next one), e.g. 1 for the row layer of a tp_mlp_block
 * call. */
void tp_debug_drop_load_after(int64_t stage_index, int launches_to_skip);

/* Test hook (not part of the method): y[i] = the attention softmax's
 * fast 2^x for i < n, x and y fp32 device arrays of n elements (4-byte
 * aligned, caller-owned).  The kernel computes part of the probabilities
 * 2^(s - m) on the FMA pipe: round x to the nearest integer n0, a fitted
 * degree-4 polynomial for 2^(x - n0) on [-1/2, 1/2], n0 added to the
 * exponent; x is first clamped to >= -126.  On [-126, 0] its relative error
 * against 2^x is at most 2.7e-6.  Asynchronous on `stream`; TP_ERR_INVALID_ARG
 * for n < 0 or NULL arrays (n == 0 is a no-op), TP_ERR_ALIGNMENT, and
 * TP_ERR_UNSUPPORTED off sm_100. */
tp_status tp_debug_exp2_poly(const float* x, float* y, int64_t n, void* stream);

/* Human-readable name of a status code. */
const char* tp_status_string(int status);

/* Detail of the last argument or CUDA error seen by this thread ("" if none). */
const char* tp_last_error_detail(void);

/* Number of GPU kernels this library has launched in this process. */
uint64_t tp_kernel_launch_count(void);

/* ABI version of this header (bumped on any signature change or added call;
 * 2: the p-GPU fold and IPC calls, the exp2 test hook, and a host-buffer
 * workspace sized for two chunks). */
int tp_abi_version(void);

#define TP_ABI_VERSION 2

#ifdef __cplusplus
}
#endif

#endif /* TP_MLP_H */
