"""Python binding of libtpmlp, the B200 (sm_100a) Megatron tensor-parallel
MLP block on p simulated shards.

Argument marshalling only: every call below forwards to the C ABI of the
same name (``include/tp_mlp.h``); all arithmetic runs in the library's CUDA
kernels.  Arguments that are device buffers accept a ``torch.Tensor`` (its
``data_ptr()`` is passed), a raw integer address, or ``None`` (NULL).
``stream=None`` means torch's current CUDA stream.

Importing this package fails loudly when the shared library has not been
built (``python megatron_tensor_sharded_b200/build.py``): there is no CPU or
PyTorch fallback.

Example -- the MLP block on p = 4 simulated shards, bf16 in, fp32 out::

    import torch, megatron_tensor_sharded_b200 as tp
    T, d, k, p = 4096, 4096, 16384, 4
    X = torch.randn(T, d, device="cuda").bfloat16()
    W1 = (0.02 * torch.randn(d, k, device="cuda")).bfloat16()    # [in, out]
    W2 = (0.02 * torch.randn(k, d, device="cuda")).bfloat16()
    Z = torch.empty(T, d, device="cuda")
    n = tp.tp_mlp_block_workspace_size(T, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    tp.tp_mlp_block(X, W1, None, None, W2, None, Z, ws, n, T, d, k, p,
                    tp.TP_BF16, tp.TP_ACT_GELU_TANH)
    tp.tp_sync_status()          # raises TPError if a device wait timed out

The same pattern serves tp_attn_block, tp_transformer_block (weights in a
BlockParams built by ``block_params(**tensors)``) and tp_mlp_block_backward.
"""

from __future__ import annotations

import ctypes
import os

__all__ = [
    "TPError", "TP_F32", "TP_BF16", "TP_ACT_GELU_TANH", "TP_ACT_SWIGLU", "TP_ACT_IDENTITY",
    "TP_ACT_RELU", "TP_FLAG_NONE", "TP_FLAG_SPLITK_FUSED", "TP_FLAG_FUSED_LAUNCH",
    "TP_FLAG_ROW_FOLD", "STATUS", "ACT", "DTYPE", "LIB_PATH", "BlockParams", "block_params",
    # the MLP block and its steps
    "tp_column_linear", "tp_row_linear", "tp_reduce_partials", "tp_mlp_block",
    "tp_mlp_block_workspace_size", "tp_mlp_block_noalloc", "tp_mlp_block_host",
    "tp_mlp_block_host_workspace_size",
    # attention, transformer block, backward
    "tp_attention_heads", "tp_attn_block", "tp_attn_block_workspace_size",
    "tp_layer_norm", "tp_reduce_partials_residual", "tp_transformer_block",
    "tp_transformer_block_workspace_size", "tp_mlp_block_backward",
    "tp_mlp_block_backward_workspace_size", "tp_mlp_block_backward_recompute",
    "tp_mlp_block_backward_recompute_workspace_size",
    # the all-reduce of partials held on p GPUs
    "TP_GATHER_MAX", "IpcHandle", "tp_reduce_partials_gather", "tp_ipc_export", "tp_ipc_import",
    "tp_ipc_release",
    # status, timeouts, introspection
    "tp_sync_status", "tp_set_wait_timeout_ns", "tp_debug_drop_load", "tp_debug_exp2_poly",
    "tp_status_string",
    "tp_last_error_detail", "tp_kernel_launch_count", "tp_abi_version",
]

LIB_PATH = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libtpmlp.so")

TP_F32, TP_BF16 = 0, 1
TP_ACT_GELU_TANH, TP_ACT_SWIGLU, TP_ACT_IDENTITY, TP_ACT_RELU = 0, 1, 2, 3
TP_FLAG_NONE, TP_FLAG_SPLITK_FUSED, TP_FLAG_FUSED_LAUNCH, TP_FLAG_ROW_FOLD = 0, 1, 2, 4
DTYPE = {"f32": TP_F32, "bf16": TP_BF16}
ACT = {"gelu_tanh": TP_ACT_GELU_TANH, "swiglu": TP_ACT_SWIGLU, "identity": TP_ACT_IDENTITY,
       "relu": TP_ACT_RELU}
STATUS = {0: "TP_OK", 1: "TP_ERR_INVALID_ARG", 2: "TP_ERR_INDIVISIBLE", 3: "TP_ERR_ALIGNMENT",
          4: "TP_ERR_UNSUPPORTED", 5: "TP_ERR_CUDA", 6: "TP_ERR_DEVICE_TIMEOUT",
          7: "TP_ERR_WORKSPACE"}


class TPError(RuntimeError):
    def __init__(self, status: int, detail: str):
        self.status = status
        self.name = STATUS.get(status, str(status))
        super().__init__(f"{self.name}: {detail}")


TP_GATHER_MAX = 16


class IpcHandle(ctypes.Structure):
    """tp_ipc_handle: an exported device buffer (plain bytes, any channel)."""
    _fields_ = [("bytes", ctypes.c_ubyte * 64), ("offset", ctypes.c_uint64),
                ("size", ctypes.c_uint64)]

    def to_bytes(self) -> bytes:
        return ctypes.string_at(ctypes.addressof(self), ctypes.sizeof(self))

    @classmethod
    def from_bytes(cls, b: bytes) -> "IpcHandle":
        h = cls()
        ctypes.memmove(ctypes.addressof(h), b, ctypes.sizeof(h))
        return h


class BlockParams(ctypes.Structure):
    """tp_block_params: device pointers of one transformer block's weights."""
    _fields_ = [(name, ctypes.c_void_p) for name in (
        "ln1_gamma", "ln1_beta", "Wq", "Wk", "Wv", "Wo", "bo", "ln2_gamma", "ln2_beta", "W1",
        "W_up", "b1", "W2", "b2")]


def _load() -> ctypes.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is not built; run "
                          "`python megatron_tensor_sharded_b200/build.py` (nvcc, sm_100a)")
    lib = ctypes.CDLL(LIB_PATH)
    vp, i64, i32, u64, sz = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int, ctypes.c_uint64, ctypes.c_size_t
    lib.tp_column_linear.argtypes = [vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32, vp]
    lib.tp_row_linear.argtypes = [vp, vp, vp, i64, i64, i64, i32, i32, vp]
    lib.tp_reduce_partials.argtypes = [vp, vp, vp, i64, i64, i32, vp]
    lib.tp_mlp_block.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, i64, i64, i64, i32, i32, i32,
                                 i32, vp]
    lib.tp_mlp_block_noalloc.argtypes = [vp, vp, vp, vp, vp, vp, vp, i64, i64, i64, i32, i32, i32,
                                         i32, vp]
    lib.tp_mlp_block_host.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, i64, i64, i64, i32, i32,
                                      i32, i32, vp]
    lib.tp_mlp_block_host_workspace_size.argtypes = [i64, i64, i64, i32, i32, i32, i32]
    lib.tp_mlp_block_host_workspace_size.restype = sz
    lib.tp_attention_heads.argtypes = [vp, vp, vp, vp, i64, i32, i32, i32, i32, i32, vp]
    lib.tp_attn_block.argtypes = [vp, vp, vp, vp, vp, vp, vp, vp, sz, i64, i64, i32, i32, i32, i32,
                                  i32, vp]
    lib.tp_attn_block_workspace_size.argtypes = [i64, i64, i32, i32, i32, i32]
    lib.tp_attn_block_workspace_size.restype = sz
    lib.tp_layer_norm.argtypes = [vp, vp, vp, vp, i64, i64, ctypes.c_float, vp]
    lib.tp_reduce_partials_residual.argtypes = [vp, vp, vp, vp, i64, i64, i32, vp]
    lib.tp_transformer_block.argtypes = [vp, ctypes.POINTER(BlockParams), vp, vp, sz, i64, i64,
                                         i32, i32, i32, i64, i32, i32, i32, ctypes.c_float, vp]
    lib.tp_transformer_block_workspace_size.argtypes = [i64, i64, i32, i32, i32, i64, i32]
    lib.tp_transformer_block_workspace_size.restype = sz
    lib.tp_mlp_block_backward.argtypes = [vp] * 15 + [sz, i64, i64, i64, i32, i32, vp]
    lib.tp_mlp_block_backward_recompute.argtypes = [vp] * 13 + [sz, i64, i64, i64, i32, i32, vp]
    lib.tp_mlp_block_backward_recompute_workspace_size.argtypes = [i64, i64, i64, i32, i32]
    lib.tp_mlp_block_backward_recompute_workspace_size.restype = sz
    lib.tp_mlp_block_backward_workspace_size.argtypes = [i64, i64, i64, i32, i32]
    lib.tp_mlp_block_backward_workspace_size.restype = sz
    lib.tp_mlp_block_workspace_size.argtypes = [i64, i64, i64, i32, i32, i32, i32]
    lib.tp_mlp_block_workspace_size.restype = sz
    lib.tp_sync_status.argtypes = [vp]
    lib.tp_set_wait_timeout_ns.argtypes = [u64]
    lib.tp_set_wait_timeout_ns.restype = None
    lib.tp_debug_drop_load.argtypes = [i64]
    lib.tp_debug_drop_load.restype = None
    lib.tp_debug_drop_load_after.argtypes = [i64, ctypes.c_int]
    lib.tp_debug_drop_load_after.restype = None
    lib.tp_debug_exp2_poly.argtypes = [vp, vp, i64, vp]
    lib.tp_reduce_partials_gather.argtypes = [ctypes.POINTER(vp), i32, vp, ctypes.POINTER(vp), i32,
                                              i64, i64, i64, vp]
    lib.tp_ipc_export.argtypes = [vp, ctypes.POINTER(IpcHandle)]
    lib.tp_ipc_import.argtypes = [ctypes.POINTER(IpcHandle), ctypes.POINTER(vp)]
    lib.tp_ipc_release.argtypes = [ctypes.POINTER(IpcHandle)]
    lib.tp_status_string.argtypes = [i32]
    lib.tp_status_string.restype = ctypes.c_char_p
    lib.tp_last_error_detail.argtypes = []
    lib.tp_last_error_detail.restype = ctypes.c_char_p
    lib.tp_kernel_launch_count.argtypes = []
    lib.tp_kernel_launch_count.restype = u64
    lib.tp_abi_version.argtypes = []
    for f in ("tp_column_linear", "tp_row_linear", "tp_reduce_partials", "tp_mlp_block",
              "tp_mlp_block_noalloc", "tp_mlp_block_host", "tp_attention_heads", "tp_attn_block", "tp_layer_norm",
              "tp_reduce_partials_residual", "tp_transformer_block", "tp_mlp_block_backward",
              "tp_mlp_block_backward_recompute", "tp_sync_status", "tp_abi_version",
              "tp_debug_exp2_poly", "tp_reduce_partials_gather", "tp_ipc_export",
              "tp_ipc_import", "tp_ipc_release"):
        getattr(lib, f).restype = i32
    return lib


_lib = _load()


def _ptr(x):
    if x is None:
        return None
    if isinstance(x, int):
        return x
    return x.data_ptr()


def _stream(stream):
    if stream is None:
        import torch
        if torch.cuda.is_available() and torch.cuda.is_initialized():
            return torch.cuda.current_stream().cuda_stream
        return None
    if isinstance(stream, int):
        return stream
    return stream.cuda_stream


def _check(status: int, check: bool) -> int:
    if check and status != 0:
        raise TPError(status, tp_last_error_detail())
    return status


def tp_column_linear(X, W1, W_up, b1, Y, T, d, k, p, dtype, act, stream=None, check=True):
    """Y_i = act(X W1_i + b1_i) for all p shards; Y is [p][T][k/p]."""
    return _check(_lib.tp_column_linear(_ptr(X), _ptr(W1), _ptr(W_up), _ptr(b1), _ptr(Y), T, d, k,
                                        p, dtype, act, _stream(stream)), check)


def tp_row_linear(Y, W2, partials, T, k, d, p, dtype, stream=None, check=True):
    """P_i = Y_i W2_i, fp32 partials [p][T][d]."""
    return _check(_lib.tp_row_linear(_ptr(Y), _ptr(W2), _ptr(partials), T, k, d, p, dtype,
                                     _stream(stream)), check)


def tp_reduce_partials(partials, b2, Z, T, d, p, stream=None, check=True):
    """Z = ((P_0 + P_1) + ...) + P_{p-1} [+ b2], fixed order, fp32."""
    return _check(_lib.tp_reduce_partials(_ptr(partials), _ptr(b2), _ptr(Z), T, d, p,
                                          _stream(stream)), check)


def tp_mlp_block(X, W1, W_up, b1, W2, b2, Z, workspace, workspace_bytes, T, d, k, p, dtype, act,
                 flags=TP_FLAG_NONE, stream=None, check=True):
    """The whole block, Z = sum_i act(X W1_i + b1_i) W2_i [+ b2]."""
    return _check(_lib.tp_mlp_block(_ptr(X), _ptr(W1), _ptr(W_up), _ptr(b1), _ptr(W2), _ptr(b2),
                                    _ptr(Z), _ptr(workspace), workspace_bytes, T, d, k, p, dtype,
                                    act, flags, _stream(stream)), check)


def tp_mlp_block_host(X_host, W1, W_up, b1, W2, b2, Z_host, workspace, workspace_bytes, T, d, k,
                      p, dtype, act, flags=TP_FLAG_NONE, stream=None, check=True):
    """The whole block with X and Z in host memory (pinned for overlap): the
    token rows are pipelined in chunks through copy-in, the block and
    copy-out on the GPU's copy engines; Z_host is complete once `stream`
    reaches the call."""
    return _check(_lib.tp_mlp_block_host(_ptr(X_host), _ptr(W1), _ptr(W_up), _ptr(b1), _ptr(W2),
                                         _ptr(b2), _ptr(Z_host), _ptr(workspace), workspace_bytes,
                                         T, d, k, p, dtype, act, flags, _stream(stream)), check)


def tp_mlp_block_host_workspace_size(T, d, k, p, dtype, act, flags=TP_FLAG_NONE) -> int:
    return int(_lib.tp_mlp_block_host_workspace_size(T, d, k, p, dtype, act, flags))


def tp_mlp_block_noalloc(X, W1, W_up, b1, W2, b2, Z, T, d, k, p, dtype, act,
                         flags=TP_FLAG_NONE, stream=None, check=True):
    """The whole block without a caller workspace (for callers that cannot
    allocate device memory): scratch comes from a fixed 16 MiB array inside
    the library, shared by all calls, so calls must not overlap on the GPU."""
    return _check(_lib.tp_mlp_block_noalloc(_ptr(X), _ptr(W1), _ptr(W_up), _ptr(b1), _ptr(W2),
                                            _ptr(b2), _ptr(Z), T, d, k, p, dtype, act, flags,
                                            _stream(stream)), check)


def tp_attention_heads(Q, K, V, O, T, p, n_heads, n_kv_heads, head_dim, causal=False, stream=None,
                       check=True):
    """Attention of every shard's own heads: O = softmax(Q K^T / sqrt(dh)) V."""
    return _check(_lib.tp_attention_heads(_ptr(Q), _ptr(K), _ptr(V), _ptr(O), T, p, n_heads,
                                          n_kv_heads, head_dim, int(bool(causal)),
                                          _stream(stream)), check)


def tp_attn_block(X, Wq, Wk, Wv, Wo, bo, Z, workspace, workspace_bytes, T, d, n_heads, n_kv_heads,
                  head_dim, p, causal=False, stream=None, check=True):
    """The tensor-parallel attention block, Z = sum_i Attn_i(X) Wo_i [+ bo]."""
    return _check(_lib.tp_attn_block(_ptr(X), _ptr(Wq), _ptr(Wk), _ptr(Wv), _ptr(Wo), _ptr(bo),
                                     _ptr(Z), _ptr(workspace), workspace_bytes, T, d, n_heads,
                                     n_kv_heads, head_dim, p, int(bool(causal)),
                                     _stream(stream)), check)


def tp_attn_block_workspace_size(T, d, n_heads, n_kv_heads, head_dim, p) -> int:
    return int(_lib.tp_attn_block_workspace_size(T, d, n_heads, n_kv_heads, head_dim, p))


def tp_layer_norm(X, gamma, beta, Y, T, d, eps=1e-5, stream=None, check=True):
    """Y = LayerNorm(X) * gamma + beta per row, fp32 statistics, bf16 Y."""
    return _check(_lib.tp_layer_norm(_ptr(X), _ptr(gamma), _ptr(beta), _ptr(Y), T, d, eps,
                                     _stream(stream)), check)


def tp_reduce_partials_residual(partials, bias, residual, Z, T, d, p, stream=None, check=True):
    """Z = ((P_0 + ... + P_{p-1}) + bias) + residual, fixed order, fp32."""
    return _check(_lib.tp_reduce_partials_residual(_ptr(partials), _ptr(bias), _ptr(residual),
                                                   _ptr(Z), T, d, p, _stream(stream)), check)


def block_params(**tensors) -> BlockParams:
    """BlockParams from device tensors (or None) named like its fields."""
    prm = BlockParams()
    for name, _ in BlockParams._fields_:
        setattr(prm, name, _ptr(tensors.get(name)))
    return prm


def tp_transformer_block(X, params: BlockParams, out, workspace, workspace_bytes, T, d, n_heads,
                         n_kv_heads, head_dim, k, p, act, causal=True, eps=1e-5, stream=None,
                         check=True):
    """H = X + attn(LN1(X)); out = H + mlp(LN2(H)), both reductions fixed-order."""
    return _check(_lib.tp_transformer_block(_ptr(X), ctypes.byref(params), _ptr(out),
                                            _ptr(workspace), workspace_bytes, T, d, n_heads,
                                            n_kv_heads, head_dim, k, p, act, int(bool(causal)),
                                            eps, _stream(stream)), check)


def tp_transformer_block_workspace_size(T, d, n_heads, n_kv_heads, head_dim, k, p) -> int:
    return int(_lib.tp_transformer_block_workspace_size(T, d, n_heads, n_kv_heads, head_dim, k, p))


def tp_mlp_block_backward(X, W1, W_up, W2, H, H_up, Y, dZ, dX, dW1, dW_up, db1, dW2, db2,
                          workspace, workspace_bytes, T, d, k, p, act, stream=None, check=True):
    """Gradients of the MLP block: dX (fold of p partials), dW1, dW_up, db1,
    dW2, db2 (any output may be None)."""
    return _check(_lib.tp_mlp_block_backward(
        _ptr(X), _ptr(W1), _ptr(W_up), _ptr(W2), _ptr(H), _ptr(H_up), _ptr(Y), _ptr(dZ), _ptr(dX),
        _ptr(dW1), _ptr(dW_up), _ptr(db1), _ptr(dW2), _ptr(db2), _ptr(workspace), workspace_bytes,
        T, d, k, p, act, _stream(stream)), check)


def tp_mlp_block_backward_recompute(X, W1, W_up, b1, W2, dZ, dX, dW1, dW_up, db1, dW2, db2,
                                    workspace, workspace_bytes, T, d, k, p, act, stream=None,
                                    check=True):
    """The backward pass from the forward inputs (H, H_up, Y recomputed)."""
    return _check(_lib.tp_mlp_block_backward_recompute(
        _ptr(X), _ptr(W1), _ptr(W_up), _ptr(b1), _ptr(W2), _ptr(dZ), _ptr(dX), _ptr(dW1),
        _ptr(dW_up), _ptr(db1), _ptr(dW2), _ptr(db2), _ptr(workspace), workspace_bytes, T, d, k, p,
        act, _stream(stream)), check)


def tp_mlp_block_backward_recompute_workspace_size(T, d, k, p, act) -> int:
    return int(_lib.tp_mlp_block_backward_recompute_workspace_size(T, d, k, p, act))


def tp_mlp_block_backward_workspace_size(T, d, k, p, act) -> int:
    return int(_lib.tp_mlp_block_backward_workspace_size(T, d, k, p, act))


def tp_mlp_block_workspace_size(T, d, k, p, dtype, act, flags=TP_FLAG_NONE) -> int:
    return int(_lib.tp_mlp_block_workspace_size(T, d, k, p, dtype, act, flags))


def tp_sync_status(stream=None, check=True):
    return _check(_lib.tp_sync_status(_stream(stream)), check)


def tp_set_wait_timeout_ns(ns: int) -> None:
    _lib.tp_set_wait_timeout_ns(ns)


def tp_debug_drop_load(stage_index: int, launches_to_skip: int = 0) -> None:
    """Test hook: the tensor-core launch after `launches_to_skip` others
    skips the load of pipeline slot `stage_index` (-1 disarms)."""
    _lib.tp_debug_drop_load_after(stage_index, launches_to_skip)


def tp_reduce_partials_gather(partials, b2, outs, row0, rows, d, stream=None, check=True):
    """Fold rows [row0, row0 + rows) of the p partials (a sequence of device
    buffers or addresses, shard order, local or peer-mapped) in shard order
    (+ b2) and write the slab to every buffer in `outs`."""
    vp = ctypes.c_void_p
    parts = (vp * len(partials))(*[_ptr(x) for x in partials])
    dst = (vp * len(outs))(*[_ptr(x) for x in outs])
    return _check(_lib.tp_reduce_partials_gather(parts, len(partials), _ptr(b2), dst, len(outs),
                                                 row0, rows, d, _stream(stream)), check)


def tp_ipc_export(buf) -> IpcHandle:
    """Handle of the device buffer `buf` (tensor or address) for another process."""
    h = IpcHandle()
    _check(_lib.tp_ipc_export(_ptr(buf), ctypes.byref(h)), True)
    return h


def tp_ipc_import(handle: IpcHandle) -> int:
    """Maps a buffer exported by another process; returns its address here."""
    out = ctypes.c_void_p()
    _check(_lib.tp_ipc_import(ctypes.byref(handle), ctypes.byref(out)), True)
    return int(out.value)


def tp_ipc_release(handle: IpcHandle) -> None:
    _check(_lib.tp_ipc_release(ctypes.byref(handle)), True)


def tp_debug_exp2_poly(x, y, n, stream=None, check=True):
    """Test hook: y[i] = the attention softmax's fast 2^x for i < n (fp32)."""
    return _check(_lib.tp_debug_exp2_poly(_ptr(x), _ptr(y), n, _stream(stream)), check)


def tp_status_string(status: int) -> str:
    return _lib.tp_status_string(status).decode()


def tp_last_error_detail() -> str:
    return _lib.tp_last_error_detail().decode()


def tp_kernel_launch_count() -> int:
    return int(_lib.tp_kernel_launch_count())


def tp_abi_version() -> int:
    return int(_lib.tp_abi_version())
