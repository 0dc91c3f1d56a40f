"""Host-side checks of the C ABI that need no GPU: the library loads, exports
every function the header declares, and rejects bad arguments with the
documented status codes before touching the device."""

import ctypes
import os
import re

import pytest

import megatron_tensor_sharded_b200 as tp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "tp_mlp.h")

FAKE = 0x10000      # never dereferenced: every case below fails validation first
FAKE2 = 0x20000


def declared_functions():
    src = open(HEADER).read()
    src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
    return sorted(set(re.findall(r"\b(tp_[a-z_0-9]+)\s*\(", src)))


def test_header_declares_the_boundary_calls():
    names = declared_functions()
    for required in ("tp_column_linear", "tp_row_linear", "tp_reduce_partials", "tp_mlp_block"):
        assert required in names


def test_library_exports_every_declared_symbol():
    lib = ctypes.CDLL(tp.LIB_PATH)
    missing = [n for n in declared_functions() if not hasattr(lib, n)]
    assert not missing, missing


def test_abi_version_matches_header():
    m = re.search(r"#define TP_ABI_VERSION (\d+)", open(HEADER).read())
    assert tp.tp_abi_version() == int(m.group(1))


def test_status_strings():
    for code, name in tp.STATUS.items():
        assert tp.tp_status_string(code).startswith(name)
    assert "unknown" in tp.tp_status_string(99)


def _col(**kw):
    a = dict(X=FAKE, W1=FAKE, W_up=None, b1=None, Y=FAKE2, T=4, d=64, k=256, p=4,
             dtype=tp.TP_BF16, act=tp.TP_ACT_GELU_TANH)
    a.update(kw)
    return tp.tp_column_linear(a["X"], a["W1"], a["W_up"], a["b1"], a["Y"], a["T"], a["d"], a["k"],
                               a["p"], a["dtype"], a["act"], stream=0, check=False)


def test_column_validation():
    assert _col(p=0) == 1
    assert _col(p=-3) == 1
    assert _col(k=10, p=4) == 2                          # indivisible (k % p != 0)
    assert _col(k=64, p=5) == 2
    assert _col(d=12) == 3                               # bf16 pitch not 16-byte multiple
    assert _col(k=4 * 12, p=4) == 3                      # s = 12
    assert _col(X=FAKE + 2) == 3                         # misaligned pointer
    assert _col(X=None) == 1
    assert _col(act=tp.TP_ACT_SWIGLU, W_up=None) == 1    # SwiGLU needs W_up
    assert _col(act=7) == 1
    assert _col(dtype=5) == 1
    assert _col(d=0) == 1
    assert _col(T=-1) == 1
    assert _col(dtype=tp.TP_F32, X=FAKE + 2) == 3        # fp32 needs 4-byte alignment


def test_empty_input_is_a_no_op():
    n0 = tp.tp_kernel_launch_count()
    assert _col(T=0, X=None, Y=None) == 0
    assert tp.tp_row_linear(None, None, None, 0, 256, 64, 4, tp.TP_BF16, stream=0, check=False) == 0
    assert tp.tp_reduce_partials(None, None, None, 0, 64, 4, stream=0, check=False) == 0
    assert tp.tp_mlp_block(None, None, None, None, None, None, None, None, 0, 0, 64, 256, 4,
                           tp.TP_BF16, tp.TP_ACT_GELU_TANH, stream=0, check=False) == 0
    assert tp.tp_kernel_launch_count() == n0


def test_row_and_reduce_validation():
    assert tp.tp_row_linear(FAKE, FAKE, FAKE2, 4, 250, 64, 4, tp.TP_BF16, stream=0, check=False) == 2
    assert tp.tp_row_linear(FAKE, FAKE, None, 4, 256, 64, 4, tp.TP_BF16, stream=0, check=False) == 1
    assert tp.tp_row_linear(FAKE, FAKE, FAKE2 + 4, 4, 256, 64, 4, tp.TP_BF16, stream=0, check=False) == 3
    assert tp.tp_reduce_partials(FAKE, None, FAKE2, 4, 64, 0, stream=0, check=False) == 1
    assert tp.tp_reduce_partials(None, None, FAKE2, 4, 64, 2, stream=0, check=False) == 1
    # Z inside the partials range
    assert tp.tp_reduce_partials(FAKE, None, FAKE + 64, 4, 64, 2, stream=0, check=False) == 1
    assert tp.tp_reduce_partials(FAKE + 2, None, FAKE2, 4, 64, 2, stream=0, check=False) == 3


def test_workspace_size_formula():
    # bf16: hidden shards T*k*2 bytes, then p*T*d*4 bytes of partials, each
    # rounded up to 256 bytes, then the counters: one int per 128-row m-tile
    # (single-launch block) or per 128-row x 64-column region at most (fold
    # beside the row layer), whichever is larger
    def r256(n):
        return -(-n // 256) * 256

    def counters(T, d):
        return max(r256(4 * (-(-T // 128))), r256(4 * (-(-T // 128)) * (-(-d // 64))))

    T, d, k, p = 1000, 768, 3072, 2
    ys = r256(T * k * 2)
    ps = r256(p * T * d * 4)
    assert tp.tp_mlp_block_workspace_size(T, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH) == \
        ys + ps + counters(T, d)
    assert tp.tp_mlp_block_workspace_size(T, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH,
                                          tp.TP_FLAG_SPLITK_FUSED) == ys + counters(T, d)
    assert tp.tp_mlp_block_workspace_size(4, 512, 2048, 4, tp.TP_F32, tp.TP_ACT_GELU_TANH) == \
        r256(4 * 2048 * 4) + r256(4 * 4 * 512 * 4) + counters(4, 512)
    assert tp.tp_mlp_block_workspace_size(4, 512, 2047, 4, tp.TP_F32, tp.TP_ACT_GELU_TANH) == 0
    # Llama-shaped prefill: room for 32 x 128 regions
    T, d, k, p = 4096, 8192, 28672, 8
    assert tp.tp_mlp_block_workspace_size(T, d, k, p, tp.TP_BF16, tp.TP_ACT_SWIGLU) == \
        r256(T * k * 2) + r256(p * T * d * 4) + 16384


def test_block_validation():
    def blk(**kw):
        a = dict(X=FAKE, W1=FAKE, W_up=None, b1=None, W2=FAKE, b2=None, Z=FAKE2, ws=0x40000,
                 wsb=1 << 30, T=4, d=64, k=256, p=4, dtype=tp.TP_BF16, act=tp.TP_ACT_GELU_TANH,
                 flags=0)
        a.update(kw)
        return tp.tp_mlp_block(a["X"], a["W1"], a["W_up"], a["b1"], a["W2"], a["b2"], a["Z"],
                               a["ws"], a["wsb"], a["T"], a["d"], a["k"], a["p"], a["dtype"],
                               a["act"], a["flags"], stream=0, check=False)
    assert blk(wsb=16) == 7
    assert blk(ws=None) == 7
    assert blk(ws=0x40000 + 16) == 3
    assert blk(k=255) == 2
    assert blk(flags=8) == 1
    assert blk(flags=16) == 1
    assert blk(flags=tp.TP_FLAG_ROW_FOLD | tp.TP_FLAG_SPLITK_FUSED) == 1
    assert blk(k=4 * 72, flags=tp.TP_FLAG_ROW_FOLD) == 4      # s = 72, not a multiple of 64
    assert blk(k=4 * 72, flags=tp.TP_FLAG_SPLITK_FUSED) == 4   # s = 72, not a multiple of 64
    assert blk(Z=None) == 1
    assert blk(Z=0x40000 + 256) == 1                           # Z inside the workspace
    assert "Z overlaps the workspace" in tp.tp_last_error_detail()
    assert blk(ws=0x40000, Z=0x40000 - 256) == 1               # Z runs into the workspace


def test_block_outputs_must_not_overlap_the_workspace():
    """The attention and transformer blocks write their output while their
    row layers still read the workspace (the running sums of the fold in the
    row layer's epilogue), so an output inside the workspace is rejected
    before anything is launched."""
    T, d, h, hkv, dh, p, k = 4, 256, 2, 2, 128, 2, 512
    ws = 0x100000
    n0 = tp.tp_kernel_launch_count()
    na = tp.tp_attn_block_workspace_size(T, d, h, hkv, dh, p)
    assert tp.tp_attn_block(FAKE, FAKE, FAKE, FAKE, FAKE, None, ws + 256, ws, na, T, d, h, hkv,
                            dh, p, True, stream=0, check=False) == 1
    assert tp.tp_attn_block(FAKE, FAKE, FAKE, FAKE, FAKE, None, ws - 256, ws, na, T, d, h, hkv,
                            dh, p, True, stream=0, check=False) == 1
    assert "Z overlaps the workspace" in tp.tp_last_error_detail()
    nt = tp.tp_transformer_block_workspace_size(T, d, h, hkv, dh, k, p)
    prm = tp.block_params(**{name: FAKE for name, _ in tp.BlockParams._fields_
                             if name not in ("W_up", "bo", "b2")})
    assert tp.tp_transformer_block(FAKE2, prm, ws + 512, ws, nt, T, d, h, hkv, dh, k, p,
                                   tp.TP_ACT_GELU_TANH, stream=0, check=False) == 1
    assert "out overlaps the workspace" in tp.tp_last_error_detail()
    assert tp.tp_kernel_launch_count() == n0


def test_valid_call_without_gpu_fails_loudly():
    """With no CUDA device the library reports a CUDA error; it never falls
    back to a host computation."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = _col()
    assert st == 5
    with pytest.raises(tp.TPError):
        tp.tp_column_linear(FAKE, FAKE, None, None, FAKE2, 4, 64, 256, 4, tp.TP_BF16,
                            tp.TP_ACT_GELU_TANH, stream=0)


def test_fused_launch_checks_the_device_before_enqueuing():
    """TP_FLAG_FUSED_LAUNCH resets its tile counters with an asynchronous
    memset; the device check runs before it, so a call that cannot run
    returns with nothing enqueued.  Without a CUDA device the error comes from
    the device query, not from the counter reset."""
    import torch
    if torch.cuda.is_available():
        pytest.skip("a GPU is present")
    st = tp.tp_mlp_block(FAKE, FAKE, None, None, FAKE, None, FAKE2, 0x40000, 1 << 30, 4, 64, 256,
                         4, tp.TP_BF16, tp.TP_ACT_GELU_TANH, tp.TP_FLAG_FUSED_LAUNCH, stream=0,
                         check=False)
    assert st == 5
    detail = tp.tp_last_error_detail()
    assert "counter" not in detail, detail


def test_bf16_bias_alignment_is_checked():
    """The bf16 column epilogue reads b1 as 16-byte vectors: a misaligned
    bias is refused before any launch."""
    st = tp.tp_column_linear(FAKE, FAKE, None, FAKE + 2, FAKE2, 4, 64, 256, 4, tp.TP_BF16,
                             tp.TP_ACT_GELU_TANH, stream=0, check=False)
    assert st == 3


def test_host_entry_workspace_and_validation():
    """tp_mlp_block_host: device copies of X and Z plus the block workspace of
    one chunk, or of two when there are several chunks (consecutive chunks run
    on two streams); chunks of >= 256 rows, multiples of 128, at most eight.
    Every argument error returns before anything is enqueued, and a valid call
    without a GPU fails loudly."""
    def r256(n):
        return -(-n // 256) * 256

    def blk(rows):
        return r256(tp.tp_mlp_block_workspace_size(rows, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH))

    T, d, k, p = 1024, 768, 3072, 2
    # 1024 rows -> four chunks of 256
    want = r256(T * d * 2) + r256(T * d * 4) + 2 * blk(256)
    assert tp.tp_mlp_block_host_workspace_size(T, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH) == want
    # 300 rows -> chunks of 256 and 44
    assert tp.tp_mlp_block_host_workspace_size(300, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH) == \
        r256(300 * d * 2) + r256(300 * d * 4) + 2 * blk(256)
    # 4096 rows -> eight chunks of 512
    assert tp.tp_mlp_block_host_workspace_size(4096, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH) == \
        r256(4096 * d * 2) + r256(4096 * d * 4) + 2 * blk(512)
    # 100 rows -> one chunk, one workspace
    assert tp.tp_mlp_block_host_workspace_size(100, d, k, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH) == \
        r256(100 * d * 2) + r256(100 * d * 4) + blk(100)
    assert tp.tp_mlp_block_host_workspace_size(T, d, 3071, p, tp.TP_BF16, tp.TP_ACT_GELU_TANH) == 0

    def call(**kw):
        a = dict(X=FAKE, W1=FAKE, W_up=None, b1=None, W2=FAKE, b2=None, Z=FAKE2, ws=0x40000,
                 wsb=1 << 30, T=4, d=64, k=256, p=4, dtype=tp.TP_BF16, act=tp.TP_ACT_GELU_TANH,
                 flags=0)
        a.update(kw)
        return tp.tp_mlp_block_host(a["X"], a["W1"], a["W_up"], a["b1"], a["W2"], a["b2"],
                                    a["Z"], a["ws"], a["wsb"], a["T"], a["d"], a["k"], a["p"],
                                    a["dtype"], a["act"], a["flags"], stream=0, check=False)
    n0 = tp.tp_kernel_launch_count()
    assert call(T=0, X=None, Z=None, ws=None, wsb=0) == 0     # empty: a no-op
    assert call(k=255) == 2
    assert call(flags=8) == 1
    assert call(X=None) == 1
    assert call(Z=None) == 1
    assert call(W1=None) == 1
    assert call(W1=FAKE + 2) == 3
    assert call(act=tp.TP_ACT_SWIGLU) == 1                   # SwiGLU needs W_up
    assert call(b1=FAKE + 2) == 3
    assert call(wsb=16) == 7
    assert call(ws=0x40000 + 16) == 3
    assert call(T=-1) == 1
    assert tp.tp_kernel_launch_count() == n0
    import torch
    if not torch.cuda.is_available():
        assert call() == 5


def test_block_workspace_layouts_hold_the_region_counters():
    """The attention block, transformer block and backward workspaces: their
    buffers, each at a 256-byte boundary, then room for one int32 counter per
    128-row x 64-column region (the fold beside the row layer)."""
    def r256(n):
        return -(-n // 256) * 256

    def regions(T, d):
        return r256(4 * (-(-T // 128)) * (-(-d // 64)))

    T, d, h, hkv, dh, p = 1000, 2048, 16, 4, 128, 4
    q, kv = r256(T * h * dh * 2), r256(T * hkv * dh * 2)
    assert tp.tp_attn_block_workspace_size(T, d, h, hkv, dh, p) == \
        2 * q + 2 * kv + r256(p * T * d * 4) + regions(T, d)
    k = 2048
    want = (r256(T * d * 2) + r256(T * d * 4) + q + 2 * kv + q + r256(T * k * 2)
            + r256(p * T * d * 4) + regions(T, d))
    assert tp.tp_transformer_block_workspace_size(T, d, h, hkv, dh, k, p) == want
    # backward: dH (and dU for SwiGLU), the dX partials, the bias-gradient
    # scratch (one row per 128 tokens of max(k, d) fp32), the counters
    for act, halves in ((tp.TP_ACT_GELU_TANH, 1), (tp.TP_ACT_SWIGLU, 2)):
        want = (halves * r256(T * k * 2) + r256(p * T * d * 4)
                + r256(-(-T // 128) * max(k, d) * 4) + regions(T, d))
        assert tp.tp_mlp_block_backward_workspace_size(T, d, k, p, act) == want
