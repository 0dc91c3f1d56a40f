"""GPU parity of the bf16 tensor-core path (tcgen05 + TMEM + TMA) against
the oracle: bit-exact on small-integer inputs (every intermediate an exact
integer), max|gpu - oracle| / max|oracle| <= 1e-2 on the workloads, which at
full size are checked on sampled token rows (each output row depends only on
its own input row, so the oracle can compute any row on its own)."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
from oracle import tp_oracle as O
import workloads as W
from gpu_util import DeviceBlock, bits, host_f32, region_fold_enabled, row_chain_enabled

pytestmark = pytest.mark.gpu

TOL_BF16 = 1e-2


def _oracle(inp, p, act, rows=None):
    X = inp.values("X")
    if rows is not None:
        X = X[rows]
    return O.mlp_sharded(X, inp.values("W1"), inp.values("b1"), inp.values("W2"),
                         inp.values("b2"), p, act, W_up=inp.values("W_up"))


@pytest.mark.parametrize("T,d,s,p", [(1, 64, 64, 1), (3, 64, 8, 4), (130, 200, 40, 4),
                                     (257, 128, 72, 2), (128, 64, 256, 1), (129, 192, 128, 3),
                                     (300, 136, 320, 2)])
@pytest.mark.parametrize("act", ["identity", "relu"])
def test_small_integer_inputs_bit_exact(T, d, s, p, act):
    """Ragged token counts (not multiples of 128), K tails (d, s not
    multiples of 64), N tails (k, d not multiples of 256), shards narrower
    than a tile: all exact."""
    k = s * p
    inp = W.small_integer_inputs(T, d, k, seed=T + 7 * d + s, lo=-1, hi=1, act=act, dtype="bf16")
    ref = _oracle(inp, p, act)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    Y = host_f32(blk.Y)
    for i in range(p):
        assert np.array_equal(Y[i], ref["Y"][i].astype(np.float32)), i
    assert np.array_equal(bits(host_f32(blk.P)), bits(ref["P"]))
    assert np.array_equal(bits(host_f32(blk.Z)), bits(ref["Z"]))
    blk.Z.fill_(float("nan"))
    blk.block()
    blk.sync()
    assert np.array_equal(bits(host_f32(blk.Z)), bits(ref["Z"]))
    if s % 64 == 0:
        blk.Z.fill_(float("nan"))
        blk.block(tp.TP_FLAG_SPLITK_FUSED)
        blk.sync()
        assert np.array_equal(bits(host_f32(blk.Z)), bits(ref["Z"]))


def _random_bf16(T, d, k, act, with_bias, seed):
    rng = np.random.default_rng(seed)
    c = W.f32_to_bf16_bits
    X = c(rng.standard_normal((T, d), dtype=np.float32))
    W1 = c(rng.standard_normal((d, k), dtype=np.float32) * 0.05)
    Wu = c(rng.standard_normal((d, k), dtype=np.float32) * 0.05) if act == "swiglu" else None
    b1 = c(rng.standard_normal(k, dtype=np.float32) * 0.05) if with_bias else None
    W2 = c(rng.standard_normal((k, d), dtype=np.float32) * 0.05)
    b2 = rng.standard_normal(d, dtype=np.float32) * 0.05 if with_bias else None
    return W.Inputs(X, W1, Wu, b1, W2, b2, "bf16")


@pytest.mark.parametrize("act,with_bias", [("gelu_tanh", True), ("gelu_tanh", False),
                                           ("swiglu", False), ("swiglu", True)])
@pytest.mark.parametrize("T,d,k,p", [(200, 256, 1024, 4), (77, 192, 768, 2), (513, 512, 1536, 3)])
def test_random_inputs(act, with_bias, T, d, k, p):
    inp = _random_bf16(T, d, k, act, with_bias, seed=T + d + k + p)
    ref = _oracle(inp, p, act)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    Y = host_f32(blk.Y)
    for i in range(p):
        assert O.rel_err(Y[i], ref["Y"][i]) <= TOL_BF16, i
    assert O.rel_err(host_f32(blk.P), ref["P"]) <= TOL_BF16
    assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_BF16
    for flags in (tp.TP_FLAG_NONE, tp.TP_FLAG_SPLITK_FUSED):
        if flags and (k // p) % 64:
            continue
        blk.Z.fill_(float("nan"))
        blk.block(flags)
        blk.sync()
        assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_BF16, flags


def test_gpt2_config_full():
    """GPT-2-small MLP, T=1024 d=768 k=3072 p=2, GELU(tanh), b1 and b2: every
    output element against the oracle."""
    w = W.WORKLOADS["gpt2"]
    inp = W.make_inputs(w)
    ref = _oracle(inp, w.p, w.act)
    blk = DeviceBlock(inp, w.T, w.d, w.k, w.p, w.act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    Y = host_f32(blk.Y)
    for i in range(w.p):
        assert O.rel_err(Y[i], ref["Y"][i]) <= TOL_BF16
    assert O.rel_err(host_f32(blk.P), ref["P"]) <= TOL_BF16
    assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_BF16
    for flags in (tp.TP_FLAG_NONE, tp.TP_FLAG_SPLITK_FUSED):
        blk.Z.fill_(float("nan"))
        blk.block(flags)
        blk.sync()
        assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_BF16


def _sample_rows(T):
    cand = [0, 1, 127, 128, 129, 255, 1000, 2047, 2048, 3071, T - 129, T - 2, T - 1]
    return sorted({r for r in cand if 0 <= r < T})


@pytest.mark.parametrize("name", ["wide", "decode", "llama"])
def test_full_size_configs_sampled_rows(name):
    """Full-size workloads, launched exactly as the bench launches them;
    the oracle recomputes sampled token rows (all rows for decode).  The
    default block (on wide and Llama the row layer folds the shards in its
    epilogue) gives every bit of the three separate calls."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w)
    rows = list(range(w.T)) if w.T <= 32 else _sample_rows(w.T)
    ref = _oracle(inp, w.p, w.act, rows=rows)
    blk = DeviceBlock(inp, w.T, w.d, w.k, w.p, w.act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    idx = torch.tensor(rows, device="cuda")
    Y = host_f32(blk.Y.index_select(1, idx))
    for i in range(w.p):
        assert O.rel_err(Y[i], ref["Y"][i]) <= TOL_BF16, i
    assert O.rel_err(host_f32(blk.P.index_select(1, idx)), ref["P"]) <= TOL_BF16
    assert O.rel_err(host_f32(blk.Z.index_select(0, idx)), ref["Z"]) <= TOL_BF16
    assert not torch.isnan(blk.Z).any().item()
    for flags in (tp.TP_FLAG_NONE, tp.TP_FLAG_SPLITK_FUSED, tp.TP_FLAG_FUSED_LAUNCH,
                  tp.TP_FLAG_SPLITK_FUSED | tp.TP_FLAG_FUSED_LAUNCH):
        Z2 = torch.full_like(blk.Z, float("nan"))
        ws = blk.block(flags, Z=Z2)
        blk.sync()
        del ws
        assert O.rel_err(host_f32(Z2.index_select(0, idx)), ref["Z"]) <= TOL_BF16, flags
        assert not torch.isnan(Z2).any().item()
        if flags == tp.TP_FLAG_NONE:
            assert torch.equal(Z2.view(torch.int32), blk.Z.view(torch.int32))


@pytest.mark.parametrize("T,d,s,p,act", [(1, 64, 64, 1, "gelu_tanh"), (130, 200, 40, 4, "relu"),
                                         (257, 128, 72, 2, "gelu_tanh"), (300, 192, 128, 3, "swiglu"),
                                         (1024, 768, 1536, 2, "gelu_tanh"), (16, 512, 448, 8, "swiglu"),
                                         (700, 256, 256, 4, "swiglu")])
def test_fused_block_matches_separate_kernels(T, d, s, p, act):
    """tp_mlp_block's fused launch of both GEMM layers gives the same bits as
    the separate column and row launches (both then take the same fixed-order
    fold); split-K agrees with the oracle within tolerance."""
    k = s * p
    inp = _random_bf16(T, d, k, act, with_bias=(act != "swiglu"), seed=T + s)
    blk = DeviceBlock(inp, T, d, k, p, act)
    Zf = torch.full_like(blk.Z, float("nan"))
    Zu = torch.full_like(blk.Z, float("nan"))
    blk.block(tp.TP_FLAG_FUSED_LAUNCH, Z=Zf)
    blk.block(tp.TP_FLAG_NONE, Z=Zu)
    blk.sync()
    assert np.array_equal(bits(host_f32(Zf)), bits(host_f32(Zu)))
    ref = _oracle(inp, p, act)
    assert O.rel_err(host_f32(Zf), ref["Z"]) <= TOL_BF16
    if s % 64 == 0:
        Zs = torch.full_like(blk.Z, float("nan"))
        blk.block(tp.TP_FLAG_SPLITK_FUSED | tp.TP_FLAG_FUSED_LAUNCH, Z=Zs)
        blk.sync()
        assert O.rel_err(host_f32(Zs), ref["Z"]) <= TOL_BF16


def test_fused_block_repeated_calls_reuse_counters():
    """The tile counters live in the workspace and are reset by every call:
    back-to-back calls on the same workspace give identical results."""
    w = W.WORKLOADS["gpt2"]
    blk = DeviceBlock(W.make_inputs(w), w.T, w.d, w.k, w.p, w.act)
    n = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, w.p, blk.dtype, blk.act)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    outs = []
    for _ in range(3):
        Z = torch.full_like(blk.Z, float("nan"))
        tp.tp_mlp_block(blk.X, blk.W1, blk.Wu, blk.b1, blk.W2, blk.b2, Z, ws, n, w.T, w.d, w.k,
                        w.p, blk.dtype, blk.act, tp.TP_FLAG_FUSED_LAUNCH)
        outs.append(Z)
    blk.sync()
    for Z in outs[1:]:
        assert torch.equal(Z, outs[0])


@pytest.mark.parametrize("act,with_bias", [("gelu_tanh", True), ("swiglu", False)])
def test_cta_pair_tiles(act, with_bias):
    """Shapes whose per-layer GEMMs take 256-wide tiles on CTA pairs
    (tcgen05 cta_group::2): ragged T=1000 (a partial second row of a 256-row
    pair tile), four shards; every element against the oracle, and the
    per-layer results against the fused block bit for bit."""
    T, d, k, p = 1000, 2048, 8192, 4
    inp = _random_bf16(T, d, k, act, with_bias, seed=11)
    ref = _oracle(inp, p, act)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    Y = host_f32(blk.Y)
    for i in range(p):
        assert O.rel_err(Y[i], ref["Y"][i]) <= TOL_BF16, i
    assert O.rel_err(host_f32(blk.P), ref["P"]) <= TOL_BF16
    assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_BF16
    Zf = torch.full_like(blk.Z, float("nan"))
    blk.block(tp.TP_FLAG_FUSED_LAUNCH, Z=Zf)
    blk.sync()
    assert np.array_equal(bits(host_f32(Zf)), bits(host_f32(blk.Z)))


@pytest.mark.parametrize("T,d,s,p,act,bias", [(1, 64, 64, 1, "gelu_tanh", True),
                                              (130, 200, 64, 4, "relu", True),
                                              (300, 192, 128, 3, "swiglu", False),
                                              (1024, 768, 1536, 2, "gelu_tanh", True),
                                              (16, 512, 448, 8, "swiglu", False),
                                              (700, 1000, 256, 4, "gelu_tanh", True),
                                              (2000, 2048, 512, 2, "swiglu", True)])
def test_row_fold_is_bit_identical_to_partials_and_fold(T, d, s, p, act, bias):
    """TP_FLAG_ROW_FOLD folds the p partials in the row layer's epilogue: the
    same fp32 accumulators and the same additions in the same order as the
    partials layer followed by the fixed-order reduction, so Z has the same
    bits."""
    k = s * p
    inp = _random_bf16(T, d, k, act, with_bias=bias, seed=T + s + p)
    blk = DeviceBlock(inp, T, d, k, p, act)
    Zr = torch.full_like(blk.Z, float("nan"))
    Zd = torch.full_like(blk.Z, float("nan"))
    blk.block(tp.TP_FLAG_ROW_FOLD, Z=Zr)
    blk.block(tp.TP_FLAG_NONE, Z=Zd)
    blk.sync()
    assert np.array_equal(bits(host_f32(Zr)), bits(host_f32(Zd)))
    if T <= 1024:
        assert O.rel_err(host_f32(Zr), _oracle(inp, p, act)["Z"]) <= TOL_BF16


@pytest.mark.parametrize("name", ["gpt2", "wide", "llama"])
def test_row_fold_full_size(name):
    w = W.WORKLOADS[name]
    blk = DeviceBlock(W.make_inputs(w), w.T, w.d, w.k, w.p, w.act)
    Zr = torch.full_like(blk.Z, float("nan"))
    blk.block(tp.TP_FLAG_ROW_FOLD, Z=Zr)
    blk.block(tp.TP_FLAG_NONE)
    blk.sync()
    assert np.array_equal(bits(host_f32(Zr)), bits(host_f32(blk.Z)))


def test_row_fold_argument_errors():
    w = W.WORKLOADS["gpt2"]
    blk = DeviceBlock(W.make_inputs(w), w.T, w.d, w.k, w.p, w.act)
    for bad in (tp.TP_FLAG_ROW_FOLD | tp.TP_FLAG_SPLITK_FUSED,
                tp.TP_FLAG_ROW_FOLD | tp.TP_FLAG_FUSED_LAUNCH):
        assert tp.tp_mlp_block(blk.X, blk.W1, None, blk.b1, blk.W2, blk.b2, blk.Z, None, 0, w.T,
                               w.d, w.k, w.p, blk.dtype, blk.act, bad, check=False) == 1
    # k/p not a multiple of 64
    inp = _random_bf16(64, 128, 2 * 72, "relu", with_bias=False, seed=1)
    b2 = DeviceBlock(inp, 64, 128, 144, 2, "relu")
    n = tp.tp_mlp_block_workspace_size(64, 128, 144, 2, b2.dtype, b2.act, tp.TP_FLAG_ROW_FOLD)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    assert tp.tp_mlp_block(b2.X, b2.W1, None, None, b2.W2, None, b2.Z, ws, n, 64, 128, 144, 2,
                           b2.dtype, b2.act, tp.TP_FLAG_ROW_FOLD, check=False) == 4


@pytest.mark.parametrize("T,d,s,p,act,bias", [(1, 64, 64, 1, "gelu_tanh", True),
                                              (130, 200, 40, 4, "relu", True),
                                              (257, 128, 72, 2, "gelu_tanh", True),
                                              (300, 192, 128, 3, "swiglu", False),
                                              (1024, 768, 1536, 2, "gelu_tanh", True),
                                              (16, 512, 448, 8, "swiglu", False),
                                              (1000, 2048, 512, 4, "gelu_tanh", True),
                                              (777, 1000, 256, 5, "relu", False)])
def test_block_is_bit_identical_to_separate_calls(T, d, s, p, act, bias):
    """tp_mlp_block's default path (PDL-chained layers, CTA-pair tiles where
    the cost model picks them) gives the same bits as tp_column_linear +
    tp_row_linear + tp_reduce_partials, call after call on one workspace."""
    k = s * p
    inp = _random_bf16(T, d, k, act, with_bias=bias, seed=T + d + p)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    want = bits(host_f32(blk.Z))
    n = tp.tp_mlp_block_workspace_size(T, d, k, p, blk.dtype, blk.act)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    for _ in range(3):
        Zb = torch.full_like(blk.Z, float("nan"))
        tp.tp_mlp_block(blk.X, blk.W1, blk.Wu, blk.b1, blk.W2, blk.b2, Zb, ws, n, T, d, k, p,
                        blk.dtype, blk.act, tp.TP_FLAG_NONE)
        blk.sync()
        assert np.array_equal(bits(host_f32(Zb)), want)


def _counter_bytes(T, d):
    r256 = lambda n: -(-n // 256) * 256  # noqa: E731
    return max(r256(4 * -(-T // 128)), r256(4 * -(-T // 128) * -(-d // 64)))


@pytest.mark.parametrize("T,d,s,p,act,bias", [(1000, 2176, 2048, 4, "gelu_tanh", True),
                                              (777, 2048, 1536, 3, "relu", False),
                                              (513, 1024, 3584, 8, "swiglu", True),
                                              (2048, 4096, 1024, 1, "relu", True),
                                              (1800, 2048, 2048, 2, "gelu_tanh", False)])
def test_block_fold_beside_row_layer(T, d, s, p, act, bias):
    """Shapes whose row layer runs on CTA-pair tiles (256 rows x 256 or 128
    columns; ragged T, a last region 128 columns wide, p = 3 on the generic
    fold, one shard, two): tp_mlp_block folds the partials in the row
    layer's epilogue (each shard's tile adds its partial to the sum the
    previous shard's tile left in Z, the last adds b2), or, with
    TP_DISABLE_ROW_CHAIN=1, beside the row layer once all p shard tiles of a
    region are in memory.  Z has the bits of the three separate calls, call
    after call on one workspace, the workspace's region counters show every
    region counted to 16 p (eight epilogue warps on each CTA of a pair, once
    per shard), and the chain leaves the partials area of the workspace
    unwritten."""
    k = s * p
    inp = _random_bf16(T, d, k, act, with_bias=bias, seed=T + d + p + 1)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    want = bits(host_f32(blk.Z))
    n = tp.tp_mlp_block_workspace_size(T, d, k, p, blk.dtype, blk.act)
    ws = torch.full((n,), 0x7F, dtype=torch.uint8, device="cuda")
    m_regions = -(-T // 256)
    for _ in range(3):
        Zb = torch.full_like(blk.Z, float("nan"))
        tp.tp_mlp_block(blk.X, blk.W1, blk.Wu, blk.b1, blk.W2, blk.b2, Zb, ws, n, T, d, k, p,
                        blk.dtype, blk.act, tp.TP_FLAG_NONE)
        blk.sync()
        assert np.array_equal(bits(host_f32(Zb)), want)
        if not region_fold_enabled():
            continue
        cnt = ws[n - _counter_bytes(T, d):].cpu().numpy().view(np.int32)
        assert cnt[0] == 16 * p
        assert set(np.unique(cnt).tolist()) <= {0, 16 * p}
        assert int((cnt == 16 * p).sum()) in (m_regions * -(-d // 256), m_regions * -(-d // 128))
        y_bytes = -(-T * k * 2 // 256) * 256
        partials = ws[y_bytes:y_bytes + p * T * d * 4]
        untouched = bool((partials == 0x7F).all().item())
        assert untouched == row_chain_enabled()
    if T <= 1024:
        assert O.rel_err(host_f32(blk.Z), _oracle(inp, p, act)["Z"]) <= TOL_BF16


def test_block_fold_after_row_layer_with_unaligned_b2():
    """A b2 that is only 4-byte aligned keeps the fold after the row layer
    (the overlapped fold reads b2 as 16-byte vectors): same bits."""
    T, d, s, p, act = 1000, 2048, 512, 4, "gelu_tanh"
    k = s * p
    inp = _random_bf16(T, d, k, act, with_bias=True, seed=5)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    want = bits(host_f32(blk.Z))
    b2u = torch.empty(d + 1, dtype=torch.float32, device="cuda")[1:]
    b2u.copy_(blk.b2)
    n = tp.tp_mlp_block_workspace_size(T, d, k, p, blk.dtype, blk.act)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    Zb = torch.full_like(blk.Z, float("nan"))
    tp.tp_mlp_block(blk.X, blk.W1, blk.Wu, blk.b1, blk.W2, b2u, Zb, ws, n, T, d, k, p,
                    blk.dtype, blk.act, tp.TP_FLAG_NONE)
    blk.sync()
    assert np.array_equal(bits(host_f32(Zb)), want)
