"""GPU parity of the transformer-block path against the oracle: LayerNorm
(tp_layer_norm), the reduction with the residual folded in
(tp_reduce_partials_residual, bit-exact), and the whole pre-norm block
(tp_transformer_block).

LayerNorm tolerance.  The kernel takes the row mean and variance in fp32
(relative error ~1e-6 at d <= 16384) and rounds the result once to bf16, an
error of at most 2^-9 relative; so |Y_gpu - Y_ref| <= 2^-8 |Y_ref| + 1e-5.

Block tolerance.  Every GEMM reads bf16 and accumulates fp32, as in the MLP
and attention tests; the block's own contribution out - X is compared with
max|err| / max|ref| <= 1e-2 (the residual X itself would otherwise hide
errors)."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
import workloads as W
from gpu_util import bits, dev, host_f32, pairs_enabled, row_chain_enabled
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu


@pytest.mark.parametrize("T,d", [(1, 768), (300, 768), (77, 100), (64, 4096), (33, 16384), (5, 4)])
def test_layer_norm_matches_oracle(T, d):
    rng = np.random.default_rng(T * 7 + d)
    X = (rng.standard_normal((T, d), dtype=np.float32) * 2.5 + 0.75).astype(np.float32)
    g = (1.0 + 0.1 * rng.standard_normal(d)).astype(np.float32)
    b = (0.1 * rng.standard_normal(d)).astype(np.float32)
    Y = torch.full((T, d), float("nan"), dtype=torch.bfloat16, device="cuda")
    tp.tp_layer_norm(dev(X), dev(g), dev(b), Y, T, d, 1e-5)
    tp.tp_sync_status()
    got = host_f32(Y).astype(np.float64)
    want = O.layer_norm(X, g, b, 1e-5)
    assert np.all(np.abs(got - want) <= 2.0 ** -8 * np.abs(want) + 1e-5)


def test_layer_norm_constant_rows_give_beta():
    T, d = 4, 512
    X = np.full((T, d), 3.0, dtype=np.float32)
    g = np.linspace(0.5, 1.5, d, dtype=np.float32)
    b = W.bf16_bits_to_f32(W.f32_to_bf16_bits(np.linspace(-1, 1, d, dtype=np.float32)))
    Y = torch.empty((T, d), dtype=torch.bfloat16, device="cuda")
    tp.tp_layer_norm(dev(X), dev(g), dev(b), Y, T, d, 1e-5)
    tp.tp_sync_status()
    assert np.array_equal(host_f32(Y), np.tile(b, (T, 1)))


@pytest.mark.parametrize("p,T,d", [(1, 5, 8), (2, 300, 768), (3, 17, 100), (4, 129, 4096),
                                   (8, 16, 8192), (2, 3, 16384)])
@pytest.mark.parametrize("bias", [True, False])
def test_residual_fold_bit_exact(p, T, d, bias):
    P = W.random_partials(p, T, d, seed=p * 31 + T)
    rng = np.random.default_rng(d)
    b = (rng.standard_normal(d) * 4.0).astype(np.float32) if bias else None
    R = (rng.standard_normal((T, d)) * 64.0).astype(np.float32)
    Z = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    tp.tp_reduce_partials_residual(dev(P), dev(b), dev(R), Z, T, d, p)
    tp.tp_sync_status()
    want = O.reduce_partials_fixed_order(P, b, R)
    assert np.array_equal(bits(host_f32(Z)), bits(want))


def test_residual_fold_in_place_and_without_residual():
    p, T, d = 4, 64, 1024
    P = W.random_partials(p, T, d, seed=9)
    R = np.random.default_rng(1).standard_normal((T, d)).astype(np.float32)
    Rd = dev(R)
    tp.tp_reduce_partials_residual(dev(P), None, Rd, Rd, T, d, p)   # Z == residual
    Z2 = torch.empty((T, d), dtype=torch.float32, device="cuda")
    tp.tp_reduce_partials_residual(dev(P), None, None, Z2, T, d, p)
    tp.tp_sync_status()
    assert np.array_equal(bits(host_f32(Rd)), bits(O.reduce_partials_fixed_order(P, None, R)))
    assert np.array_equal(bits(host_f32(Z2)), bits(O.reduce_partials_fixed_order(P)))


def test_row_op_argument_errors():
    T, d = 8, 102   # d % 4 != 0
    X = torch.zeros((T, 104), dtype=torch.float32, device="cuda")
    Y = torch.zeros((T, 104), dtype=torch.bfloat16, device="cuda")
    g = torch.ones(104, dtype=torch.float32, device="cuda")
    assert tp.tp_layer_norm(X, g, g, Y, T, d, 1e-5, check=False) == 4
    assert tp.tp_layer_norm(X, g, g, Y, T, 20000, 1e-5, check=False) == 4
    assert tp.tp_layer_norm(X, g, g, Y, T, 104, 0.0, check=False) == 1
    assert tp.tp_layer_norm(X, None, g, Y, T, 104, 1e-5, check=False) == 1
    P = torch.zeros((2, T, 104), dtype=torch.float32, device="cuda")
    assert tp.tp_reduce_partials_residual(P, None, None, P[1], T, 104, 2, check=False) == 1


class DeviceTransformerBlock:
    def __init__(self, inp, T, d, h, hkv, dh, k, p, act):
        self.T, self.d, self.h, self.hkv, self.dh, self.k, self.p = T, d, h, hkv, dh, k, p
        self.act = tp.ACT[act]
        self.X = dev(inp.X)
        self.t = {name: dev(v) for name, v in inp.prm.items()}
        self.prm = tp.block_params(**self.t)
        self.n = tp.tp_transformer_block_workspace_size(T, d, h, hkv, dh, k, p)
        self.ws = torch.empty(self.n, dtype=torch.uint8, device="cuda")
        self.out = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")

    def run(self, causal=True, out=None):
        out = self.out if out is None else out
        tp.tp_transformer_block(self.X, self.prm, out, self.ws, self.n, self.T, self.d, self.h,
                                self.hkv, self.dh, self.k, self.p, self.act, causal)
        tp.tp_sync_status()
        return host_f32(out)


BLOCK_CASES = [
    # T, d, h, h_kv, k, p, act, causal
    (300, 256, 4, 2, 512, 2, "gelu_tanh", True),
    (129, 512, 4, 4, 1024, 4, "swiglu", True),
    (200, 256, 2, 2, 768, 2, "gelu_tanh", False),
    (1, 128, 2, 1, 256, 1, "swiglu", True),
    (333, 1024, 8, 8, 2048, 8, "swiglu", True),     # one K/V head per shard, ragged T
    (257, 768, 6, 2, 3072, 2, "gelu_tanh", True),   # GPT-2 width, 3 query heads per K/V head
]


@pytest.mark.parametrize("T,d,h,hkv,k,p,act,causal", BLOCK_CASES)
def test_transformer_block_matches_oracle(T, d, h, hkv, k, p, act, causal):
    inp = W.make_block_inputs(T, d, h, hkv, 128, k, act, seed=T + d, w_std=0.05)
    blk = DeviceTransformerBlock(inp, T, d, h, hkv, 128, k, p, act)
    got = blk.run(causal)
    ref = O.transformer_block_sharded(inp.X, inp.value_dict(), p, h, hkv, 128, act, causal,
                                      hidden_round="bf16")["out"]
    assert np.isfinite(got).all()
    assert O.rel_err(got - inp.X, ref - inp.X) <= 1e-2


def test_transformer_block_in_place():
    T, d, h, k, p = 130, 256, 2, 512, 2
    inp = W.make_block_inputs(T, d, h, h, 128, k, "gelu_tanh", seed=3, w_std=0.05)
    blk = DeviceTransformerBlock(inp, T, d, h, h, 128, k, p, "gelu_tanh")
    want = blk.run(True)
    got = blk.run(True, out=blk.X)     # out == X
    assert np.array_equal(bits(got), bits(want))


@pytest.mark.parametrize("name,n", [("block_wide", 128), ("block_llama", 32)])
def test_transformer_block_full_size_prefix(name, n):
    """Full-size causal blocks.  Every step is row-wise except causal
    attention, so rows 0..n-1 of the output depend only on the first n rows
    of X: the oracle runs on that prefix."""
    w = W.BLOCK_WORKLOADS[name]
    inp = W.make_block_inputs(w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, w.k, w.act, seed=42)
    blk = DeviceTransformerBlock(inp, w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, w.k, w.p,
                                 w.act)
    got = blk.run(True)
    assert np.isfinite(got).all()
    ref = O.transformer_block_sharded(inp.X[:n], inp.value_dict(), w.p, w.n_heads, w.n_kv_heads,
                                      w.head_dim, w.act, True, hidden_round="bf16")["out"]
    assert O.rel_err(got[:n] - inp.X[:n], ref - inp.X[:n]) <= 1e-2


@pytest.mark.parametrize("T,act", [(1000, "gelu_tanh"), (1000, "swiglu"), (2048, "gelu_tanh")])
def test_transformer_block_is_bit_identical_to_separate_calls(T, act):
    """Shapes whose MLP row layer runs on CTA-pair tiles (d=2048, k=2048 on
    p=4), so reduction #2 (+ b2 + H) runs in that layer's epilogue, or beside
    it with TP_DISABLE_ROW_CHAIN=1 (at T=2048 the Q, K, V projections also
    run as one launch): the block gives the bits of its
    steps called one by one (LayerNorm, the three projections, attention,
    W_O, fold + bo + X, LayerNorm, the MLP layers, fold + b2 + H), call
    after call on one workspace."""
    d, h, hkv, k, p = 2048, 16, 4, 2048, 4
    inp = W.make_block_inputs(T, d, h, hkv, 128, k, act, seed=11, w_std=0.03)
    blk = DeviceTransformerBlock(inp, T, d, h, hkv, 128, k, p, act)
    t, X = blk.t, blk.X
    kq, kkv, s = h * 128, hkv * 128, k // p
    bf = torch.bfloat16
    A = torch.empty((T, d), dtype=bf, device="cuda")
    Q = torch.empty((p, T, kq // p), dtype=bf, device="cuda")
    K = torch.empty((p, T, kkv // p), dtype=bf, device="cuda")
    V = torch.empty_like(K)
    Oh = torch.empty_like(Q)
    P = torch.empty((p, T, d), dtype=torch.float32, device="cuda")
    H = torch.empty((T, d), dtype=torch.float32, device="cuda")
    Yh = torch.empty((p, T, s), dtype=bf, device="cuda")
    out = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ident, a = tp.TP_ACT_IDENTITY, tp.ACT[act]
    tp.tp_layer_norm(X, t["ln1_gamma"], t["ln1_beta"], A, T, d)
    tp.tp_column_linear(A, t["Wq"], None, None, Q, T, d, kq, p, tp.TP_BF16, ident)
    tp.tp_column_linear(A, t["Wk"], None, None, K, T, d, kkv, p, tp.TP_BF16, ident)
    tp.tp_column_linear(A, t["Wv"], None, None, V, T, d, kkv, p, tp.TP_BF16, ident)
    tp.tp_attention_heads(Q, K, V, Oh, T, p, h, hkv, 128, 1)
    tp.tp_row_linear(Oh, t["Wo"], P, T, kq, d, p, tp.TP_BF16)
    tp.tp_reduce_partials_residual(P, t["bo"], X, H, T, d, p)
    tp.tp_layer_norm(H, t["ln2_gamma"], t["ln2_beta"], A, T, d)
    tp.tp_column_linear(A, t["W1"], t.get("W_up"), t["b1"], Yh, T, d, k, p, tp.TP_BF16, a)
    tp.tp_row_linear(Yh, t["W2"], P, T, k, d, p, tp.TP_BF16)
    tp.tp_reduce_partials_residual(P, t["b2"], H, out, T, d, p)
    tp.tp_sync_status()
    want = bits(host_f32(out))
    for _ in range(2):
        before = tp.tp_kernel_launch_count()
        got = blk.run(True)
        launches = tp.tp_kernel_launch_count() - before
        assert np.array_equal(bits(got), want)
        # LN, Q K V (one launch at T=2048, three at T=1000), attention, W_O,
        # fold + LN, the two MLP layers, and the fold unless the row layer
        # does it
        qkv = 1 if T >= 2000 and pairs_enabled() else 3
        assert launches == qkv + (6 if row_chain_enabled() else 7)
