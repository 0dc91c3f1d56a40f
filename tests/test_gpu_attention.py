"""GPU parity of the tensor-parallel attention path against the oracle.

tp_attention_heads (every shard's heads, tcgen05 flash attention) is checked
head by head against the oracle's float64 softmax attention on the same bf16
Q, K, V; tp_attn_block (column Q/K/V -> attention -> row Wo -> fold) against
the oracle's sharded block with bf16 storage of Q, K, V and O.

Tolerance of one attention output element.  The kernel keeps scores,
maxima, sums and the O accumulator in fp32; it rounds the probabilities
P = exp(s - m) to bf16 before P V and rounds O to bf16 once at the end.  A
relative error of at most 2^-9 on every probability moves O by at most
2^-9 * max|v| (a convex combination of the value rows), and the final
rounding adds at most 2^-9 * |O|.  The scores themselves carry fp32
rounding: the tensor core's fp32 sum of 128 exact bf16 products is off by at
most 128 * 2^-24 * sum|q_i k_i| (about 2.5e-3 for the std-2 inputs of the
peaked test, far less for the others); scaled by log2(e)/sqrt(128) = 0.1275
and turned into a relative error of the probability by ln 2, that is below
2^-12 on every probability, so at most 2^-12 * max|v| on O (the fma forming
the exponent argument and the exp2 approximation add about 2^-20).  So
    |O_gpu - O_ref| <= 2^-9 * (max|v| + |O_ref|) + 2^-12 * max|v|."""

import math

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
import workloads as W
from gpu_util import bits, dev, host_f32, pairs_enabled, row_chain_enabled
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

EPS = 2.0 ** -9          # bf16 rounding of P and of O
EPS_SCORE = 2.0 ** -12   # fp32 rounding of the scores and exponent argument


def _bf16_vals(a):
    return W.bf16_bits_to_f32(a).astype(np.float64)


def _run_heads(Qb, Kb, Vb, p, T, h, hkv, causal):
    Qd, Kd, Vd = dev(Qb), dev(Kb), dev(Vb)
    Od = torch.full((p, T, (h // p) * 128), float("nan"), dtype=torch.bfloat16, device="cuda")
    tp.tp_attention_heads(Qd, Kd, Vd, Od, T, p, h, hkv, 128, causal)
    tp.tp_sync_status()
    return host_f32(Od).astype(np.float64)


def _check_head(got, q, k, v, causal):
    want = O.sdpa_head(q, k, v, causal)
    bound = EPS * (np.abs(v).max() + np.abs(want)) + EPS_SCORE * np.abs(v).max()
    err = np.abs(got - want)
    assert np.all(err <= bound), (float(err.max()), float((err / bound).max()))
    return want


HEAD_CASES = [
    # p, T, h, h_kv, causal
    (1, 128, 1, 1, False),     # one query block, one key block
    (1, 1, 2, 1, False),       # a single token
    (2, 300, 4, 2, True),      # ragged tail, grouped K/V, causal
    (2, 300, 4, 2, False),
    (2, 129, 4, 4, True),      # one row past a block
    (4, 517, 8, 4, True),      # several blocks per unit, more units than rounds
    (2, 640, 8, 2, False),     # group of 4 query heads per K/V head
    (8, 383, 16, 8, True),     # one K/V head per shard, 8 shards
    (1, 1200, 3, 1, True),     # odd head count, 3 query heads on one K/V head
]


@pytest.mark.parametrize("p,T,h,hkv,causal", HEAD_CASES)
def test_attention_heads_match_oracle(p, T, h, hkv, causal):
    hq, hk = h // p, hkv // p
    Qb, Kb, Vb = W.make_qkv(p, T, hq, hk, 128, seed=T + 7 * h + hkv)
    got = _run_heads(Qb, Kb, Vb, p, T, h, hkv, causal)
    Q, K, V = _bf16_vals(Qb), _bf16_vals(Kb), _bf16_vals(Vb)
    group = h // hkv
    assert np.isfinite(got).all()
    for i in range(p):
        for j in range(hq):
            g = j // group
            cs, gs = slice(j * 128, (j + 1) * 128), slice(g * 128, (g + 1) * 128)
            _check_head(got[i][:, cs], Q[i][:, cs], K[i][:, gs], V[i][:, gs], causal)


def test_attention_heads_peaked_scores():
    """Large scores (std 2 inputs): the running maximum changes from block to
    block and the O rescaling in tensor memory is exercised."""
    p, T, h, hkv = 1, 700, 2, 2
    Qb, Kb, Vb = W.make_qkv(p, T, h, hkv, 128, seed=5, std=2.0)
    got = _run_heads(Qb, Kb, Vb, p, T, h, hkv, causal=False)
    Q, K, V = _bf16_vals(Qb), _bf16_vals(Kb), _bf16_vals(Vb)
    for j in range(h):
        cs = slice(j * 128, (j + 1) * 128)
        _check_head(got[0][:, cs], Q[0][:, cs], K[0][:, cs], V[0][:, cs], False)


@pytest.mark.parametrize("name", ["attn_wide", "attn_llama"])
def test_attention_heads_full_size_sampled(name):
    """The full-size head layout (4096 tokens, all shards and heads in one
    launch); sampled query rows are checked one by one."""
    w = W.ATTN_WORKLOADS[name]
    p, T, hq, hk = w.p, w.T, w.n_heads // w.p, w.n_kv_heads // w.p
    Qb, Kb, Vb = W.make_qkv(p, T, hq, hk, 128, seed=11)
    got = _run_heads(Qb, Kb, Vb, p, T, w.n_heads, w.n_kv_heads, w.causal)
    assert np.isfinite(got).all()
    group = w.n_heads // w.n_kv_heads
    rng = np.random.default_rng(3)
    rows = [0, 1, 127, 128, 2047, T - 1] + list(rng.integers(0, T, 4))
    for i in sorted({0, p - 1}):
        for j in sorted({0, hq - 1}):
            g = j // group
            cs, gs = slice(j * 128, (j + 1) * 128), slice(g * 128, (g + 1) * 128)
            K, V = _bf16_vals(Kb[i][:, gs]), _bf16_vals(Vb[i][:, gs])
            for t in rows:
                q = _bf16_vals(Qb[i][t:t + 1, cs])
                n = t + 1 if w.causal else T
                want = O.sdpa_head(q, K[:n], V[:n], False)[0]
                bound = EPS * (np.abs(V[:n]).max() + np.abs(want)) + EPS_SCORE * np.abs(V[:n]).max()
                assert np.all(np.abs(got[i][t, cs] - want) <= bound), (i, j, t)


def _run_block(inp, T, d, h, hkv, p, causal):
    X, Wq, Wk, Wv, Wo = dev(inp.X), dev(inp.Wq), dev(inp.Wk), dev(inp.Wv), dev(inp.Wo)
    bo = dev(inp.bo)
    Z = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    n = tp.tp_attn_block_workspace_size(T, d, h, hkv, 128, p)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    tp.tp_attn_block(X, Wq, Wk, Wv, Wo, bo, Z, ws, n, T, d, h, hkv, 128, p, causal)
    tp.tp_sync_status()
    return host_f32(Z)


BLOCK_CASES = [
    # T, d, h, h_kv, p, causal, bias
    (300, 256, 4, 2, 2, True, True),
    (300, 256, 4, 4, 4, False, False),
    (1, 128, 2, 2, 1, True, True),
    (520, 512, 8, 2, 2, True, False),
    (130, 256, 16, 16, 1, True, True),   # 16 heads on one shard: 2048-row W_O shard
    (200, 384, 32, 8, 2, False, True),   # 4 query heads per K/V head, 16 per shard
]


@pytest.mark.parametrize("T,d,h,hkv,p,causal,bias", BLOCK_CASES)
def test_attention_block_matches_oracle(T, d, h, hkv, p, causal, bias):
    inp = W.make_attn_inputs(T, d, h, hkv, 128, seed=T + d, with_bias=bias, w_std=0.05)
    got = _run_block(inp, T, d, h, hkv, p, causal)
    ref = O.attention_sharded(inp.values("X"), inp.values("Wq"), inp.values("Wk"),
                              inp.values("Wv"), inp.values("Wo"), inp.bo, p, h, hkv, 128, causal,
                              hidden_round="bf16")["Z"]
    assert np.isfinite(got).all()
    assert O.rel_err(got, ref) <= 1e-2


@pytest.mark.parametrize("name", ["attn_wide", "attn_llama"])
def test_attention_block_full_size_prefix(name):
    """Full-size causal blocks; with a causal mask row t depends only on
    tokens 0..t, so the oracle run on the first rows of X gives those rows of
    the full result exactly."""
    w = W.ATTN_WORKLOADS[name]
    inp = W.make_attn_inputs(w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, seed=42)
    got = _run_block(inp, w.T, w.d, w.n_heads, w.n_kv_heads, w.p, w.causal)
    assert np.isfinite(got).all()
    n = 160
    ref = O.attention_sharded(inp.values("X")[:n], inp.values("Wq"), inp.values("Wk"),
                              inp.values("Wv"), inp.values("Wo"), None, w.p, w.n_heads,
                              w.n_kv_heads, w.head_dim, True, hidden_round="bf16")["Z"]
    assert O.rel_err(got[:n], ref) <= 1e-2


def test_attention_argument_errors():
    T, p = 64, 2
    Q = torch.zeros((p, T, 2 * 128), dtype=torch.bfloat16, device="cuda")
    Ob = torch.zeros_like(Q)
    assert tp.tp_attention_heads(Q, Q, Q, Ob, T, p, 4, 4, 64, False, check=False) == 4
    assert tp.tp_attention_heads(Q, Q, Q, Ob, T, p, 3, 3, 128, False, check=False) == 2
    assert tp.tp_attention_heads(Q, Q, Q, Ob, T, p, 4, 3, 128, False, check=False) == 2
    assert tp.tp_attention_heads(None, Q, Q, Ob, T, p, 4, 4, 128, False, check=False) == 1
    assert tp.tp_attention_heads(Q, Q, Q, Ob, 0, p, 4, 4, 128, False, check=False) == 0
    assert tp.tp_attn_block_workspace_size(T, 256, 4, 4, 64, p) == 0
    with pytest.raises(tp.TPError, match="divisible"):
        tp.tp_attention_heads(Q, Q, Q, Ob, T, p, 6, 3, 128, False)


def test_attention_dropped_load_times_out():
    """A K/V load the producer never issues: the MMA warp's bounded wait runs
    out, every role stops, TMEM is freed and the status word reports the
    timeout; the next launch computes correctly."""
    p, T, h, hkv = 2, 300, 4, 2
    Qb, Kb, Vb = W.make_qkv(p, T, h // p, hkv // p, 128, seed=1)
    Qd, Kd, Vd = dev(Qb), dev(Kb), dev(Vb)
    Od = torch.zeros((p, T, (h // p) * 128), dtype=torch.bfloat16, device="cuda")
    tp.tp_set_wait_timeout_ns(50_000_000)
    try:
        assert tp.tp_sync_status(check=False) == 0
        tp.tp_debug_drop_load(2)
        tp.tp_attention_heads(Qd, Kd, Vd, Od, T, p, h, hkv, 128, True)
        assert tp.tp_sync_status(check=False) == 6
    finally:
        tp.tp_set_wait_timeout_ns(0)
        tp.tp_debug_drop_load(-1)
    got = _run_heads(Qb, Kb, Vb, p, T, h, hkv, True)
    Q, K, V = _bf16_vals(Qb), _bf16_vals(Kb), _bf16_vals(Vb)
    _check_head(got[1][:, :128], Q[1][:, :128], K[1][:, :128], V[1][:, :128], True)


@pytest.mark.parametrize("T,h,hkv,bias", [(1000, 16, 4, True), (1000, 16, 4, False),
                                          (2048, 16, 4, True), (2000, 12, 4, False),
                                          (2048, 32, 8, False)])
def test_attention_block_is_bit_identical_to_separate_calls(T, h, hkv, bias):
    """Shapes whose output projection runs on CTA-pair tiles (d=2048, p=4).
    At T >= 2000 the Q, K, V projections also run as one launch of pair
    tiles: 256 x 128 tiles at 16 and 12 query heads (T=2000: a ragged last
    row tile and 384-column Q shards that start inside a tile), 256 x 256
    tiles at 32 / 8 heads.  tp_attn_block, whose fold runs in the output
    projection's epilogue, gives the bits of the separate calls (three column
    projections, tp_attention_heads, tp_row_linear, tp_reduce_partials),
    call after call on one workspace."""
    d, p = 2048, 4
    inp = W.make_attn_inputs(T, d, h, hkv, 128, seed=7, with_bias=bias, w_std=0.03)
    X, Wq, Wk, Wv, Wo = dev(inp.X), dev(inp.Wq), dev(inp.Wk), dev(inp.Wv), dev(inp.Wo)
    bo = dev(inp.bo)
    kq, kkv = h * 128, hkv * 128
    Q = torch.empty((p, T, kq // p), dtype=torch.bfloat16, device="cuda")
    K = torch.empty((p, T, kkv // p), dtype=torch.bfloat16, device="cuda")
    V = torch.empty_like(K)
    Oh = torch.empty_like(Q)
    P = torch.empty((p, T, d), dtype=torch.float32, device="cuda")
    Zs = torch.empty((T, d), dtype=torch.float32, device="cuda")
    ident = tp.TP_ACT_IDENTITY
    tp.tp_column_linear(X, Wq, None, None, Q, T, d, kq, p, tp.TP_BF16, ident)
    tp.tp_column_linear(X, Wk, None, None, K, T, d, kkv, p, tp.TP_BF16, ident)
    tp.tp_column_linear(X, Wv, None, None, V, T, d, kkv, p, tp.TP_BF16, ident)
    tp.tp_attention_heads(Q, K, V, Oh, T, p, h, hkv, 128, 1)
    tp.tp_row_linear(Oh, Wo, P, T, kq, d, p, tp.TP_BF16)
    tp.tp_reduce_partials(P, bo, Zs, T, d, p)
    tp.tp_sync_status()
    want = bits(host_f32(Zs))
    n = tp.tp_attn_block_workspace_size(T, d, h, hkv, 128, p)
    ws = torch.full((n,), 0x7F, dtype=torch.uint8, device="cuda")
    for _ in range(2):
        Z = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
        before = tp.tp_kernel_launch_count()
        tp.tp_attn_block(X, Wq, Wk, Wv, Wo, bo, Z, ws, n, T, d, h, hkv, 128, p, 1)
        launches = tp.tp_kernel_launch_count() - before
        tp.tp_sync_status()
        assert np.array_equal(bits(host_f32(Z)), want)
        # Q, K, V in one launch at T >= 2000, three below; then attention,
        # and W_O with the fold in its epilogue, or W_O and the fold
        qkv = 1 if T >= 2000 and pairs_enabled() else 3
        assert launches == qkv + (2 if row_chain_enabled() else 3)
