"""Bounded device waits: a load the producer never issues makes the consumer's
wait run out; the kernel records TP_ERR_DEVICE_TIMEOUT, stops every role of
the CTA, frees its TMEM and returns, and the context stays usable.  The fault
is injected on the host (tp_debug_drop_load: the next tensor-core launch skips
one pipeline slot) -- nothing traps or faults."""

import re

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
from oracle import tp_oracle as O
import workloads as W
from gpu_util import DeviceBlock, host_f32, region_fold_enabled

pytestmark = pytest.mark.gpu

SHORT = 50_000_000  # 50 ms


@pytest.fixture
def short_timeout():
    tp.tp_set_wait_timeout_ns(SHORT)
    yield
    tp.tp_set_wait_timeout_ns(0)
    tp.tp_debug_drop_load(-1)


def _block():
    rng = np.random.default_rng(0)
    c = W.f32_to_bf16_bits
    T, d, k, p = 300, 256, 1024, 4
    inp = W.Inputs(c(rng.standard_normal((T, d), dtype=np.float32)),
                   c(rng.standard_normal((d, k), dtype=np.float32) * 0.05), None,
                   c(rng.standard_normal(k, dtype=np.float32) * 0.05),
                   c(rng.standard_normal((k, d), dtype=np.float32) * 0.05),
                   rng.standard_normal(d, dtype=np.float32) * 0.05, "bf16")
    return inp, DeviceBlock(inp, T, d, k, p, "gelu_tanh")


def _check_healthy(inp, blk):
    blk.Z.fill_(float("nan"))
    blk.block()
    assert tp.tp_sync_status(check=False) == 0
    ref = O.mlp_sharded(inp.values("X"), inp.values("W1"), inp.values("b1"), inp.values("W2"),
                        inp.values("b2"), blk.p, "gelu_tanh")["Z"]
    assert O.rel_err(host_f32(blk.Z), ref) <= 1e-2


@pytest.mark.parametrize("slot", [0, 3])
def test_dropped_load_in_column_gemm_times_out(short_timeout, slot):
    inp, blk = _block()
    assert tp.tp_sync_status(check=False) == 0
    tp.tp_debug_drop_load(slot)
    tp.tp_column_linear(blk.X, blk.W1, None, blk.b1, blk.Y, blk.T, blk.d, blk.k, blk.p,
                        tp.TP_BF16, tp.TP_ACT_GELU_TANH)
    st = tp.tp_sync_status(check=False)
    assert st == 6, tp.tp_status_string(st)
    assert "status bits" in tp.tp_last_error_detail()
    # the status word was cleared and the device still computes correctly
    assert tp.tp_sync_status(check=False) == 0
    _check_healthy(inp, blk)


def test_dropped_load_in_fused_block_times_out(short_timeout):
    inp, blk = _block()
    tp.tp_debug_drop_load(2)
    blk.block(tp.TP_FLAG_FUSED_LAUNCH)
    st = tp.tp_sync_status(check=False)
    assert st == 6, tp.tp_status_string(st)
    _check_healthy(inp, blk)


def test_drop_applies_to_one_launch_only(short_timeout):
    inp, blk = _block()
    tp.tp_debug_drop_load(1)
    blk.column()
    assert tp.tp_sync_status(check=False) == 6
    blk.column()   # no drop armed any more
    assert tp.tp_sync_status(check=False) == 0


def test_dropped_load_in_cta_pair_gemm_times_out(short_timeout):
    """A shape whose column layer runs on CTA pairs (256 x 256 tiles): the
    first pair's even CTA's MMA wait runs out, both CTAs of that pair stop,
    meet at the cluster barrier and free their TMEM; the other pairs finish."""
    rng = np.random.default_rng(1)
    c = W.f32_to_bf16_bits
    T, d, k, p = 1000, 2048, 8192, 4
    inp = W.Inputs(c(rng.standard_normal((T, d), dtype=np.float32)),
                   c(rng.standard_normal((d, k), dtype=np.float32) * 0.02), None, None,
                   c(rng.standard_normal((k, d), dtype=np.float32) * 0.02), None, "bf16")
    blk = DeviceBlock(inp, T, d, k, p, "gelu_tanh")
    tp.tp_debug_drop_load(5)
    blk.column()
    assert tp.tp_sync_status(check=False) == 6
    blk.column()
    blk.row()
    blk.reduce()
    assert tp.tp_sync_status(check=False) == 0
    ref = O.mlp_sharded(inp.values("X")[:64], inp.values("W1"), None, inp.values("W2"), None, p,
                        "gelu_tanh")["Z"]
    assert O.rel_err(host_f32(blk.Z)[:64], ref) <= 1e-2



def test_dropped_load_in_attention_times_out(short_timeout):
    """The attention kernel: a K/V block the producer never loads makes the
    MMA issuer's wait run out; the softmax warps see the abort flag and stop;
    the next launch is correct."""
    rng = np.random.default_rng(2)
    p, T, h, hkv = 2, 300, 4, 2
    shape = lambda heads: (p, T, (heads // p) * 128)  # noqa: E731
    Q = rng.standard_normal(shape(h), dtype=np.float32)
    K = rng.standard_normal(shape(hkv), dtype=np.float32)
    V = rng.standard_normal(shape(hkv), dtype=np.float32)
    c = W.f32_to_bf16_bits
    dv = lambda a: torch.from_numpy(c(a).view(np.int16)).view(torch.bfloat16).cuda()  # noqa: E731
    Qd, Kd, Vd = dv(Q), dv(K), dv(V)
    Od = torch.full(shape(h), float("nan"), dtype=torch.bfloat16, device="cuda")
    tp.tp_debug_drop_load(2)
    tp.tp_attention_heads(Qd, Kd, Vd, Od, T, p, h, hkv, 128, 1)
    st = tp.tp_sync_status(check=False)
    assert st == 6, tp.tp_status_string(st)
    Od.fill_(float("nan"))
    tp.tp_attention_heads(Qd, Kd, Vd, Od, T, p, h, hkv, 128, 1)
    assert tp.tp_sync_status(check=False) == 0
    got = host_f32(Od).astype(np.float64)
    qv = W.bf16_bits_to_f32(c(Q)).astype(np.float64)
    kv = W.bf16_bits_to_f32(c(K)).astype(np.float64)
    vv = W.bf16_bits_to_f32(c(V)).astype(np.float64)
    for s in range(p):
        for hh in range(h // p):
            g = hh // (h // hkv)   # the shard's K/V head of its query head hh
            want = O.sdpa_head(qv[s, :, hh * 128:(hh + 1) * 128], kv[s, :, g * 128:(g + 1) * 128],
                               vv[s, :, g * 128:(g + 1) * 128], True)
            err = np.abs(got[s, :, hh * 128:(hh + 1) * 128] - want)
            assert err.max() <= 2.0 ** -8 * (np.abs(vv).max() + 1.0)


def test_dropped_load_in_block_row_layer_times_out(short_timeout):
    """tp_mlp_block on a shape whose row layer runs on CTA pairs, with the
    fold in its epilogue (or beside it): a load the row layer (the call's
    second tensor-core launch) never issues makes its MMA wait run out, the
    layer stops without counting its remaining tiles, and the later shards'
    waits for those regions (or the fold's) run out as well (status bit
    0x80); the next call is correct."""
    rng = np.random.default_rng(3)
    c = W.f32_to_bf16_bits
    T, d, k, p = 1000, 2048, 2048, 4
    inp = W.Inputs(c(rng.standard_normal((T, d), dtype=np.float32)),
                   c(rng.standard_normal((d, k), dtype=np.float32) * 0.02), None, None,
                   c(rng.standard_normal((k, d), dtype=np.float32) * 0.02), None, "bf16")
    blk = DeviceBlock(inp, T, d, k, p, "gelu_tanh")
    assert tp.tp_sync_status(check=False) == 0
    tp.tp_debug_drop_load(3, 1)
    blk.block()
    st = tp.tp_sync_status(check=False)
    assert st == 6, tp.tp_status_string(st)
    word = int(re.search(r"status bits 0x([0-9a-f]+)", tp.tp_last_error_detail()).group(1), 16)
    assert word & 0x1, hex(word)
    if region_fold_enabled():
        assert word & 0x80, hex(word)
    blk.Z.fill_(float("nan"))
    blk.block()
    assert tp.tp_sync_status(check=False) == 0
    ref = O.mlp_sharded(inp.values("X")[:64], inp.values("W1"), None, inp.values("W2"), None, p,
                        "gelu_tanh")["Z"]
    assert O.rel_err(host_f32(blk.Z)[:64], ref) <= 1e-2
