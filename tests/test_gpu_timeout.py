"""Bounded device waits: a load the producer never issues makes the consumer's
wait run out; the kernel records TP_ERR_DEVICE_TIMEOUT, stops every role of
the CTA, frees its TMEM and returns, and the context stays usable.  The fault
is injected on the host (tp_debug_drop_load: the next tensor-core launch skips
one pipeline slot) -- nothing traps or faults."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
from oracle import tp_oracle as O
import workloads as W
from gpu_util import DeviceBlock, host_f32

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
    even CTA's MMA wait runs out, both CTAs of every pair stop, meet at the
    cluster barrier and free their TMEM."""
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

