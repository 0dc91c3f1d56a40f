"""GPU parity of the fp32 path (plain fp32 FMA, no TF32) against the oracle:
max|gpu - oracle| / max|oracle| <= 1e-5, and bit-exact on small-integer
inputs where every intermediate is an exact integer."""

import numpy as np
import pytest

import megatron_tensor_sharded_b200 as tp
from oracle import tp_oracle as O
import workloads as W
from gpu_util import DeviceBlock, bits, host_f32

pytestmark = pytest.mark.gpu

TOL_F32 = 1e-5


def _oracle(inp, p, act):
    return O.mlp_sharded(inp.values("X"), inp.values("W1"), inp.values("b1"), inp.values("W2"),
                         inp.values("b2"), p, act, W_up=inp.values("W_up"))


def test_toy_config_the_pages_shape():
    """X[4,512], W1[512,2048], b1[2048], W2[2048,512], p = 4, GELU(tanh),
    seed 42 drawn as on the day-41 walkthrough."""
    w = W.WORKLOADS["toy"]
    inp = W.make_inputs(w)
    ref = _oracle(inp, w.p, w.act)
    blk = DeviceBlock(inp, w.T, w.d, w.k, w.p, w.act)
    blk.column()
    blk.row()
    blk.reduce()
    blk.sync()
    Y = host_f32(blk.Y)
    for i in range(w.p):
        assert O.rel_err(Y[i], ref["Y"][i]) <= TOL_F32, i
    assert O.rel_err(host_f32(blk.P), ref["P"]) <= TOL_F32
    assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_F32
    # the concatenated column shards are the unsharded first layer
    h = inp.values("X").astype(np.float64) @ inp.values("W1").astype(np.float64) + inp.values("b1")
    assert O.rel_err(np.concatenate(list(Y), axis=1), O.gelu_tanh(h)) <= TOL_F32
    for flags in (tp.TP_FLAG_NONE, tp.TP_FLAG_SPLITK_FUSED):
        blk.Z.fill_(float("nan"))
        blk.block(flags)
        blk.sync()
        assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_F32, flags


@pytest.mark.parametrize("T,d,k,p", [(1, 1, 1, 1), (2, 3, 4, 2), (3, 8, 16, 4), (3, 5, 8, 2),
                                     (70, 33, 132, 3), (65, 130, 192, 4)])
@pytest.mark.parametrize("act", ["identity", "relu"])
def test_small_integer_inputs_bit_exact(T, d, k, p, act):
    inp = W.small_integer_inputs(T, d, k, seed=T * 31 + d, act=act)
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
    for flags in (tp.TP_FLAG_NONE, tp.TP_FLAG_SPLITK_FUSED):
        blk.Z.fill_(float("nan"))
        blk.block(flags)
        blk.sync()
        assert np.array_equal(bits(host_f32(blk.Z)), bits(ref["Z"])), flags


@pytest.mark.parametrize("p", [1, 2, 4])
def test_swiglu_f32(p):
    rng = np.random.default_rng(p)
    T, d, k = 37, 96, 256
    inp = W.Inputs(rng.standard_normal((T, d), dtype=np.float32),
                   (rng.standard_normal((d, k), dtype=np.float32) * 0.1),
                   (rng.standard_normal((d, k), dtype=np.float32) * 0.1),
                   None, (rng.standard_normal((k, d), dtype=np.float32) * 0.1),
                   rng.standard_normal(d, dtype=np.float32), "f32")
    ref = _oracle(inp, p, "swiglu")
    blk = DeviceBlock(inp, T, d, k, p, "swiglu")
    blk.block()
    blk.sync()
    assert O.rel_err(host_f32(blk.Z), ref["Z"]) <= TOL_F32
    blk.column()
    blk.sync()
    Y = host_f32(blk.Y)
    for i in range(p):
        assert O.rel_err(Y[i], ref["Y"][i]) <= TOL_F32
