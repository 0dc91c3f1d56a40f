"""GPU parity of the fixed-order partial-sum reduction (the on-device
stand-in for the all-reduce): bit-exact against the oracle's float32 left
fold of the same seeded partials."""

import json
import os

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
from oracle import tp_oracle as O
import workloads as W
from gpu_util import bits, dev

pytestmark = pytest.mark.gpu

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _run(P, b2):
    p, T, d = P.shape
    Pd = dev(P)
    bd = dev(b2)
    Z = torch.full((T, d), float("nan"), device="cuda")
    tp.tp_reduce_partials(Pd, bd, Z, T, d, p)
    tp.tp_sync_status()
    return Z.cpu().numpy()


@pytest.mark.parametrize("p", [1, 2, 3, 4, 5, 8, 11])
@pytest.mark.parametrize("T,d", [(1, 4), (3, 100), (37, 768), (129, 4100), (2, 6)])
@pytest.mark.parametrize("with_bias", [False, True])
def test_reduce_bit_exact(p, T, d, with_bias):
    P = W.random_partials(p, T, d, seed=1000 * p + T + d)
    b2 = W.random_partials(1, 1, d, seed=7)[0, 0] if with_bias else None
    got = _run(P, b2)
    want = O.reduce_partials_fixed_order(P, b2)
    assert np.array_equal(bits(got), bits(want))


def test_reduce_golden_cases():
    g = json.load(open(os.path.join(GOLDEN, "fold_order.json")))
    for c in g["cases"]:
        p = len(c["partials"])
        P = np.tile(np.array(c["partials"], dtype=np.float32).reshape(p, 1, 1), (1, 3, 4))
        b2 = None if c["b2"] is None else np.full(4, c["b2"], dtype=np.float32)
        got = _run(P, b2)
        want = np.full((3, 4), c["expected"], dtype=np.float32)
        assert np.array_equal(bits(got), bits(want)), c["name"]


def test_reduce_scalar_path_unaligned():
    """Buffers that are not 16-byte aligned take the scalar kernel; same bits."""
    p, T, d = 3, 5, 7
    P = W.random_partials(p, T, d, seed=3)
    b2 = W.random_partials(1, 1, d, seed=4)[0, 0]
    buf = torch.empty(p * T * d + 1, device="cuda")
    buf[1:] = dev(P).reshape(-1)
    zbuf = torch.empty(T * d + 1, device="cuda")
    bbuf = torch.empty(d + 1, device="cuda")
    bbuf[1:] = dev(b2)
    tp.tp_reduce_partials(buf[1:], bbuf[1:], zbuf[1:], T, d, p)
    tp.tp_sync_status()
    want = O.reduce_partials_fixed_order(P, b2)
    assert np.array_equal(bits(zbuf[1:].cpu().numpy().reshape(T, d)), bits(want))


def test_reduce_full_size_llama_shape():
    """p = 8 partials of the Llama-shaped prefill, [8][4096][8192] fp32."""
    p, T, d = 8, 4096, 8192
    P = W.random_partials(p, T, d, seed=99)
    got = _run(P, None)
    want = O.reduce_partials_fixed_order(P, None)
    assert np.array_equal(bits(got), bits(want))


def test_reduce_is_reproducible():
    P = W.random_partials(4, 300, 1000, seed=5)
    a = _run(P, None)
    b = _run(P, None)
    assert np.array_equal(bits(a), bits(b))
