"""The attention softmax's fast 2^x (a fitted degree-4 polynomial on the FMA
pipe, used for part of the probabilities) checked directly against float64
2^x on a dense grid over [-126, 0], at integers and half-integers (where the
range reduction switches), next to them, and at the clamp.

Bound: the polynomial's fitted relative error on [-1/2, 1/2] is 2.6e-6;
evaluating it in fp32 (four FMAs, the exponent added exactly) adds at most
a few fp32 roundings, so every point must be within 2.6e-6 + 3 * 2^-24
(about 2.78e-6) of 2^x.  Below -126 the input is clamped: the result is the
one at -126 (the probabilities are bf16, for which 2^-126 and 0 agree)."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp

pytestmark = pytest.mark.gpu

BOUND = 2.6e-6 + 3 * 2.0 ** -24


def _run(x: np.ndarray) -> np.ndarray:
    xd = torch.from_numpy(np.ascontiguousarray(x, dtype=np.float32)).cuda()
    yd = torch.full_like(xd, float("nan"))
    tp.tp_debug_exp2_poly(xd, yd, xd.numel())
    tp.tp_sync_status()
    return yd.cpu().numpy()


def _grid() -> np.ndarray:
    ints = np.arange(-126, 1, dtype=np.float32)
    halves = (np.arange(-126, 0) + 0.5).astype(np.float32)
    pts = [np.linspace(-126.0, 0.0, 4_000_001, dtype=np.float32), ints, halves]
    for a in (ints, halves):
        pts.append(np.nextafter(a, np.float32(1.0)))
        pts.append(np.nextafter(a, np.float32(-200.0)))
    x = np.concatenate(pts)
    return x[(x >= -126.0) & (x <= 0.0)]


def test_relative_error_on_minus_126_to_0():
    x = _grid()
    y = _run(x).astype(np.float64)
    want = np.exp2(x.astype(np.float64))
    rel = np.abs(y - want) / want
    worst = int(np.argmax(rel))
    assert rel[worst] <= BOUND, (float(x[worst]), float(rel[worst]))
    assert y[-1] > 0 and np.all(np.isfinite(y))


def test_one_step_of_the_exponent_halves_the_result():
    # 2^(x - 1) is exactly half of 2^x: the polynomial sees only the
    # distance to the nearest integer, which x and x - 1 share (x is a
    # multiple of 2^-12 and never a half-integer, so x - 1 is exact and both
    # round to neighbouring integers): checks the exponent step
    x = (-(4 * np.arange(600, 100000, 3) + 1) / 4096.0).astype(np.float32)
    y = _run(np.concatenate([x, x - np.float32(1.0)]))
    a, b = y[:x.size], y[x.size:]
    assert np.array_equal(b * np.float32(2.0), a)


def test_clamp_below_minus_126():
    x = np.array([-126.0, -126.25, -126.49, -127.0, -150.0, -1e30, -np.inf], dtype=np.float32)
    y = _run(x)
    assert np.all(y == y[0]), y
    assert abs(float(y[0]) / 2.0 ** -126 - 1.0) <= BOUND


def test_odd_length_tail_and_empty():
    x = np.array([-1.0, -2.0, -3.0], dtype=np.float32)
    y = _run(x)
    assert np.all(np.abs(y / np.exp2(x.astype(np.float64)) - 1.0) <= BOUND)
    z = torch.zeros(1, device="cuda")
    assert tp.tp_debug_exp2_poly(z, z, 0) == 0
    assert tp.tp_debug_exp2_poly(z, z, -1, check=False) == 1
