"""Pins for the backward pass in the oracle: PyTorch autograd in float64 on
the plain block (a library route), central finite differences on tiny
inputs, closed-form activation derivatives, the sharded gradients against
the unsharded ones, and planted mistakes."""

import math

import numpy as np
import pytest
import torch

from oracle import tp_oracle as O


def _torch_grads(X, W1, b1, W2, b2, dZ, act, W_up=None):
    t = {n: torch.tensor(v, dtype=torch.float64, requires_grad=True)
         for n, v in (("X", X), ("W1", W1), ("b1", b1), ("W2", W2), ("b2", b2), ("W_up", W_up))
         if v is not None}
    H = t["X"] @ t["W1"] + (t["b1"] if "b1" in t else 0.0)
    if act == "gelu_tanh":
        Y = torch.nn.functional.gelu(H, approximate="tanh")
    elif act == "relu":
        Y = torch.relu(H)
    elif act == "identity":
        Y = H
    else:
        Y = torch.nn.functional.silu(H) * (t["X"] @ t["W_up"])
    Z = Y @ t["W2"] + (t["b2"] if "b2" in t else 0.0)
    Z.backward(torch.tensor(dZ, dtype=torch.float64))
    return {n: v.grad.numpy() for n, v in t.items()}


def check_unsharded_matches_autograd():
    rng = np.random.default_rng(0)
    T, d, k = 7, 12, 20
    for act in ("gelu_tanh", "swiglu", "relu", "identity"):
        X = rng.standard_normal((T, d))
        W1, W2 = rng.standard_normal((d, k)) * 0.3, rng.standard_normal((k, d)) * 0.3
        Wu = rng.standard_normal((d, k)) * 0.3 if act == "swiglu" else None
        b1, b2 = rng.standard_normal(k) * 0.1, rng.standard_normal(d) * 0.1
        dZ = rng.standard_normal((T, d))
        got = O.mlp_backward_unsharded(X, W1, b1, W2, dZ, act, W_up=Wu)
        want = _torch_grads(X, W1, b1, W2, b2, dZ, act, Wu)
        for mine, theirs in (("dX", "X"), ("dW1", "W1"), ("db1", "b1"), ("dW2", "W2"),
                             ("db2", "b2")):
            assert O.rel_err(got[mine], want[theirs]) < 1e-12, (act, mine)
        if Wu is not None:
            assert O.rel_err(got["dW_up"], want["W_up"]) < 1e-12


def check_finite_differences():
    """Central differences of L = sum(dZ * Z) on a tiny block, float64."""
    rng = np.random.default_rng(1)
    T, d, k = 3, 4, 6
    X = rng.standard_normal((T, d))
    W1, W2 = rng.standard_normal((d, k)) * 0.5, rng.standard_normal((k, d)) * 0.5
    b1 = rng.standard_normal(k) * 0.1
    dZ = rng.standard_normal((T, d))
    for act in ("gelu_tanh", "swiglu"):
        Wu = rng.standard_normal((d, k)) * 0.5 if act == "swiglu" else None
        g = O.mlp_backward_unsharded(X, W1, b1, W2, dZ, act, W_up=Wu)

        def loss(X_=X, W1_=W1, b1_=b1, W2_=W2, Wu_=Wu):
            return float(np.sum(dZ * O.mlp_unsharded(X_, W1_, b1_, W2_, None, act, W_up=Wu_)))

        eps = 1e-6
        for name, arr in (("dX", X), ("dW1", W1), ("db1", b1), ("dW2", W2)):
            num = np.zeros_like(arr)
            for idx in np.ndindex(arr.shape):
                plus, minus = arr.copy(), arr.copy()
                plus[idx] += eps
                minus[idx] -= eps
                key = {"dX": "X_", "dW1": "W1_", "db1": "b1_", "dW2": "W2_"}[name]
                num[idx] = (loss(**{key: plus}) - loss(**{key: minus})) / (2 * eps)
            assert np.allclose(g[name], num, rtol=1e-6, atol=1e-7), (act, name)


def check_activation_derivative_closed_forms():
    assert O.gelu_tanh_grad(np.array([0.0]))[0] == 0.5
    assert O.silu_grad(np.array([0.0]))[0] == 0.5
    # far tails: GELU' -> 1 and 0, SiLU' -> 1 and 0
    assert abs(O.gelu_tanh_grad(np.array([30.0]))[0] - 1.0) < 1e-15
    assert abs(O.gelu_tanh_grad(np.array([-30.0]))[0]) < 1e-15
    assert abs(O.silu_grad(np.array([40.0]))[0] - 1.0) < 1e-15
    # SiLU'(x) = s(x) + x s(x)(1 - s(x)); at x = ln 3, s = 3/4
    x = math.log(3.0)
    assert abs(O.silu_grad(np.array([x]))[0] - (0.75 + x * 0.75 * 0.25)) < 1e-15
    # identity and ReLU backward
    dY = np.array([[1.5, -2.0, 3.0]])
    h = np.array([[-1.0, 0.5, 2.0]])
    assert np.array_equal(O.activation_backward("relu", dY, h)[0], np.array([[0.0, -2.0, 3.0]]))
    assert np.array_equal(O.activation_backward("identity", dY, h)[0], dY)


def check_sharded_matches_unsharded():
    """Shard by shard (dZ replicated by g's identity backward, local
    activation backward, local weight gradients, dX folded from p partials)
    reproduces the plain gradients."""
    rng = np.random.default_rng(2)
    T, d, k = 9, 16, 32
    for act in ("gelu_tanh", "swiglu"):
        X = rng.standard_normal((T, d))
        W1, W2 = rng.standard_normal((d, k)) * 0.3, rng.standard_normal((k, d)) * 0.3
        Wu = rng.standard_normal((d, k)) * 0.3 if act == "swiglu" else None
        b1 = rng.standard_normal(k) * 0.1
        dZ = rng.standard_normal((T, d))
        want = O.mlp_backward_unsharded(X, W1, b1, W2, dZ, act, W_up=Wu)
        for p in (1, 2, 4):
            got = O.mlp_backward_sharded(X, W1, b1, W2, dZ, p, act, W_up=Wu)
            for name in ("dW1", "db1", "dW2", "db2"):
                assert O.rel_err(got[name], want[name]) < 1e-12, (act, p, name)
            assert O.rel_err(got["dX"], want["dX"]) < 1e-6
            assert O.rel_err(got["dX_partials"].astype(np.float64).sum(0), want["dX"]) < 1e-6
            if Wu is not None:
                assert O.rel_err(got["dW_up"], want["dW_up"]) < 1e-12


BACKWARD_PINS = [check_unsharded_matches_autograd, check_finite_differences,
                 check_activation_derivative_closed_forms, check_sharded_matches_unsharded]


@pytest.mark.parametrize("pin", BACKWARD_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _mut_gelu_grad_no_cubic_factor(h):
    h = np.asarray(h, dtype=np.float64)
    t = np.tanh(math.sqrt(2 / math.pi) * (h + 0.044715 * h ** 3))
    du = math.sqrt(2 / math.pi) * (1.0 + 0.044715 * h * h)
    return 0.5 * (1.0 + t) + 0.5 * h * (1.0 - t * t) * du


def _mut_silu_grad_sigmoid_only(h):
    h = np.asarray(h, dtype=np.float64)
    return 1.0 / (1.0 + np.exp(-h))


_orig_act_bwd = O.activation_backward


def _mut_swiglu_up_grad_from_gate(act, dY, h, up=None):
    dH, dU = _orig_act_bwd(act, dY, h, up)
    if dU is not None:
        dU = np.asarray(dY, dtype=np.float64) * np.asarray(h, dtype=np.float64)
    return dH, dU


_orig_sharded_bwd = O.mlp_backward_sharded


def _mut_dx_drops_last_shard(X, W1, b1, W2, dZ, p, act, W_up=None, hidden_round=None):
    out = _orig_sharded_bwd(X, W1, b1, W2, dZ, p, act, W_up, hidden_round)
    if p > 1:
        out["dX"] = O.reduce_partials_fixed_order(out["dX_partials"][:-1])
    return out


MUTATIONS = {
    "gelu_grad_without_3x_cubic_factor": ("gelu_tanh_grad", _mut_gelu_grad_no_cubic_factor),
    "silu_grad_is_sigmoid": ("silu_grad", _mut_silu_grad_sigmoid_only),
    "swiglu_up_grad_uses_gate": ("activation_backward", _mut_swiglu_up_grad_from_gate),
    "dx_fold_drops_a_shard": ("mlp_backward_sharded", _mut_dx_drops_last_shard),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in BACKWARD_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, TypeError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} was not caught"
