"""Pins for the LayerNorm, residual fold and transformer-block part of the
oracle: PyTorch's layer_norm (float64, CPU), closed forms of the
normalisation, the unsharded block against the sharded one, special cases
with zero weights, and planted mistakes."""

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import tp_oracle as O


def check_layer_norm_matches_library():
    rng = np.random.default_rng(0)
    for (T, d) in [(5, 16), (3, 768), (7, 33)]:
        x = rng.standard_normal((T, d)) * 3.0 + 1.5
        g = rng.standard_normal(d)
        b = rng.standard_normal(d)
        want = F.layer_norm(torch.from_numpy(x), (d,), torch.from_numpy(g), torch.from_numpy(b),
                            eps=1e-5).numpy()
        assert O.rel_err(O.layer_norm(x, g, b, 1e-5), want) < 1e-13


def check_layer_norm_closed_forms():
    rng = np.random.default_rng(1)
    d, eps = 64, 1e-5
    x = rng.standard_normal((4, d)) * 2.0 - 0.5
    y = O.layer_norm(x, np.ones(d), np.zeros(d), eps)
    var = x.var(axis=1)
    # unit gain, zero bias: every row has mean 0 and mean square var/(var+eps)
    assert np.allclose(y.mean(1), 0.0, atol=1e-14)
    assert np.allclose((y * y).mean(1), var / (var + eps), rtol=1e-13)
    # a constant row normalises to zero, so the output is the bias
    beta = rng.standard_normal(d)
    yc = O.layer_norm(np.full((1, d), 7.25), rng.standard_normal(d), beta, eps)
    assert np.array_equal(yc[0], beta)
    # two-valued row {-a, +a}: variance a^2 exactly, output +-a/sqrt(a^2+eps)
    a = 3.0
    row = np.array([[-a, a] * (d // 2)])
    y2 = O.layer_norm(row, np.ones(d), np.zeros(d), eps)
    assert np.allclose(np.abs(y2), a / np.sqrt(a * a + eps), rtol=1e-15)


def _params(rng, d, h, hkv, dh, k, act, bias=True, scale=0.1):
    def r(*shape):
        return rng.standard_normal(shape) * scale
    return {"ln1_gamma": 1.0 + r(d), "ln1_beta": r(d), "Wq": r(d, h * dh), "Wk": r(d, hkv * dh),
            "Wv": r(d, hkv * dh), "Wo": r(h * dh, d), "bo": r(d) if bias else None,
            "ln2_gamma": 1.0 + r(d), "ln2_beta": r(d), "W1": r(d, k),
            "W_up": r(d, k) if act == "swiglu" else None, "b1": r(k) if bias else None,
            "W2": r(k, d), "b2": r(d) if bias else None}


def check_block_sharded_matches_unsharded():
    rng = np.random.default_rng(2)
    T, d, dh = 9, 32, 4
    for (h, hkv, k, act, causal) in [(4, 4, 64, "gelu_tanh", True), (4, 2, 48, "swiglu", False)]:
        prm = _params(rng, d, h, hkv, dh, k, act)
        X = rng.standard_normal((T, d)).astype(np.float32)
        want = O.transformer_block_unsharded(X, prm, h, hkv, dh, act, causal)
        for p in (1, 2):
            got = O.transformer_block_sharded(X, prm, p, h, hkv, dh, act, causal)["out"]
            assert O.rel_err(got, want) < 1e-6, (h, hkv, act, p)


def check_block_zero_weights_is_residual_plus_biases():
    """With zero output projections both blocks reduce to their biases, so
    out = (X + bo) + b2 in float32, exactly."""
    rng = np.random.default_rng(3)
    T, d, h, dh, k = 6, 16, 2, 4, 32
    prm = _params(rng, d, h, h, dh, k, "gelu_tanh")
    prm["Wo"] = np.zeros_like(prm["Wo"])
    prm["W2"] = np.zeros_like(prm["W2"])
    for key in ("bo", "b2"):
        prm[key] = prm[key].astype(np.float32)
    X = rng.standard_normal((T, d)).astype(np.float32)
    out = O.transformer_block_sharded(X, prm, 2, h, h, dh, "gelu_tanh", True)
    H = np.add(np.float32(0.0) + prm["bo"][None, :], X, dtype=np.float32)
    assert np.array_equal(out["H"], H)
    assert np.array_equal(out["out"], np.add(prm["b2"][None, :], H, dtype=np.float32))


def check_residual_fold_order():
    """Partials, then bias, then residual, in float32: with P = [1], b = 1 and
    residual 2^24, (1 + 1) + 2^24 = 2^24 + 2 is exact, whereas adding the
    residual first would give (1 + 2^24) + 1 = 2^24 (each step rounds the
    tie to even)."""
    P = np.array([[[1.0]]], dtype=np.float32)
    b = np.array([1.0], dtype=np.float32)
    R = np.array([[2.0 ** 24]], dtype=np.float32)
    assert O.reduce_partials_fixed_order(P, b, R)[0, 0] == np.float32(2.0 ** 24 + 2.0)
    # and the p partials come before the bias: P = [2^24, 1, 1], b = 0
    P3 = np.array([[[2.0 ** 24]], [[1.0]], [[1.0]]], dtype=np.float32)
    assert O.reduce_partials_fixed_order(P3, None, None)[0, 0] == np.float32(2.0 ** 24)


BLOCK_PINS = [check_layer_norm_matches_library, check_layer_norm_closed_forms,
              check_block_sharded_matches_unsharded, check_block_zero_weights_is_residual_plus_biases,
              check_residual_fold_order]


@pytest.mark.parametrize("pin", BLOCK_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _mut_ln_unbiased(X, gamma, beta, eps=1e-5):
    x = np.asarray(X, dtype=np.float64)
    c = x - x.mean(1, keepdims=True)
    var = (c * c).sum(1, keepdims=True) / (x.shape[1] - 1)
    return c / np.sqrt(var + eps) * np.asarray(gamma)[None, :] + np.asarray(beta)[None, :]


def _mut_ln_eps_outside(X, gamma, beta, eps=1e-5):
    x = np.asarray(X, dtype=np.float64)
    c = x - x.mean(1, keepdims=True)
    var = (c * c).mean(1, keepdims=True)
    return c / (np.sqrt(var) + eps) * np.asarray(gamma)[None, :] + np.asarray(beta)[None, :]


_orig_reduce = O.reduce_partials_fixed_order


def _mut_fold_drops_residual(P, b2=None, residual=None):
    return _orig_reduce(P, b2, None)


def _mut_fold_residual_first(P, b2=None, residual=None):
    parts = [np.asarray(x) for x in P]
    acc = parts[0].copy()
    if residual is not None:
        acc = np.add(acc, residual, dtype=np.float32)
    for x in parts[1:]:
        acc = np.add(acc, x, dtype=np.float32)
    if b2 is not None:
        acc = np.add(acc, np.asarray(b2)[None, :], dtype=np.float32)
    return acc


_orig_attn = O.attention_sharded


def _mut_attention_ignores_mask(X, Wq, Wk, Wv, Wo, bo, p, n_heads, n_kv_heads, head_dim, causal,
                                hidden_round=None):
    return _orig_attn(X, Wq, Wk, Wv, Wo, bo, p, n_heads, n_kv_heads, head_dim, False, hidden_round)


MUTATIONS = {
    "layer_norm_unbiased_variance": ("layer_norm", _mut_ln_unbiased),
    "layer_norm_eps_outside_sqrt": ("layer_norm", _mut_ln_eps_outside),
    "fold_drops_residual": ("reduce_partials_fixed_order", _mut_fold_drops_residual),
    "fold_adds_residual_first": ("reduce_partials_fixed_order", _mut_fold_residual_first),
    "sharded_attention_ignores_mask": ("attention_sharded", _mut_attention_ignores_mask),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in BLOCK_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, TypeError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} was not caught"
