"""Pins for the CPU oracle, against what the pages and the mathematics fix.

Each ``check_*`` function raises AssertionError when the oracle disagrees with
an outside fact (a value printed on a page, a hand-worked example, a closed
form, a library routine for a special case, brute force on tiny inputs).  The
tests call them as they are; ``test_planted_mistakes_are_caught`` plants
plausible mistakes in the oracle (on the CPU) and checks that some pin fails.
"""

import json
import math
import os

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from oracle import tp_oracle as O
import workloads as W

GOLDEN = os.path.join(os.path.dirname(__file__), "golden")


def _golden(name):
    with open(os.path.join(GOLDEN, name)) as f:
        return json.load(f)


# --------------------------------------------------------------------------
# the pins
# --------------------------------------------------------------------------

def check_page_column_concat():
    """Day-41 post worked example: concat of the 4 column shards equals the
    unsharded x@W+b with max error 0.00e+00; and both agree with the page's
    own float32 computation within the float32 dot-product error bound."""
    g = _golden("column_concat_seed42.json")
    x, Wm, b = W.toy_page_example(g["seed"])
    assert x.shape == (g["batch"], g["in_features"])
    assert Wm.shape == (g["in_features"], g["out_features"])
    ys = O.column_parallel_linear(x, Wm, b, g["num_gpus"], "identity")
    assert all(y.shape == (g["batch"], g["slice_size"]) for y in ys)
    ycat = np.concatenate(ys, axis=1)
    # the unsharded first layer: the plain block with identity activation and
    # W2 = I (multiplying by the identity matrix is exact in float64)
    full = O.mlp_unsharded(x, Wm, b, np.eye(g["out_features"]), None, "identity")
    assert float(np.max(np.abs(ycat - full))) == g["max_error"]
    # the page's float32 numbers: |fp32 - exact| <= gamma_K * sum|x||w| + u|b|
    y32 = (x @ Wm + b).astype(np.float64)
    K = g["in_features"]
    u = 2.0 ** -24
    gamma = (K + 1) * u / (1 - (K + 1) * u)
    bound = gamma * (np.abs(x).astype(np.float64) @ np.abs(Wm).astype(np.float64)
                     + np.abs(b).astype(np.float64)[None, :])
    assert np.all(np.abs(ycat - y32) <= bound)


def check_shard_shapes():
    g = _golden("shard_shapes.json")
    for c in g["cases"]:
        T, d, k, p = c["T"], c["d"], c["k"], c["p"]
        s = O.shard_width(k, p)
        assert [d, s] == c["column_shard"]
        assert [s, d] == c["row_shard"]
        rng = np.random.default_rng(0)
        # shapes only: tiny values, the real sizes of the column/row blocks
        Wsl = O._column_slice(np.empty((d, k), dtype=np.float32), p - 1, s)
        assert list(Wsl.shape) == c["column_shard"]
        Rsl = O._row_slice(np.empty((k, d), dtype=np.float32), p - 1, s)
        assert list(Rsl.shape) == c["row_shard"]
        if T * d * k <= 1 << 26:
            X = rng.standard_normal((T, d))
            Wt = rng.standard_normal((d, k)) * 0.01
            Ys = O.column_parallel_linear(X, Wt, None, p, "identity")
            assert [list(y.shape) for y in Ys] == [c["hidden_shard"]] * p
            Ps = O.row_parallel_partials(Ys, rng.standard_normal((k, d)) * 0.01, p)
            assert [list(x.shape) for x in Ps] == [c["partial"]] * p
    for c in g["indivisible"]:
        with pytest.raises(ValueError):
            O.shard_width(c["k"], c["p"])


def check_tiny_block_by_hand():
    g = _golden("tiny_block_by_hand.json")
    X = np.array(g["X"], dtype=np.float32)
    W1 = np.array(g["W1"], dtype=np.float32)
    b1 = np.array(g["b1"], dtype=np.float32)
    W2 = np.array(g["W2"], dtype=np.float32)
    b2 = np.array(g["b2"], dtype=np.float32)
    for act in ("relu", "identity"):
        out = O.mlp_sharded(X, W1, b1, W2, b2, g["p"], act)
        want = g[act]
        for i in range(g["p"]):
            assert np.array_equal(out["Y"][i], np.array(want["Y"][i], dtype=np.float64)), (act, i)
            assert np.array_equal(out["P"][i], np.array(want["P"][i], dtype=np.float32)), (act, i)
        assert np.array_equal(out["Z"], np.array(want["Z"], dtype=np.float32)), act
        assert np.array_equal(O.mlp_unsharded(X, W1, b1, W2, b2, act),
                              np.array(want["Z"], dtype=np.float64)), act


def check_fold_order():
    g = _golden("fold_order.json")
    for c in g["cases"]:
        P = np.array(c["partials"], dtype=np.float32).reshape(len(c["partials"]), 1, 1)
        b2 = None if c["b2"] is None else np.array([c["b2"]], dtype=np.float32)
        z = O.reduce_partials_fixed_order(P, b2)
        assert z.dtype == np.float32
        got = float(z[0, 0])
        assert got == c["expected"], c["name"]
        assert math.copysign(1.0, got) == math.copysign(1.0, c["expected"]), c["name"]


def _brute_force_block(X, W1, b1, W2, b2, p, act):
    """Pure-Python loops straight from the walkthrough's three steps."""
    T, d = len(X), len(X[0])
    k = len(W1[0])
    s = k // p
    partials = []
    for i in range(p):
        Yi = [[0.0] * s for _ in range(T)]
        for t in range(T):
            for j in range(s):
                h = float(b1[i * s + j]) if b1 is not None else 0.0
                for c in range(d):
                    h += float(X[t][c]) * float(W1[c][i * s + j])
                Yi[t][j] = max(0.0, h) if act == "relu" else h
        Pi = [[0.0] * d for _ in range(T)]
        for t in range(T):
            for n in range(d):
                acc = 0.0
                for j in range(s):
                    acc += Yi[t][j] * float(W2[i * s + j][n])
                Pi[t][n] = acc
        partials.append(Pi)
    Z = [[0.0] * d for _ in range(T)]
    for t in range(T):
        for n in range(d):
            z = sum(partials[i][t][n] for i in range(p))
            Z[t][n] = z + (float(b2[n]) if b2 is not None else 0.0)
    return np.array(partials), np.array(Z)


def check_brute_force_tiny():
    """Small-integer inputs: every value is an exact integer, so the oracle
    must equal the brute-force loops bit for bit, for several p."""
    for (T, d, k, seed) in [(1, 1, 1, 0), (2, 3, 4, 1), (3, 8, 16, 2), (3, 5, 8, 3)]:
        for p in (1, 2, 4):
            if k % p:
                continue
            for act in ("identity", "relu"):
                inp = W.small_integer_inputs(T, d, k, seed, act=act)
                out = O.mlp_sharded(inp.X, inp.W1, inp.b1, inp.W2, inp.b2, p, act)
                P_bf, Z_bf = _brute_force_block(inp.X.tolist(), inp.W1.tolist(), inp.b1.tolist(),
                                                inp.W2.tolist(), inp.b2.tolist(), p, act)
                assert np.array_equal(out["P"].astype(np.float64), P_bf), (T, d, k, p, act)
                assert np.array_equal(out["Z"].astype(np.float64), Z_bf), (T, d, k, p, act)


def check_closed_form_identity():
    """Identity activation: sum_i X W_i W'_i = X (W W') ('Tensor Parallelism
    Explained', section 1.B); with biases, Z = X (W1 W2) + b1 W2 + b2."""
    rng = np.random.default_rng(7)
    T, d, k = 5, 24, 48
    X = rng.standard_normal((T, d))
    W1 = rng.standard_normal((d, k))
    b1 = rng.standard_normal(k)
    W2 = rng.standard_normal((k, d))
    b2 = rng.standard_normal(d)
    closed = X @ (W1 @ W2) + (b1 @ W2)[None, :] + b2[None, :]
    for p in (1, 2, 3, 4, 6, 8):
        Y = O.column_parallel_linear(X, W1, b1, p, "identity")
        P = O.row_parallel_partials(Y, W2, p)
        Z = sum(P) + b2[None, :]
        assert O.rel_err(Z, closed) < 1e-12, p
    assert O.rel_err(O.mlp_unsharded(X, W1, b1, W2, b2, "identity"), closed) < 1e-12


def check_activation_values():
    """GELU(tanh) and SiLU against the PyTorch CPU library routines (float64)
    on a grid, plus special values and asymptotes."""
    xs = np.concatenate([np.linspace(-12, 12, 2001), [-60.0, -30.0, 0.0, 30.0, 60.0]])
    tx = torch.from_numpy(xs)
    g_ref = F.gelu(tx, approximate="tanh").numpy()
    s_ref = F.silu(tx).numpy()
    assert np.max(np.abs(O.gelu_tanh(xs) - g_ref)) < 1e-14
    assert np.max(np.abs(O.silu(xs) - s_ref)) < 1e-14
    assert O.gelu_tanh(np.array([0.0]))[0] == 0.0 and O.silu(np.array([0.0]))[0] == 0.0
    assert abs(O.gelu_tanh(np.array([1.0]))[0] - 0.8411919906082768) < 1e-15
    assert abs(O.silu(np.array([1.0]))[0] - 1.0 / (1.0 + math.exp(-1.0))) < 1e-16
    # the tanh form stays within 1e-3 of the exact erf GELU everywhere
    erf_gelu = F.gelu(tx).numpy()
    assert np.max(np.abs(O.gelu_tanh(xs) - erf_gelu)) < 1e-3
    # asymptotes: -> x for large x, -> 0 for very negative x
    assert abs(O.gelu_tanh(np.array([40.0]))[0] - 40.0) < 1e-12
    assert abs(O.silu(np.array([-60.0]))[0]) < 1e-20
    # swiglu = silu(gate) * up
    g, u = np.array([1.5, -2.0]), np.array([3.0, 0.5])
    assert np.allclose(O.apply_activation("swiglu", g, u), s_ref[0] * 0 + F.silu(torch.from_numpy(g)).numpy() * u,
                       rtol=0, atol=1e-15)


def check_p1_is_the_textbook_block():
    """p = 1 is the plain layer ('TP=1 ... functionally identical to the
    original model', Part 9): compare with torch.nn.functional in float64."""
    rng = np.random.default_rng(11)
    T, d, k = 7, 32, 96
    X = rng.standard_normal((T, d))
    W1 = rng.standard_normal((d, k)) * 0.2
    Wu = rng.standard_normal((d, k)) * 0.2
    b1 = rng.standard_normal(k) * 0.2
    W2 = rng.standard_normal((k, d)) * 0.2
    b2 = rng.standard_normal(d) * 0.2
    tX, tW1, tWu, tb1, tW2, tb2 = (torch.from_numpy(a) for a in (X, W1, Wu, b1, W2, b2))
    # nn.Linear stores [out, in]; pass the transpose of our [in, out] weight
    ref_gelu = F.linear(F.gelu(F.linear(tX, tW1.T, tb1), approximate="tanh"), tW2.T, tb2).numpy()
    ref_swiglu = F.linear(F.silu(F.linear(tX, tW1.T)) * F.linear(tX, tWu.T), tW2.T).numpy()
    out = O.mlp_sharded(X, W1, b1, W2, b2, 1, "gelu_tanh")
    assert O.rel_err(out["Z"], ref_gelu) < 1e-6        # Z is float32
    assert O.rel_err(O.mlp_unsharded(X, W1, b1, W2, b2, "gelu_tanh"), ref_gelu) < 1e-13
    out = O.mlp_sharded(X, W1, None, W2, None, 1, "swiglu", W_up=Wu)
    assert O.rel_err(out["Z"], ref_swiglu) < 1e-6
    assert O.rel_err(O.mlp_unsharded(X, W1, None, W2, None, "swiglu", W_up=Wu), ref_swiglu) < 1e-13


def check_sharded_matches_unsharded():
    """Sum over shards of Y_i W2_i equals Y W2 ('Tensor parallel math',
    row-parallel identity), for GELU and SwiGLU and several p."""
    rng = np.random.default_rng(5)
    T, d, k = 6, 40, 120
    X = rng.standard_normal((T, d))
    W1 = rng.standard_normal((d, k)) * 0.3
    Wu = rng.standard_normal((d, k)) * 0.3
    b1 = rng.standard_normal(k) * 0.3
    W2 = rng.standard_normal((k, d)) * 0.3
    for act, wu, bb in (("gelu_tanh", None, b1), ("swiglu", Wu, None), ("relu", None, b1)):
        want = O.mlp_unsharded(X, W1, bb, W2, None, act, W_up=wu)
        for p in (1, 2, 3, 4, 5, 8):
            Y = O.column_parallel_linear(X, W1, bb, p, act, W_up=wu)
            Ycat = np.concatenate(Y, axis=1)
            assert O.rel_err(Ycat, O.apply_activation(act, X @ W1 + (0 if bb is None else bb),
                                                      None if wu is None else X @ wu)) < 1e-13
            Z = sum(O.row_parallel_partials(Y, W2, p))
            assert O.rel_err(Z, want) < 1e-12, (act, p)


def check_rel_err():
    """The parity measure on hand-worked cases: max|got - want| / max|want|,
    with the largest difference and the largest reference element at
    different places, a negative reference maximum, a negative difference,
    a reference whose mean is far below its maximum, an all-zero reference
    (absolute difference) and empty arrays."""
    g = _golden("rel_err_by_hand.json")
    for c in g["cases"]:
        got = np.array(c["got"], dtype=np.float64)
        want = np.array(c["want"], dtype=np.float64)
        expected = c["expected_num"] / c["expected_den"]
        r = O.rel_err(got, want)
        assert isinstance(r, float), c["name"]
        assert r == expected, (c["name"], r, expected)


# --------------------------------------------------------------------------
# tests
# --------------------------------------------------------------------------

PINS = [check_page_column_concat, check_shard_shapes, check_tiny_block_by_hand, check_fold_order,
        check_brute_force_tiny, check_closed_form_identity, check_activation_values,
        check_p1_is_the_textbook_block, check_sharded_matches_unsharded, check_rel_err]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def test_negative_order_activation_on_partial_sums_fails():
    """The pairing must apply the activation before the row-parallel sum:
    GeLU(Z1 + Z2) != GeLU(Z1) + GeLU(Z2) ('Tensor parallel math', 'The MLP
    block').  Sharding the other way round must fail parity."""
    z1, z2 = np.array([1.0]), np.array([1.0])
    assert abs(O.gelu_tanh(z1 + z2)[0] - (O.gelu_tanh(z1) + O.gelu_tanh(z2))[0]) > 0.1
    rng = np.random.default_rng(3)
    T, d, k, p = 4, 16, 32, 4
    X = rng.standard_normal((T, d))
    W1 = rng.standard_normal((d, k))
    W2 = rng.standard_normal((k, d))
    want = O.mlp_unsharded(X, W1, None, W2, None, "gelu_tanh")
    # wrong: row-split the first layer, activate each partial, then sum
    s = k // p
    wrong = 0
    for i in range(p):
        Hi = X[:, i * (d // p):(i + 1) * (d // p)] @ W1[i * (d // p):(i + 1) * (d // p), :]
        wrong = wrong + O.gelu_tanh(Hi)
    wrong = wrong @ W2
    assert O.rel_err(wrong, want) > 1e-2


def test_round_to_bf16_matches_library_on_float32_values():
    rng = np.random.default_rng(1)
    v = np.concatenate([rng.standard_normal(20000).astype(np.float32),
                        np.array([1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8, -1.0 - 2 ** -8, 0.0, 2.0 ** -100], np.float32)])
    ref = torch.from_numpy(v).to(torch.bfloat16).to(torch.float64).numpy()
    assert np.array_equal(O.round_to_bf16(v.astype(np.float64)), ref)


def test_reduce_rejects_non_float32():
    with pytest.raises(TypeError):
        O.reduce_partials_fixed_order(np.zeros((2, 1, 1), dtype=np.float64))


# --------------------------------------------------------------------------
# planted mistakes: each must make at least one pin fail
# --------------------------------------------------------------------------

def _mut_row_slice_uses_columns(W, i, s):
    return W[:, i * s:(i + 1) * s].T if W.shape[1] >= (i + 1) * s else W[i * s:(i + 1) * s, :]


def _mut_row_slice_off_by_one(W, i, s):
    j = (i + 1) % (W.shape[0] // s)
    return W[j * s:(j + 1) * s, :]


def _mut_column_slice_wrong_shard(W, i, s):
    j = (i + 1) % (W.shape[1] // s)
    return W[:, j * s:(j + 1) * s]


def _mut_vector_slice_always_first(b, i, s):
    return b[0:s]


def _mut_gelu_constant(h):
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1.0 + np.tanh(math.sqrt(2.0 / math.pi) * (h + 0.0447 * h ** 3)))


def _mut_gelu_sign(h):
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1.0 - np.tanh(math.sqrt(2.0 / math.pi) * (h + 0.044715 * h ** 3)))


def _mut_silu_sign(h):
    h = np.asarray(h, dtype=np.float64)
    return h / (1.0 + np.exp(h))


_orig_reduce = O.reduce_partials_fixed_order


def _mut_reduce_from_zero(P, b2=None):
    acc = np.zeros_like(np.asarray(P[0]))
    for x in P:
        acc = np.add(acc, x, dtype=np.float32)
    if b2 is not None:
        acc = np.add(acc, np.asarray(b2)[None, :], dtype=np.float32)
    return acc


def _mut_reduce_bias_first(P, b2=None):
    parts = [np.asarray(x) for x in P]
    acc = parts[0].copy()
    if b2 is not None:
        acc = np.add(acc, np.asarray(b2)[None, :], dtype=np.float32)
    for x in parts[1:]:
        acc = np.add(acc, x, dtype=np.float32)
    return acc


def _mut_reduce_reversed(P, b2=None):
    parts = [np.asarray(x) for x in P][::-1]
    acc = parts[0].copy()
    for x in parts[1:]:
        acc = np.add(acc, x, dtype=np.float32)
    if b2 is not None:
        acc = np.add(acc, np.asarray(b2)[None, :], dtype=np.float32)
    return acc


def _mut_reduce_in_float64(P, b2=None):
    acc = np.sum(np.asarray(P, dtype=np.float64), axis=0)
    if b2 is not None:
        acc = acc + np.asarray(b2, dtype=np.float64)[None, :]
    return acc.astype(np.float32)


_orig_apply = O.apply_activation


def _mut_swiglu_swapped(act, h, up=None):
    if act == "swiglu":
        return O.silu(up) * np.asarray(h, dtype=np.float64)
    return _orig_apply(act, h, up)


def _mut_relu_leaky(h):
    h = np.asarray(h, dtype=np.float64)
    return np.where(h > 0, h, 0.01 * h)


def _mut_rel_err_mean_denominator(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if not want.size:
        return 0.0
    den = float(np.mean(np.abs(want)))
    num = float(np.max(np.abs(got - want)))
    return num if den == 0.0 else num / den


def _mut_rel_err_per_element(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if not want.size:
        return 0.0
    diff = np.abs(got - want)
    a = np.abs(want)
    ratio = np.where(a > 0, diff / np.where(a > 0, a, 1.0), diff)
    return float(np.max(ratio))


def _mut_rel_err_signed_max(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if not want.size:
        return 0.0
    den = float(np.max(want))
    num = float(np.max(np.abs(got - want)))
    return num if den == 0.0 else num / den


def _mut_rel_err_no_abs(got, want):
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    if not want.size:
        return 0.0
    den = float(np.max(np.abs(want)))
    num = float(np.max(got - want))
    return num if den == 0.0 else num / den


MUTATIONS = {
    "row_slice_uses_columns": ("_row_slice", _mut_row_slice_uses_columns),
    "row_slice_wrong_shard": ("_row_slice", _mut_row_slice_off_by_one),
    "column_slice_wrong_shard": ("_column_slice", _mut_column_slice_wrong_shard),
    "bias_slice_always_first": ("_vector_slice", _mut_vector_slice_always_first),
    "gelu_constant_typo": ("gelu_tanh", _mut_gelu_constant),
    "gelu_sign": ("gelu_tanh", _mut_gelu_sign),
    "silu_sign": ("silu", _mut_silu_sign),
    "relu_leaky": ("relu", _mut_relu_leaky),
    "reduce_seeded_with_plus_zero": ("reduce_partials_fixed_order", _mut_reduce_from_zero),
    "reduce_bias_first": ("reduce_partials_fixed_order", _mut_reduce_bias_first),
    "reduce_reversed_order": ("reduce_partials_fixed_order", _mut_reduce_reversed),
    "reduce_in_float64": ("reduce_partials_fixed_order", _mut_reduce_in_float64),
    "swiglu_gate_up_swapped": ("apply_activation", _mut_swiglu_swapped),
    "rel_err_mean_denominator": ("rel_err", _mut_rel_err_mean_denominator),
    "rel_err_per_element_ratio": ("rel_err", _mut_rel_err_per_element),
    "rel_err_signed_max": ("rel_err", _mut_rel_err_signed_max),
    "rel_err_abs_missing": ("rel_err", _mut_rel_err_no_abs),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError, TypeError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} was not caught by any pin"
