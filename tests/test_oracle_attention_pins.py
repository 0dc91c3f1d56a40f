"""Pins for the tensor-parallel attention part of the oracle, against what
the pages and the mathematics fix: PyTorch's scaled_dot_product_attention
(float64, CPU) for the unsharded case, closed forms of softmax attention,
head counts and shard shapes printed on the pages, and planted mistakes."""

import math

import numpy as np
import pytest
import torch
import torch.nn.functional as F

from oracle import tp_oracle as O


def _weights(rng, d, h, hkv, dh, scale=0.2):
    return (rng.standard_normal((d, h * dh)) * scale, rng.standard_normal((d, hkv * dh)) * scale,
            rng.standard_normal((d, hkv * dh)) * scale, rng.standard_normal((h * dh, d)) * scale)


def _torch_reference(X, Wq, Wk, Wv, Wo, bo, h, hkv, dh, causal):
    """Library route: project with F.linear, expand grouped K/V heads, run
    F.scaled_dot_product_attention, project out."""
    tX = torch.from_numpy(X)
    q = F.linear(tX, torch.from_numpy(Wq).T).view(-1, h, dh).transpose(0, 1)
    k = F.linear(tX, torch.from_numpy(Wk).T).view(-1, hkv, dh).transpose(0, 1)
    v = F.linear(tX, torch.from_numpy(Wv).T).view(-1, hkv, dh).transpose(0, 1)
    k = k.repeat_interleave(h // hkv, dim=0)
    v = v.repeat_interleave(h // hkv, dim=0)
    o = F.scaled_dot_product_attention(q, k, v, is_causal=causal)
    o = o.transpose(0, 1).reshape(-1, h * dh)
    z = F.linear(o, torch.from_numpy(Wo).T, None if bo is None else torch.from_numpy(bo))
    return z.numpy()


def check_unsharded_matches_library():
    rng = np.random.default_rng(0)
    for (T, d, h, hkv, dh) in [(9, 16, 4, 4, 4), (13, 24, 6, 2, 8), (5, 8, 2, 1, 4)]:
        X = rng.standard_normal((T, d))
        Wq, Wk, Wv, Wo = _weights(rng, d, h, hkv, dh)
        bo = rng.standard_normal(d)
        for causal in (False, True):
            got = O.attention_unsharded(X, Wq, Wk, Wv, Wo, bo, h, hkv, dh, causal)
            want = _torch_reference(X, Wq, Wk, Wv, Wo, bo, h, hkv, dh, causal)
            assert O.rel_err(got, want) < 1e-12, (T, h, hkv, causal)


def check_sharded_matches_unsharded():
    """Summing the per-shard head groups' partials reproduces the plain block
    ("Tensor parallel math": attention heads are independent; W_O row blocks
    sum)."""
    rng = np.random.default_rng(1)
    T, d, dh = 11, 32, 4
    for (h, hkv) in [(8, 8), (8, 4), (8, 2)]:
        X = rng.standard_normal((T, d))
        Wq, Wk, Wv, Wo = _weights(rng, d, h, hkv, dh)
        for causal in (False, True):
            want = O.attention_unsharded(X, Wq, Wk, Wv, Wo, None, h, hkv, dh, causal)
            for p in (1, 2):
                if hkv % p:
                    continue
                out = O.attention_sharded(X, Wq, Wk, Wv, Wo, None, p, h, hkv, dh, causal)
                assert O.rel_err(out["Z"], want) < 1e-6, (h, hkv, p, causal)
                assert len(out["O"]) == p and out["O"][0].shape == (T, h // p * dh)
                # the P partials sum (in float64) to the unsharded result
                assert O.rel_err(out["P"].astype(np.float64).sum(0), want) < 1e-6


def check_closed_forms():
    rng = np.random.default_rng(2)
    T, dh = 7, 4
    v = rng.standard_normal((T, dh))
    q = rng.standard_normal((T, dh))
    # identical keys: uniform weights, every output row is the mean of V
    k_same = np.tile(rng.standard_normal((1, dh)), (T, 1))
    out = O.sdpa_head(q, k_same, v, causal=False)
    assert np.allclose(out, np.tile(v.mean(0), (T, 1)), rtol=0, atol=1e-14)
    # causal: the first query sees only key 0, so its output is V[0]
    k = rng.standard_normal((T, dh))
    out = O.sdpa_head(q, k, v, causal=True)
    assert np.allclose(out[0], v[0], rtol=0, atol=1e-15)
    # one key: output is that value row
    out = O.sdpa_head(q, k[:1], v[:1], causal=False)
    assert np.allclose(out, np.tile(v[:1], (T, 1)), rtol=0, atol=1e-15)
    # two keys with scores 0 and s: weights 1/(1+e^s) and e^s/(1+e^s)
    qq = np.array([[1.0, 0.0, 0.0, 0.0]])
    kk = np.array([[0.0, 0.0, 0.0, 0.0], [math.log(3.0) * 2.0, 0.0, 0.0, 0.0]])  # score ln3
    vv = np.array([[4.0, 0, 0, 0], [8.0, 0, 0, 0]])
    out = O.sdpa_head(qq, kk, vv, causal=False)
    assert abs(out[0, 0] - (4.0 * 0.25 + 8.0 * 0.75)) < 1e-14


def check_head_shards_from_the_pages():
    # Part 9, "Splitting the Attention Layer": 32 heads of 128 on 4 GPUs -> each
    # GPU's QKV columns [4096, 3 x 1024] and W_out rows [1024, 4096]
    hq = O.heads_per_shard(32, 4)
    assert hq * 128 == 1024
    Wq = np.zeros((4096, 32 * 128), dtype=np.float32)
    assert O._column_slice(Wq, 3, hq * 128).shape == (4096, 1024)
    Wo = np.zeros((32 * 128, 4096), dtype=np.float32)
    assert O._row_slice(Wo, 3, hq * 128).shape == (1024, 4096)
    # aquanode worked example: 64 query heads / 8 = 8, 8 key/value heads / 8 = 1
    assert O.heads_per_shard(64, 8) == 8 and O.heads_per_shard(8, 8) == 1
    # "Tensor Parallelism Explained" section 2.A: 64 heads at TP=4 -> 16 per GPU
    assert O.heads_per_shard(64, 4) == 16
    # section 4 failure mode: 64 heads cannot be split over 5
    with pytest.raises(ValueError, match="divisible"):
        O.heads_per_shard(64, 5)


ATTN_PINS = [check_unsharded_matches_library, check_sharded_matches_unsharded, check_closed_forms,
             check_head_shards_from_the_pages]


@pytest.mark.parametrize("pin", ATTN_PINS, ids=lambda f: f.__name__)
def test_pin(pin):
    pin()


def _mut_sdpa_no_scale(q, k, v, causal):
    q = np.asarray(q, dtype=np.float64)
    s = q @ np.asarray(k, dtype=np.float64).T
    if causal:
        s = np.where(np.arange(s.shape[1])[None, :] > np.arange(s.shape[0])[:, None], -np.inf, s)
    w = np.exp(s - s.max(1, keepdims=True))
    return (w / w.sum(1, keepdims=True)) @ np.asarray(v, dtype=np.float64)


def _mut_sdpa_causal_off_by_one(q, k, v, causal):
    q = np.asarray(q, dtype=np.float64)
    s = q @ np.asarray(k, dtype=np.float64).T / math.sqrt(q.shape[1])
    if causal:
        s = np.where(np.arange(s.shape[1])[None, :] >= np.arange(s.shape[0])[:, None] + 2, -np.inf, s)
    w = np.exp(s - s.max(1, keepdims=True))
    return (w / w.sum(1, keepdims=True)) @ np.asarray(v, dtype=np.float64)


_orig_sharded = O.attention_sharded
_orig_unsharded = O.attention_unsharded


def _mut_gqa_modulo(X, Wq, Wk, Wv, Wo, bo, n_heads, n_kv_heads, head_dim, causal):
    X64 = np.asarray(X, dtype=np.float64)
    Q, K, V = X64 @ Wq, X64 @ Wk, X64 @ Wv
    outs = []
    for h in range(n_heads):
        g = h % n_kv_heads
        outs.append(O.sdpa_head(Q[:, h * head_dim:(h + 1) * head_dim], K[:, g * head_dim:(g + 1) * head_dim],
                                V[:, g * head_dim:(g + 1) * head_dim], causal))
    Z = np.concatenate(outs, 1) @ Wo
    return Z + (0 if bo is None else bo)


MUTATIONS = {
    "attention_without_sqrt_dk": ("sdpa_head", _mut_sdpa_no_scale),
    "causal_mask_off_by_one": ("sdpa_head", _mut_sdpa_causal_off_by_one),
    "kv_head_map_modulo": ("attention_unsharded", _mut_gqa_modulo),
}


@pytest.mark.parametrize("name", sorted(MUTATIONS))
def test_planted_mistakes_are_caught(name, monkeypatch):
    attr, fn = MUTATIONS[name]
    monkeypatch.setattr(O, attr, fn)
    failed = []
    for pin in ATTN_PINS:
        try:
            pin()
        except (AssertionError, ValueError, IndexError):
            failed.append(pin.__name__)
    assert failed, f"planted mistake {name} was not caught"
