"""CPU oracle for the Megatron tensor-parallel MLP block.

TEST INFRASTRUCTURE ONLY.  Nothing in the product path may import, call or
execute this module: only the tests, the smoke check and the bench's CPU
baseline arm use it.  It shares no code with the CUDA library.

What it computes, and where the pages state it:

* Column-parallel linear -- W [d, k] is cut by output columns into p slices
  W_i = W[:, i*s:(i+1)*s], s = k/p; every shard sees the whole X and forms
  Y_i = act(X W_i + b_i) with no communication.  (skandtandon.pages.dev day-41
  post, "Simulating column parallel linear"; "Tensor parallel math",
  "Column-parallel: split the weight by output columns"; "Tensor Parallelism
  Explained", section 1.A.)
* Row-parallel linear -- W' [k, d] is cut by input rows into W'_i =
  W'[i*s:(i+1)*s, :]; shard i consumes Y_i and emits a full-shape partial
  Z_i = Y_i W'_i [T, d].  (day-41 post, "Simulating row parallel linear";
  "Tensor parallel math", "Row-parallel: split the weight by input rows";
  "Tensor Parallelism Explained", section 1.B.)
* The all-reduce -- Z = sum_i Z_i; the output bias is added once, after the
  sum.  On one device this is a fixed-order fp32 fold (day-41 post,
  ``sum(partial_sums) + bias``; "Building GPT from Scratch -- Part 9",
  "Implementation Sketch", RowParallelLinear.forward).
* Tensor-parallel attention -- QKV projections column-parallel by heads,
  attention local to each shard's heads, row-parallel output projection,
  one reduction (day-41 post, "Attention heads: naturally parallel";
  "Tensor parallel math", "Attention: parallel across heads"; "Tensor
  Parallelism Explained", section 2.A; "Building GPT from Scratch -- Part 9",
  "Splitting the Attention Layer").  Grouped key/value heads (the aquanode
  Llama worked example: 64 query heads, 8 key/value heads, 1 per GPU at
  TP = 8) are supported; the mask is optional (the pages write the plain
  softmax(Q K^T / sqrt(d_k)) V).
* The transformer block -- LayerNorm, attention block, residual add,
  LayerNorm, MLP block, residual add: two reductions per layer, the
  residual added in each fold ("Building GPT from Scratch -- Part 9",
  "Communication Pattern per Transformer Block"; "Tensor parallel math",
  "Counting all-reduces").  Pre-norm order as the diagram draws it.
* The Megatron MLP pairing -- column-parallel first layer, element-wise
  activation applied per shard, row-parallel second layer, one reduction
  ("Tensor parallel math", "The MLP block: column then row, one all-reduce";
  day-41 post, "Pairing them: the Megatron-LM MLP").  SwiGLU variant:
  Swish(X W_gate,i) * (X W_up,i) per shard, W_down row-parallel
  ("Tensor Parallelism Explained", section 2.B).

Readings taken where the pages are silent (each also listed in the design
notes): GELU is the tanh form 0.5 h (1 + tanh(sqrt(2/pi) (h + 0.044715 h^3)))
(Hendrycks & Gimpel); Swish is SiLU, h / (1 + e^-h); weights are stored
[in, out] row-major (Y = X W); the fixed-order reduction is a left fold that
starts from Z_0 (not from 0.0) and adds the bias last.

Precision: every product and sum is taken in float64 from the exact input
values; partials are rounded once to float32; the fold is float32
round-to-nearest-even, one addition at a time.  A library matmul (numpy's
float64 ``@``) serves as the dot-product step.
"""

from __future__ import annotations

import math
from typing import List, Optional, Sequence

import numpy as np

ACTIVATIONS = ("gelu_tanh", "swiglu", "identity", "relu")

_SQRT_2_OVER_PI = math.sqrt(2.0 / math.pi)


# --------------------------------------------------------------------------
# element-wise activations (applied locally on each shard)
# --------------------------------------------------------------------------

def gelu_tanh(h: np.ndarray) -> np.ndarray:
    """GELU, tanh form, in float64."""
    h = np.asarray(h, dtype=np.float64)
    return 0.5 * h * (1.0 + np.tanh(_SQRT_2_OVER_PI * (h + 0.044715 * h * h * h)))


def silu(h: np.ndarray) -> np.ndarray:
    """Swish with beta = 1 (SiLU), h / (1 + e^-h), in float64."""
    h = np.asarray(h, dtype=np.float64)
    with np.errstate(over="ignore"):
        return h / (1.0 + np.exp(-h))


def relu(h: np.ndarray) -> np.ndarray:
    """max(0, h): the day-41 walkthrough's activation 'for simplicity'."""
    return np.maximum(0.0, np.asarray(h, dtype=np.float64))


def apply_activation(act: str, h: np.ndarray, up: Optional[np.ndarray] = None) -> np.ndarray:
    """act(h); for SwiGLU ``h`` is the gate pre-activation X W_gate and ``up``
    is X W_up."""
    if act == "gelu_tanh":
        return gelu_tanh(h)
    if act == "relu":
        return relu(h)
    if act == "identity":
        return np.asarray(h, dtype=np.float64)
    if act == "swiglu":
        if up is None:
            raise ValueError("swiglu needs the up projection")
        return silu(h) * np.asarray(up, dtype=np.float64)
    raise ValueError(f"unknown activation {act!r}")


# --------------------------------------------------------------------------
# the plain (unsharded) block: the definition the sharded method must reach
# --------------------------------------------------------------------------

def _f64(a):
    return None if a is None else np.asarray(a, dtype=np.float64)


def mlp_unsharded(X, W1, b1, W2, b2, act: str, W_up=None) -> np.ndarray:
    """Z = act(X W1 + b1) W2 + b2 in float64, no sharding at all.

    For SwiGLU, W1 is W_gate and Z = (SiLU(X W_gate) * (X W_up)) W_down.
    Returns the unrounded float64 result."""
    X, W1, W2 = _f64(X), _f64(W1), _f64(W2)
    H = X @ W1
    if b1 is not None:
        H = H + _f64(b1)[None, :]
    U = None
    if act == "swiglu":
        U = X @ _f64(W_up)
    Y = apply_activation(act, H, U)
    Z = Y @ W2
    if b2 is not None:
        Z = Z + _f64(b2)[None, :]
    return Z


# --------------------------------------------------------------------------
# the sharded method, written separately, one shard at a time
# --------------------------------------------------------------------------

def shard_width(k: int, p: int) -> int:
    """s = k/p; the walkthrough asserts divisibility before slicing."""
    if p < 1:
        raise ValueError("p must be >= 1")
    if k % p != 0:
        raise ValueError(f"{k} features cannot be split evenly over {p} shards")
    return k // p


def _column_slice(W: np.ndarray, i: int, s: int) -> np.ndarray:
    """Shard i's column block of an [in, out] weight: W[:, i*s:(i+1)*s]."""
    return W[:, i * s:(i + 1) * s]


def _vector_slice(b: np.ndarray, i: int, s: int) -> np.ndarray:
    return b[i * s:(i + 1) * s]


def _row_slice(W: np.ndarray, i: int, s: int) -> np.ndarray:
    """Shard i's row block of a [k, d] weight: W[i*s:(i+1)*s, :]."""
    return W[i * s:(i + 1) * s, :]


def column_parallel_linear(X, W1, b1, p: int, act: str, W_up=None) -> List[np.ndarray]:
    """Per-shard Y_i = act(X W1_i + b1_i), i = 0..p-1, each [T, s], float64.

    The activation runs on each shard's slice alone, as the pairing allows
    (it is element-wise)."""
    k = np.shape(W1)[1]
    s = shard_width(k, p)
    X64 = _f64(X)
    out = []
    for i in range(p):
        Wi = np.asarray(_column_slice(W1, i, s), dtype=np.float64)
        Hi = X64 @ Wi
        if b1 is not None:
            Hi = Hi + np.asarray(_vector_slice(b1, i, s), dtype=np.float64)[None, :]
        Ui = None
        if act == "swiglu":
            Ui = X64 @ np.asarray(_column_slice(W_up, i, s), dtype=np.float64)
        out.append(apply_activation(act, Hi, Ui))
    return out


def row_parallel_partials(Y_shards: Sequence[np.ndarray], W2, p: int) -> List[np.ndarray]:
    """Per-shard full-shape partials Z_i = Y_i W2_i, each [T, d], float64."""
    if len(Y_shards) != p:
        raise ValueError("need one hidden shard per partition")
    k = np.shape(W2)[0]
    s = shard_width(k, p)
    out = []
    for i in range(p):
        W2i = np.asarray(_row_slice(W2, i, s), dtype=np.float64)
        out.append(np.asarray(Y_shards[i], dtype=np.float64) @ W2i)
    return out


def reduce_partials_fixed_order(P: np.ndarray, b2: Optional[np.ndarray] = None,
                                residual: Optional[np.ndarray] = None) -> np.ndarray:
    """Z = ((P_0 + P_1) + ...) + P_{p-1}  [+ b2]  [+ residual], every
    addition a single float32 round-to-nearest-even operation, shard index
    ascending, the bias after the partials and the residual stream last (the
    transformer block's "residual connection (element-wise add)" after each
    reduced block; "Building GPT from Scratch -- Part 9", "Communication
    Pattern per Transformer Block").

    ``P`` is float32 [p][T][d] (or a sequence of [T][d] float32 arrays);
    ``b2`` is float32 [d] or None; ``residual`` float32 [T][d] or None.
    Returns float32 [T][d]."""
    parts = [np.asarray(x) for x in P]
    for x in parts:
        if x.dtype != np.float32:
            raise TypeError("partials must be float32")
    acc = parts[0].copy()
    for x in parts[1:]:
        acc = np.add(acc, x, dtype=np.float32)
    if b2 is not None:
        b = np.asarray(b2)
        if b.dtype != np.float32:
            raise TypeError("b2 must be float32")
        acc = np.add(acc, b[None, :], dtype=np.float32)
    if residual is not None:
        r = np.asarray(residual)
        if r.dtype != np.float32:
            raise TypeError("residual must be float32")
        acc = np.add(acc, r, dtype=np.float32)
    return acc


def round_to_bf16(x: np.ndarray) -> np.ndarray:
    """Round float64 values to the nearest bf16 value (8 significant bits,
    ties to even), returned as float64.  Used for the device-faithful mode,
    where the hidden shards are stored as bf16 between the two layers."""
    x = np.asarray(x, dtype=np.float64)
    m, e = np.frexp(x)                      # x = m * 2**e, 0.5 <= |m| < 1
    return np.ldexp(np.rint(m * 256.0), e - 8)


def mlp_sharded(X, W1, b1, W2, b2, p: int, act: str, W_up=None,
                hidden_round: Optional[str] = None) -> dict:
    """The whole method on p simulated shards.

    Returns a dict with
      ``Y``  -- list of p float64 hidden shards [T, s] (after the optional
                storage rounding),
      ``P``  -- float32 partials [p, T, d] (each rounded once from float64),
      ``Z``  -- float32 result of the fixed-order fold (+ b2 last).

    ``hidden_round`` = None keeps Y unrounded; "bf16" or "f32" rounds each
    hidden shard to that storage type before the row-parallel layer."""
    Y = column_parallel_linear(X, W1, b1, p, act, W_up)
    if hidden_round == "bf16":
        Y = [round_to_bf16(y) for y in Y]
    elif hidden_round == "f32":
        Y = [y.astype(np.float32).astype(np.float64) for y in Y]
    elif hidden_round is not None:
        raise ValueError(hidden_round)
    P64 = row_parallel_partials(Y, W2, p)
    P = np.stack([x.astype(np.float32) for x in P64])
    b2_32 = None if b2 is None else np.asarray(b2, dtype=np.float32)
    Z = reduce_partials_fixed_order(P, b2_32)
    return {"Y": Y, "P": P, "Z": Z}


def rel_err(got: np.ndarray, want: np.ndarray) -> float:
    """max|got - want| / max|want| (the parity measure for float results)."""
    got = np.asarray(got, dtype=np.float64)
    want = np.asarray(want, dtype=np.float64)
    den = float(np.max(np.abs(want))) if want.size else 0.0
    num = float(np.max(np.abs(got - want))) if want.size else 0.0
    if den == 0.0:
        return num
    return num / den


# --------------------------------------------------------------------------
# tensor-parallel attention block (column-parallel QKV by heads, local
# attention per head, row-parallel output projection, one reduction)
# --------------------------------------------------------------------------

def heads_per_shard(n_heads: int, p: int) -> int:
    """h/p heads on every shard; the head count must divide evenly ("Tensor
    Parallelism Explained", section 4, head-divisibility failure mode; day-41
    post, "Attention heads: naturally parallel")."""
    if p < 1:
        raise ValueError("p must be >= 1")
    if n_heads % p != 0:
        raise ValueError(f"number of attention heads ({n_heads}) must be divisible by "
                         f"tensor_parallel_size ({p})")
    return n_heads // p


def sdpa_head(q: np.ndarray, k: np.ndarray, v: np.ndarray, causal: bool) -> np.ndarray:
    """softmax(q k^T / sqrt(d_k)) v for one head, float64 ("Tensor parallel
    math", "Attention: parallel across heads").  q [T, dh], k/v [S, dh].
    With `causal`, query t sees keys 0..t only."""
    q = np.asarray(q, dtype=np.float64)
    k = np.asarray(k, dtype=np.float64)
    v = np.asarray(v, dtype=np.float64)
    scores = (q @ k.T) / math.sqrt(q.shape[1])
    if causal:
        T, S = scores.shape
        mask = np.arange(S)[None, :] > np.arange(T)[:, None]
        scores = np.where(mask, -np.inf, scores)
    scores = scores - np.max(scores, axis=1, keepdims=True)
    w = np.exp(scores)
    w = w / np.sum(w, axis=1, keepdims=True)
    return w @ v


def attention_unsharded(X, Wq, Wk, Wv, Wo, bo, n_heads: int, n_kv_heads: int, head_dim: int,
                        causal: bool) -> np.ndarray:
    """Plain multi-head attention with grouped key/value heads, float64:
    Z = concat_h softmax(Q_h K_g(h)^T / sqrt(dh)) V_g(h) @ Wo + bo, where query
    head h uses key/value head g(h) = h // (n_heads / n_kv_heads).  Weights
    [in, out]: Wq [d, n_heads*dh], Wk/Wv [d, n_kv_heads*dh], Wo [n_heads*dh, d]."""
    X64 = _f64(X)
    Q = X64 @ _f64(Wq)
    K = X64 @ _f64(Wk)
    V = X64 @ _f64(Wv)
    group = n_heads // n_kv_heads
    outs = []
    for h in range(n_heads):
        g = h // group
        outs.append(sdpa_head(Q[:, h * head_dim:(h + 1) * head_dim],
                              K[:, g * head_dim:(g + 1) * head_dim],
                              V[:, g * head_dim:(g + 1) * head_dim], causal))
    Z = np.concatenate(outs, axis=1) @ _f64(Wo)
    if bo is not None:
        Z = Z + _f64(bo)[None, :]
    return Z


def attention_sharded(X, Wq, Wk, Wv, Wo, bo, p: int, n_heads: int, n_kv_heads: int,
                      head_dim: int, causal: bool, hidden_round: Optional[str] = None) -> dict:
    """The attention block on p simulated shards, written shard by shard:
    shard i takes query heads [i*h/p, (i+1)*h/p) and key/value heads
    [i*hkv/p, (i+1)*hkv/p) -- column blocks of Wq, Wk, Wv -- runs attention
    on them locally, and multiplies by its row block of Wo; the partials are
    folded in shard order (float32), bias last (day-41 post, "Attention
    heads: naturally parallel"; "Building GPT from Scratch -- Part 9",
    TensorParallelAttention).

    Returns Q, K, V shards (float64, as the column layer produces them), the
    attention outputs O_i [T, h/p*dh] (optionally rounded to bf16 storage),
    float32 partials P [p, T, d] and the float32 result Z."""
    hq = heads_per_shard(n_heads, p)
    hkv = heads_per_shard(n_kv_heads, p)
    if n_heads % n_kv_heads != 0:
        raise ValueError("n_heads must be a multiple of n_kv_heads")
    group = n_heads // n_kv_heads
    X64 = _f64(X)
    Qs, Ks, Vs, Os, Ps = [], [], [], [], []
    for i in range(p):
        Qi = X64 @ np.asarray(_column_slice(Wq, i, hq * head_dim), dtype=np.float64)
        Ki = X64 @ np.asarray(_column_slice(Wk, i, hkv * head_dim), dtype=np.float64)
        Vi = X64 @ np.asarray(_column_slice(Wv, i, hkv * head_dim), dtype=np.float64)
        if hidden_round == "bf16":
            Qi, Ki, Vi = round_to_bf16(Qi), round_to_bf16(Ki), round_to_bf16(Vi)
        heads = []
        for hh in range(hq):
            g = hh // group
            heads.append(sdpa_head(Qi[:, hh * head_dim:(hh + 1) * head_dim],
                                   Ki[:, g * head_dim:(g + 1) * head_dim],
                                   Vi[:, g * head_dim:(g + 1) * head_dim], causal))
        Oi = np.concatenate(heads, axis=1)
        if hidden_round == "bf16":
            Oi = round_to_bf16(Oi)
        Wo_i = np.asarray(_row_slice(Wo, i, hq * head_dim), dtype=np.float64)
        Ps.append((Oi @ Wo_i).astype(np.float32))
        Qs.append(Qi); Ks.append(Ki); Vs.append(Vi); Os.append(Oi)
    P = np.stack(Ps)
    bo32 = None if bo is None else np.asarray(bo, dtype=np.float32)
    Z = reduce_partials_fixed_order(P, bo32)
    return {"Q": Qs, "K": Ks, "V": Vs, "O": Os, "P": P, "Z": Z}


# --------------------------------------------------------------------------
# the tensor-parallel transformer block: LayerNorm -> attention (one
# reduction) -> residual -> LayerNorm -> MLP (one reduction) -> residual
# --------------------------------------------------------------------------

def layer_norm(X, gamma, beta, eps: float = 1e-5) -> np.ndarray:
    """Per row of X [T, d]: (x - mean) / sqrt(var + eps) * gamma + beta, with
    the biased (divide by d) variance, float64.  The pages only name the
    step ("LayerNorm (replicated, no communication)", "Building GPT from
    Scratch -- Part 9", "Communication Pattern per Transformer Block"); this
    is the standard layer normalisation (Ba, Kiros & Hinton) with a learned
    gain and bias."""
    x = _f64(X)
    mean = x.mean(axis=1, keepdims=True)
    c = x - mean
    var = (c * c).mean(axis=1, keepdims=True)
    y = c / np.sqrt(var + eps)
    return y * _f64(gamma)[None, :] + _f64(beta)[None, :]


def transformer_block_unsharded(X, prm: dict, n_heads: int, n_kv_heads: int, head_dim: int,
                                act: str, causal: bool, eps: float = 1e-5) -> np.ndarray:
    """Pre-norm block, float64: H = X + Attn(LN1(X)); out = H + MLP(LN2(H)).
    ``prm`` holds ln1_gamma, ln1_beta, Wq, Wk, Wv, Wo, bo, ln2_gamma, ln2_beta, W1, W_up, b1,
    W2, b2 (bo, W_up, b1, b2 may be None)."""
    X64 = _f64(X)
    a = layer_norm(X64, prm["ln1_gamma"], prm["ln1_beta"], eps)
    H = X64 + attention_unsharded(a, prm["Wq"], prm["Wk"], prm["Wv"], prm["Wo"], prm["bo"],
                                  n_heads, n_kv_heads, head_dim, causal)
    m = layer_norm(H, prm["ln2_gamma"], prm["ln2_beta"], eps)
    return H + mlp_unsharded(m, prm["W1"], prm["b1"], prm["W2"], prm["b2"], act,
                             W_up=prm.get("W_up"))


def transformer_block_sharded(X, prm: dict, p: int, n_heads: int, n_kv_heads: int, head_dim: int,
                              act: str, causal: bool, eps: float = 1e-5,
                              hidden_round: Optional[str] = None) -> dict:
    """The block on p simulated shards: the attention and MLP blocks each end
    in one fixed-order float32 fold, with the residual stream added in that
    fold (two reductions per layer; "Building GPT from Scratch -- Part 9",
    "Communication Pattern per Transformer Block"; "Tensor parallel math",
    "Counting all-reduces").  The residual stream X, H, out is float32.
    With ``hidden_round == "bf16"`` every tensor a GEMM reads (the LayerNorm
    outputs, Q, K, V, the attention output, the MLP hidden shards) is
    rounded to bf16, as the device stores them.

    Returns LN1 output ``A``, ``H`` (float32), LN2 output ``M`` and ``out``
    (float32)."""
    X32 = np.asarray(X, dtype=np.float32)
    A = layer_norm(X32, prm["ln1_gamma"], prm["ln1_beta"], eps)
    if hidden_round == "bf16":
        A = round_to_bf16(A)
    att = attention_sharded(A, prm["Wq"], prm["Wk"], prm["Wv"], prm["Wo"], None, p, n_heads,
                            n_kv_heads, head_dim, causal, hidden_round=hidden_round)
    bo = None if prm["bo"] is None else np.asarray(prm["bo"], dtype=np.float32)
    H = reduce_partials_fixed_order(att["P"], bo, residual=X32)
    M = layer_norm(H, prm["ln2_gamma"], prm["ln2_beta"], eps)
    if hidden_round == "bf16":
        M = round_to_bf16(M)
    mlp = mlp_sharded(M, prm["W1"], prm["b1"], prm["W2"], None, p, act, W_up=prm.get("W_up"),
                      hidden_round=hidden_round)
    b2 = None if prm["b2"] is None else np.asarray(prm["b2"], dtype=np.float32)
    out = reduce_partials_fixed_order(mlp["P"], b2, residual=H)
    return {"A": A, "H": H, "M": M, "out": out}


# --------------------------------------------------------------------------
# backward pass of the MLP block: the f / g conjugate operators ("Tensor
# parallel math", "The f and g conjugate operators"; "Counting all-reduces":
# one all-reduce per block in the backward pass as well)
# --------------------------------------------------------------------------

def gelu_tanh_grad(h: np.ndarray) -> np.ndarray:
    """d/dh of the tanh-form GELU, float64:
    0.5 (1 + tanh u) + 0.5 h (1 - tanh^2 u) sqrt(2/pi) (1 + 3 * 0.044715 h^2),
    u = sqrt(2/pi) (h + 0.044715 h^3)."""
    h = np.asarray(h, dtype=np.float64)
    t = np.tanh(_SQRT_2_OVER_PI * (h + 0.044715 * h * h * h))
    du = _SQRT_2_OVER_PI * (1.0 + 3.0 * 0.044715 * h * h)
    return 0.5 * (1.0 + t) + 0.5 * h * (1.0 - t * t) * du


def silu_grad(h: np.ndarray) -> np.ndarray:
    """d/dh of h * sigma(h): sigma(h) (1 + h (1 - sigma(h))), float64."""
    h = np.asarray(h, dtype=np.float64)
    with np.errstate(over="ignore"):
        sg = 1.0 / (1.0 + np.exp(-h))
    return sg * (1.0 + h * (1.0 - sg))


def activation_backward(act: str, dY, h, up=None):
    """Gradient through the element-wise activation: returns (dH, dUp) where
    dUp is None except for SwiGLU (Y = SiLU(h) * up)."""
    dY = np.asarray(dY, dtype=np.float64)
    h = np.asarray(h, dtype=np.float64)
    if act == "gelu_tanh":
        return dY * gelu_tanh_grad(h), None
    if act == "relu":
        return dY * (h > 0.0), None
    if act == "identity":
        return dY.copy(), None
    if act == "swiglu":
        u = np.asarray(up, dtype=np.float64)
        return dY * u * silu_grad(h), dY * silu(h)
    raise ValueError(f"unknown activation {act!r}")


def mlp_backward_unsharded(X, W1, b1, W2, dZ, act: str, W_up=None) -> dict:
    """Gradients of Z = act(X W1 + b1) W2 + b2 for the upstream gradient dZ,
    float64, no sharding: dX, dW1, dW_up (SwiGLU), db1, dW2, db2."""
    X, W1, W2, dZ = _f64(X), _f64(W1), _f64(W2), _f64(dZ)
    H = X @ W1
    if b1 is not None:
        H = H + _f64(b1)[None, :]
    U = X @ _f64(W_up) if act == "swiglu" else None
    Y = apply_activation(act, H, U)
    dY = dZ @ W2.T
    dH, dU = activation_backward(act, dY, H, U)
    out = {"dW2": Y.T @ dZ, "db2": dZ.sum(axis=0), "dW1": X.T @ dH, "db1": dH.sum(axis=0),
           "dX": dH @ W1.T, "dW_up": None}
    if dU is not None:
        out["dW_up"] = X.T @ dU
        out["dX"] = out["dX"] + dU @ _f64(W_up).T
    return out


def mlp_backward_sharded(X, W1, b1, W2, dZ, p: int, act: str, W_up=None,
                         hidden_round: Optional[str] = None) -> dict:
    """The backward pass on p simulated shards, shard by shard.

    g (after the row-parallel layer) is the identity backward: every shard
    receives the whole dZ.  Shard i forms dY_i = dZ W2_i^T, goes back through
    its activation locally (dH_i), and computes its own weight gradients
    dW2_i = Y_i^T dZ, dW1_i = X^T dH_i, db1_i = sum_t dH_i -- no
    communication.  f (before the column-parallel layer) is the all-reduce
    backward: the input gradient dX = sum_i dH_i W1_i^T (+ dU_i W_up,i^T) is
    a sum of full-shape partials, folded in shard order in float32 ("Tensor
    parallel math", "The f and g conjugate operators").  db2 belongs to the
    replicated bias: sum_t dZ, once.

    ``hidden_round == "bf16"`` rounds what the device stores in bf16: the
    pre-activations H_i (and up projections), the activations Y_i and dH_i
    (and dU_i).  Returns per-shard lists and the assembled gradients:
    dW1 [d, k], dW_up, db1 [k], dW2 [k, d], db2 [d] (float64), the dX partials
    (float32 [p, T, d]) and dX (float32 fold)."""
    rnd = round_to_bf16 if hidden_round == "bf16" else (lambda a: a)
    if hidden_round not in (None, "bf16"):
        raise ValueError(hidden_round)
    k = np.shape(W1)[1]
    s = shard_width(k, p)
    X64, dZ64 = _f64(X), _f64(dZ)
    dW1, dWu, db1, dW2, parts = [], [], [], [], []
    for i in range(p):
        W1i = np.asarray(_column_slice(W1, i, s), dtype=np.float64)
        Hi = X64 @ W1i
        if b1 is not None:
            Hi = Hi + np.asarray(_vector_slice(b1, i, s), dtype=np.float64)[None, :]
        Ui = Wui = None
        if act == "swiglu":
            Wui = np.asarray(_column_slice(W_up, i, s), dtype=np.float64)
            Ui = X64 @ Wui
        Yi = rnd(apply_activation(act, Hi, Ui))
        Hi = rnd(Hi)
        Ui = None if Ui is None else rnd(Ui)
        W2i = np.asarray(_row_slice(W2, i, s), dtype=np.float64)
        dYi = dZ64 @ W2i.T
        dHi, dUi = activation_backward(act, dYi, Hi, Ui)
        dHi = rnd(dHi)
        dUi = None if dUi is None else rnd(dUi)
        dW2.append(Yi.T @ dZ64)
        dW1.append(X64.T @ dHi)
        db1.append(dHi.sum(axis=0))
        part = dHi @ W1i.T
        if dUi is not None:
            dWu.append(X64.T @ dUi)
            part = part + dUi @ Wui.T
        parts.append(part.astype(np.float32))
    P = np.stack(parts)
    return {"dW1": np.concatenate(dW1, axis=1), "db1": np.concatenate(db1),
            "dW_up": np.concatenate(dWu, axis=1) if dWu else None,
            "dW2": np.concatenate(dW2, axis=0), "db2": dZ64.sum(axis=0),
            "dX_partials": P, "dX": reduce_partials_fixed_order(P)}
