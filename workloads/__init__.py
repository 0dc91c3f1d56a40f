"""Seeded synthetic inputs for the sharded Megatron MLP block.

This module only draws random numbers and stores them in the element types the
kernels read (fp32, or bf16 held as raw uint16 bit patterns).  It holds none of
the block's arithmetic: no matmul, no activation, no sharding, no reduction.
Both the CPU oracle (through the tests) and the CUDA path read the arrays it
returns, so they see bit-identical inputs.

Workload table (shapes from the worked examples on the pages):

* ``toy``    -- the NumPy walkthrough's own shape: X[4,512], W1[512,2048],
  b1[2048], W2[2048,512], fp32, p=4 (skandtandon.pages.dev day-41 post,
  "Simulating column parallel linear").  Drawn exactly as that example draws
  them: legacy ``np.random.seed(42)`` then ``randn`` for X, W1, b1 (cast to
  float32), followed by W2.
* ``gpt2``   -- GPT-2-small MLP: T=1024, d=768, k=3072, GELU(tanh), p=2,
  biases b1 and b2.
* ``wide``   -- the d=4096 / d_ff=16384 / p=4 / T=4096 worked example
  ("Tensor parallel math", "A worked example"), no bias.
* ``decode`` -- Llama-3.1-70B FFN widths (d=8192, k=28672, p=8, 3584 columns
  per shard; aquanode glossary "Worked example: Llama 3.1 70B on 8 GPUs") at
  T=16 tokens, SwiGLU, no bias.
* ``llama``  -- the same FFN at T=4096 tokens (prefill), SwiGLU, no bias.

bf16 workloads: ``numpy.random.default_rng(seed)`` draws float32 standard
normals in the order X, W1 (W_gate for SwiGLU), W_up, b1, W2 (W_down), b2;
X has std 1, weights and biases std 0.02; values are then rounded to bf16
with round-to-nearest-even.  b2 is kept as fp32 holding bf16-representable
values (the output side of the block is fp32).
"""

from __future__ import annotations

import dataclasses
from typing import Optional

import numpy as np


@dataclasses.dataclass(frozen=True)
class Workload:
    name: str
    T: int          # tokens (rows of X)
    d: int          # model width
    k: int          # FFN width (d_ff)
    p: int          # number of simulated shards
    act: str        # "gelu_tanh" | "swiglu" | "identity" | "relu"
    dtype: str      # "f32" | "bf16"
    has_b1: bool
    has_b2: bool
    description: str

    @property
    def s(self) -> int:
        """Columns per shard, k/p."""
        return self.k // self.p

    def gemm_flops(self) -> int:
        """Algorithmic FLOPs of the two GEMMs (2*T*d*k each; SwiGLU has two
        column-side products)."""
        col = 2 * self.T * self.d * self.k * (2 if self.act == "swiglu" else 1)
        row = 2 * self.T * self.k * self.d
        return col + row


WORKLOADS = {
    "toy": Workload("toy", 4, 512, 2048, 4, "gelu_tanh", "f32", True, False,
                    "fp32 toy: X[4,512] W1[512,2048] b1[2048] W2[2048,512], p=4, GELU(tanh)"),
    "gpt2": Workload("gpt2", 1024, 768, 3072, 2, "gelu_tanh", "bf16", True, True,
                     "GPT-2-small MLP: T=1024 d=768 k=3072 p=2 GELU(tanh) bf16, biases"),
    "wide": Workload("wide", 4096, 4096, 16384, 4, "gelu_tanh", "bf16", False, False,
                     "wide FFN prefill: T=4096 d=4096 k=16384 p=4 GELU(tanh) bf16, no bias"),
    "decode": Workload("decode", 16, 8192, 28672, 8, "swiglu", "bf16", False, False,
                       "decode: T=16 d=8192 k=28672 p=8 SwiGLU bf16, no bias"),
    "llama": Workload("llama", 4096, 8192, 28672, 8, "swiglu", "bf16", False, False,
                      "Llama-70B-shaped SwiGLU prefill: T=4096 d=8192 k=28672 p=8 bf16"),
}


@dataclasses.dataclass(frozen=True)
class AttnWorkload:
    """The tensor-parallel attention block: Q, K, V column-parallel by heads,
    attention per shard, output projection row-parallel, one fold."""
    name: str
    T: int            # tokens (one sequence)
    d: int            # model width
    n_heads: int      # query heads h
    n_kv_heads: int   # key/value heads (h for plain multi-head attention)
    head_dim: int
    p: int
    causal: bool
    description: str

    def flops(self) -> dict:
        """Algorithmic FLOPs: projections 2*T*d*(h + 2*h_kv)*dh and 2*T*h*dh*d;
        attention 4*T*T*h*dh (Q K^T and P V), halved when causal."""
        qkv = 2 * self.T * self.d * (self.n_heads + 2 * self.n_kv_heads) * self.head_dim
        out = 2 * self.T * self.n_heads * self.head_dim * self.d
        attn = 4 * self.T * self.T * self.n_heads * self.head_dim
        if self.causal:
            attn //= 2
        return {"qkv": qkv, "attention": attn, "out": out, "total": qkv + attn + out}


ATTN_WORKLOADS = {
    "attn_wide": AttnWorkload("attn_wide", 4096, 4096, 32, 32, 128, 4, True,
                              "attention block: T=4096 d=4096 32 heads x 128 on p=4 shards "
                              "(8 heads each), causal, bf16"),
    "attn_llama": AttnWorkload("attn_llama", 4096, 8192, 64, 8, 128, 8, True,
                               "grouped-query attention block: T=4096 d=8192 64 query heads, "
                               "8 key/value heads x 128 on p=8 shards, causal, bf16"),
}


@dataclasses.dataclass
class AttnInputs:
    """bf16 bit patterns (uint16) of X and the four projection weights
    ([in, out] layout), plus the fp32 output bias (or None)."""
    X: np.ndarray
    Wq: np.ndarray
    Wk: np.ndarray
    Wv: np.ndarray
    Wo: np.ndarray
    bo: Optional[np.ndarray]

    def values(self, name: str) -> Optional[np.ndarray]:
        a = getattr(self, name)
        if a is None:
            return None
        return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a


def make_attn_inputs(T: int, d: int, n_heads: int, n_kv_heads: int, head_dim: int,
                     seed: int = 42, with_bias: bool = False, w_std: float = 0.02) -> AttnInputs:
    """``default_rng(seed)`` float32 normals in the order X (std 1), Wq, Wk,
    Wv, Wo (std ``w_std``), bo (std 0.02), rounded to bf16 (bo kept as fp32
    holding bf16-representable values)."""
    rng = np.random.default_rng(seed)

    def draw(shape, std):
        v = rng.standard_normal(shape, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        return v

    c = f32_to_bf16_bits
    X = c(draw((T, d), 1.0))
    Wq = c(draw((d, n_heads * head_dim), w_std))
    Wk = c(draw((d, n_kv_heads * head_dim), w_std))
    Wv = c(draw((d, n_kv_heads * head_dim), w_std))
    Wo = c(draw((n_heads * head_dim, d), w_std))
    bo = bf16_bits_to_f32(c(draw((d,), 0.02))) if with_bias else None
    return AttnInputs(X, Wq, Wk, Wv, Wo, bo)


def make_qkv(p: int, T: int, hq: int, hkv: int, head_dim: int, seed: int, std: float = 1.0):
    """Per-shard bf16 (uint16) Q [p][T][hq*dh], K and V [p][T][hkv*dh] with
    standard-normal entries times ``std``, drawn in the order Q, K, V."""
    rng = np.random.default_rng(seed)
    out = []
    for cols in (hq * head_dim, hkv * head_dim, hkv * head_dim):
        v = rng.standard_normal((p, T, cols), dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        out.append(f32_to_bf16_bits(v))
    return tuple(out)


@dataclasses.dataclass(frozen=True)
class BlockWorkload:
    """One pre-norm transformer block: LayerNorm, the attention block, the
    residual add, LayerNorm, the MLP block, the residual add."""
    name: str
    T: int
    d: int
    n_heads: int
    n_kv_heads: int
    head_dim: int
    k: int            # FFN width
    p: int
    act: str
    causal: bool
    description: str

    def attn(self) -> AttnWorkload:
        return AttnWorkload(self.name + "/attn", self.T, self.d, self.n_heads, self.n_kv_heads,
                            self.head_dim, self.p, self.causal, "")

    def mlp_flops(self) -> int:
        return 2 * self.T * self.d * self.k * (3 if self.act == "swiglu" else 2)

    def flops(self) -> dict:
        a = self.attn().flops()
        m = self.mlp_flops()
        return {"attention_block": a["total"], "mlp_block": m, "total": a["total"] + m}


BLOCK_WORKLOADS = {
    "block_wide": BlockWorkload("block_wide", 4096, 4096, 32, 32, 128, 16384, 4, "gelu_tanh", True,
                                "transformer block: T=4096 d=4096, 32 heads x 128, d_ff=16384, "
                                "GELU(tanh), p=4, causal, bf16 GEMMs, fp32 residual stream"),
    "block_llama": BlockWorkload("block_llama", 4096, 8192, 64, 8, 128, 28672, 8, "swiglu", True,
                                 "Llama-70B-shaped block: T=4096 d=8192, 64 query / 8 key-value "
                                 "heads x 128, SwiGLU d_ff=28672, p=8, causal"),
}


@dataclasses.dataclass
class BlockInputs:
    """X (fp32 residual stream), LayerNorm gains/biases (fp32), projection
    weights and b1 as bf16 bit patterns (uint16), bo and b2 fp32."""
    X: np.ndarray
    prm: dict

    def values(self, name: str) -> Optional[np.ndarray]:
        a = self.X if name == "X" else self.prm[name]
        if a is None:
            return None
        return bf16_bits_to_f32(a) if a.dtype == np.uint16 else a

    def value_dict(self) -> dict:
        return {k: self.values(k) for k in self.prm}


def make_block_inputs(T: int, d: int, n_heads: int, n_kv_heads: int, head_dim: int, k: int,
                      act: str, seed: int = 42, w_std: float = 0.02,
                      with_bias: bool = True) -> BlockInputs:
    """``default_rng(seed)`` float32 normals in the order X (std 1), ln1 gain
    (1 + 0.1 N), ln1 bias (0.1 N), Wq, Wk, Wv, Wo (std ``w_std``), bo
    (0.02 N), ln2 gain, ln2 bias, W1, W_up (SwiGLU only), b1, W2, b2; matrices
    and b1 rounded to bf16, bo and b2 kept fp32 holding bf16 values."""
    rng = np.random.default_rng(seed)

    def draw(shape, std, mean=0.0):
        v = rng.standard_normal(shape, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        if mean != 0.0:
            v += np.float32(mean)
        return v

    c = f32_to_bf16_bits

    def vec_bf16_f32(n):
        return bf16_bits_to_f32(c(draw((n,), 0.02)))

    X = draw((T, d), 1.0)
    prm = {"ln1_gamma": draw((d,), 0.1, 1.0), "ln1_beta": draw((d,), 0.1)}
    prm["Wq"] = c(draw((d, n_heads * head_dim), w_std))
    prm["Wk"] = c(draw((d, n_kv_heads * head_dim), w_std))
    prm["Wv"] = c(draw((d, n_kv_heads * head_dim), w_std))
    prm["Wo"] = c(draw((n_heads * head_dim, d), w_std))
    prm["bo"] = vec_bf16_f32(d) if with_bias else None
    prm["ln2_gamma"] = draw((d,), 0.1, 1.0)
    prm["ln2_beta"] = draw((d,), 0.1)
    prm["W1"] = c(draw((d, k), w_std))
    prm["W_up"] = c(draw((d, k), w_std)) if act == "swiglu" else None
    prm["b1"] = c(draw((k,), 0.02)) if with_bias else None
    prm["W2"] = c(draw((k, d), w_std))
    prm["b2"] = vec_bf16_f32(d) if with_bias else None
    return BlockInputs(X, prm)


def f32_to_bf16_bits(x: np.ndarray) -> np.ndarray:
    """Round float32 values to bf16 (round to nearest, ties to even) and
    return the 16-bit patterns as uint16.  Inputs here are finite."""
    u = np.ascontiguousarray(x, dtype=np.float32).view(np.uint32)
    lsb = (u >> np.uint32(16)) & np.uint32(1)
    r = (u + np.uint32(0x7FFF) + lsb) >> np.uint32(16)
    return r.astype(np.uint16)


def bf16_bits_to_f32(b: np.ndarray) -> np.ndarray:
    """Exact widening of bf16 bit patterns (uint16) to float32."""
    return (np.ascontiguousarray(b, dtype=np.uint16).astype(np.uint32) << np.uint32(16)).view(np.float32)


@dataclasses.dataclass
class Inputs:
    """Host arrays of one workload instance.

    For ``dtype == "bf16"`` the X, W1, W_up, b1, W2 arrays are uint16 bf16 bit
    patterns; for ``"f32"`` they are float32.  b2 is always float32 (or None).
    """
    X: np.ndarray
    W1: np.ndarray
    W_up: Optional[np.ndarray]
    b1: Optional[np.ndarray]
    W2: np.ndarray
    b2: Optional[np.ndarray]
    dtype: str

    def values(self, name: str) -> Optional[np.ndarray]:
        """The array as float32 values (bf16 patterns widened exactly)."""
        a = getattr(self, name)
        if a is None:
            return None
        if a.dtype == np.uint16:
            return bf16_bits_to_f32(a)
        return a


def toy_page_example(seed: int = 42):
    """The column-parallel walkthrough's draw: legacy seed, then randn for
    x[4,512], W[512,2048], b[2048], each cast to float32."""
    np.random.seed(seed)
    x = np.random.randn(4, 512).astype(np.float32)
    W = np.random.randn(512, 2048).astype(np.float32)
    b = np.random.randn(2048).astype(np.float32)
    return x, W, b


def make_inputs(w: Workload, seed: int = 42, T: Optional[int] = None) -> Inputs:
    """Draw one instance of workload ``w``.  ``T`` overrides the token count
    (the weights are drawn identically; X gets ``T`` rows)."""
    T = w.T if T is None else T
    if w.name == "toy" and T == w.T:
        x, W1, b1 = toy_page_example(seed)
        W2 = np.random.randn(w.k, w.d).astype(np.float32)
        return Inputs(x, W1, None, b1, W2, None, "f32")
    rng = np.random.default_rng(seed)

    def draw(shape, std):
        v = rng.standard_normal(shape, dtype=np.float32)
        if std != 1.0:
            v *= np.float32(std)
        return v

    if w.dtype == "f32":
        X = draw((T, w.d), 1.0)
        W1 = draw((w.d, w.k), 1.0)
        W_up = draw((w.d, w.k), 1.0) if w.act == "swiglu" else None
        b1 = draw((w.k,), 1.0) if w.has_b1 else None
        W2 = draw((w.k, w.d), 1.0)
        b2 = draw((w.d,), 1.0) if w.has_b2 else None
        return Inputs(X, W1, W_up, b1, W2, b2, "f32")

    X = f32_to_bf16_bits(draw((T, w.d), 1.0))
    W1 = f32_to_bf16_bits(draw((w.d, w.k), 0.02))
    W_up = f32_to_bf16_bits(draw((w.d, w.k), 0.02)) if w.act == "swiglu" else None
    b1 = f32_to_bf16_bits(draw((w.k,), 0.02)) if w.has_b1 else None
    W2 = f32_to_bf16_bits(draw((w.k, w.d), 0.02))
    b2 = bf16_bits_to_f32(f32_to_bf16_bits(draw((w.d,), 0.02))) if w.has_b2 else None
    return Inputs(X, W1, W_up, b1, W2, b2, "bf16")


def small_integer_inputs(T: int, d: int, k: int, seed: int, lo: int = -2, hi: int = 2,
                         act: str = "identity", dtype: str = "f32",
                         with_b1: bool = True, with_b2: bool = True) -> Inputs:
    """Small-integer inputs (entries in [lo, hi]) for exact-arithmetic cases:
    every product and partial sum stays an integer far below 2**8 (bf16) or
    2**24 (fp32) for the sizes the tests use, so any summation order gives
    the same bits."""
    rng = np.random.default_rng(seed)

    def ints(shape):
        return rng.integers(lo, hi + 1, size=shape).astype(np.float32)

    X = ints((T, d))
    W1 = ints((d, k))
    W_up = ints((d, k)) if act == "swiglu" else None
    b1 = ints((k,)) if with_b1 else None
    W2 = ints((k, d))
    b2 = ints((d,)) if with_b2 else None
    if dtype == "bf16":
        conv = f32_to_bf16_bits
        return Inputs(conv(X), conv(W1), None if W_up is None else conv(W_up),
                      None if b1 is None else conv(b1), conv(W2), b2, "bf16")
    return Inputs(X, W1, W_up, b1, W2, b2, "f32")


def random_partials(p: int, T: int, d: int, seed: int) -> np.ndarray:
    """Random fp32 partials [p][T][d] spanning several binades (so that the
    order of the fp32 additions changes the rounded result)."""
    rng = np.random.default_rng(seed)
    mant = rng.standard_normal((p, T, d), dtype=np.float32)
    expo = rng.integers(-6, 7, size=(p, T, d)).astype(np.float32)
    return (mant * np.exp2(expo)).astype(np.float32)
