"""GPU parity of the MLP block's backward pass (tp_mlp_block_backward)
against the oracle's sharded backward.

The device path stores the pre-activations H, the activations Y and the
activation gradients dH in bf16 and accumulates every GEMM in fp32; the
oracle runs the same steps in float64 with the same bf16 storage rounding
(hidden_round="bf16"), so each gradient is compared with
max|gpu - oracle| / max|oracle| <= 1e-2, the bf16-path tolerance.  The dX
fold is checked bit-exact against the oracle's fixed-order fold of the
device's own partials elsewhere (the reduction tests); here dX is the
end-to-end value."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
import workloads as W
from gpu_util import dev, host_f32, region_fold_enabled
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

TOL = 1e-2


def _inputs(T, d, k, act, seed, dz_std=1.0, w_std=0.05):
    rng = np.random.default_rng(seed)
    c = W.f32_to_bf16_bits
    X = c(rng.standard_normal((T, d), dtype=np.float32))
    W1 = c(rng.standard_normal((d, k), dtype=np.float32) * np.float32(w_std))
    Wu = c(rng.standard_normal((d, k), dtype=np.float32) * np.float32(w_std)) if act == "swiglu" else None
    b1 = c(rng.standard_normal(k, dtype=np.float32) * np.float32(0.05))
    W2 = c(rng.standard_normal((k, d), dtype=np.float32) * np.float32(w_std))
    dZ = c(rng.standard_normal((T, d), dtype=np.float32) * np.float32(dz_std))
    return {"X": X, "W1": W1, "W_up": Wu, "b1": b1, "W2": W2, "dZ": dZ}


def _vals(a):
    return None if a is None else W.bf16_bits_to_f32(a)


class DeviceBackward:
    """Forward tensors the backward call needs (H, H_up, Y from
    tp_column_linear) and the gradient buffers."""

    def __init__(self, inp, T, d, k, p, act):
        self.T, self.d, self.k, self.p, self.s = T, d, k, p, k // p
        self.act = tp.ACT[act]
        t = {n: dev(v) for n, v in inp.items()}
        self.t = t
        bf = tp.TP_BF16
        sh = (p, T, self.s)
        self.H = torch.empty(sh, dtype=torch.bfloat16, device="cuda")
        self.Hu = torch.empty(sh, dtype=torch.bfloat16, device="cuda") if act == "swiglu" else None
        self.Y = torch.empty(sh, dtype=torch.bfloat16, device="cuda")
        ident = tp.TP_ACT_IDENTITY
        tp.tp_column_linear(t["X"], t["W1"], None, t["b1"], self.H, T, d, k, p, bf, ident)
        if self.Hu is not None:
            tp.tp_column_linear(t["X"], t["W_up"], None, None, self.Hu, T, d, k, p, bf, ident)
        tp.tp_column_linear(t["X"], t["W1"], t["W_up"], t["b1"], self.Y, T, d, k, p, bf, self.act)

        def f32(*shape):
            return torch.full(shape, float("nan"), dtype=torch.float32, device="cuda")
        self.dX, self.dW1, self.db1 = f32(T, d), f32(d, k), f32(k)
        self.dWu = f32(d, k) if act == "swiglu" else None
        self.dW2, self.db2 = f32(k, d), f32(d)
        self.n = tp.tp_mlp_block_backward_workspace_size(T, d, k, p, self.act)
        self.ws = torch.empty(self.n, dtype=torch.uint8, device="cuda")

    def run(self, check=True, sync=True):
        t = self.t
        st = tp.tp_mlp_block_backward(t["X"], t["W1"], t["W_up"], t["W2"], self.H, self.Hu, self.Y,
                                      t["dZ"], self.dX, self.dW1, self.dWu, self.db1, self.dW2,
                                      self.db2, self.ws, self.n, self.T, self.d, self.k, self.p,
                                      self.act, check=check)
        if sync:
            tp.tp_sync_status()
        return st

    def grads(self):
        out = {"dX": self.dX, "dW1": self.dW1, "db1": self.db1, "dW2": self.dW2, "db2": self.db2}
        if self.dWu is not None:
            out["dW_up"] = self.dWu
        return {k: host_f32(v) for k, v in out.items()}


CASES = [
    # T, d, k, p, act
    (300, 256, 512, 2, "gelu_tanh"),
    (129, 512, 1024, 4, "swiglu"),
    (64, 128, 256, 1, "relu"),
    (1000, 1024, 4096, 4, "gelu_tanh"),
    (1, 256, 512, 2, "swiglu"),
    (200, 384, 768, 3, "identity"),
    (513, 1024, 4096, 8, "swiglu"),
    # large enough for CTA-pair tiles (256-row tiles on two SMs) in all four
    # GEMMs (so the dX fold runs beside its GEMM), one with a ragged last
    # pair tile (1800 = 7 x 256 + 8 rows)
    (2048, 2048, 4096, 4, "swiglu"),
    (1800, 2048, 4096, 4, "gelu_tanh"),
]


@pytest.mark.parametrize("T,d,k,p,act", CASES)
def test_backward_matches_oracle(T, d, k, p, act):
    inp = _inputs(T, d, k, act, seed=T + d + k)
    blk = DeviceBackward(inp, T, d, k, p, act)
    blk.run()
    got = blk.grads()
    ref = O.mlp_backward_sharded(_vals(inp["X"]), _vals(inp["W1"]), _vals(inp["b1"]),
                                 _vals(inp["W2"]), _vals(inp["dZ"]), p, act,
                                 W_up=_vals(inp["W_up"]), hidden_round="bf16")
    for name, g in got.items():
        assert np.isfinite(g).all(), name
        assert O.rel_err(g, ref[name]) <= TOL, (name, O.rel_err(g, ref[name]))


@pytest.mark.parametrize("name", ["wide", "llama"])
def test_backward_full_size_sampled(name):
    """Full-size shapes.  dX rows depend only on their own token, so the
    oracle runs on a few rows; the weight gradients of a hidden unit depend
    only on that unit's column of W1 (and W_up) and row of W2, so the oracle
    runs on a few hidden units (p = 1 restricted to those columns)."""
    w = W.WORKLOADS[name]
    T, d, k, p, act = w.T, w.d, w.k, w.p, w.act
    inp = _inputs(T, d, k, act, seed=7, w_std=0.02)
    blk = DeviceBackward(inp, T, d, k, p, act)
    blk.run()
    got = blk.grads()
    for v in got.values():
        assert np.isfinite(v).all()
    X, W1, b1, W2, dZ = (_vals(inp[n]) for n in ("X", "W1", "b1", "W2", "dZ"))
    Wu = _vals(inp["W_up"])
    rows = np.array([0, 1, 127, 128, T // 2, T - 1])
    ref_rows = O.mlp_backward_sharded(X[rows], W1, b1, W2, dZ[rows], p, act, W_up=Wu,
                                      hidden_round="bf16")
    assert O.rel_err(got["dX"][rows], ref_rows["dX"]) <= TOL
    cols = np.array([0, 63, 64, k // p - 1, k // p, k // 2 + 5, k - 1])
    ref_cols = O.mlp_backward_sharded(X, W1[:, cols], b1[cols], W2[cols, :], dZ, 1, act,
                                      W_up=None if Wu is None else Wu[:, cols],
                                      hidden_round="bf16")
    assert O.rel_err(got["dW1"][:, cols], ref_cols["dW1"]) <= TOL
    assert O.rel_err(got["db1"][cols], ref_cols["db1"]) <= TOL
    assert O.rel_err(got["dW2"][cols, :], ref_cols["dW2"]) <= TOL
    if Wu is not None:
        assert O.rel_err(got["dW_up"][:, cols], ref_cols["dW_up"]) <= TOL
    assert O.rel_err(got["db2"], ref_cols["db2"]) <= 1e-5


def test_backward_optional_outputs_and_errors():
    T, d, k, p = 128, 256, 512, 2
    inp = _inputs(T, d, k, "gelu_tanh", seed=3)
    blk = DeviceBackward(inp, T, d, k, p, "gelu_tanh")
    blk.run()
    full = blk.grads()
    # only dX: the other buffers must stay untouched (NaN)
    blk.dW1.fill_(float("nan"))
    blk.dW2.fill_(float("nan"))
    dW1, dW2 = blk.dW1, blk.dW2
    blk.dW1 = blk.dW2 = None
    blk.db1 = blk.db2 = None
    blk.run()
    assert np.array_equal(host_f32(blk.dX), full["dX"])
    assert torch.isnan(dW1).all() and torch.isnan(dW2).all()
    # k/p not a multiple of 64
    t = blk.t
    assert tp.tp_mlp_block_backward(t["X"], t["W1"], None, t["W2"], blk.H, None, blk.Y, t["dZ"],
                                    blk.dX, None, None, None, None, None, blk.ws, blk.n, T, d,
                                    k - 64, p, blk.act, check=False) in (2, 4)
    # SwiGLU without the up projection
    assert tp.tp_mlp_block_backward(t["X"], t["W1"], None, t["W2"], blk.H, None, blk.Y, t["dZ"],
                                    blk.dX, None, None, None, None, None, blk.ws, blk.n, T, d, k,
                                    p, tp.TP_ACT_SWIGLU, check=False) == 1


def test_backward_dropped_load_times_out():
    tp.tp_set_wait_timeout_ns(50_000_000)
    try:
        T, d, k, p = 256, 256, 512, 2
        inp = _inputs(T, d, k, "gelu_tanh", seed=5)
        blk = DeviceBackward(inp, T, d, k, p, "gelu_tanh")
        assert tp.tp_sync_status(check=False) == 0
        tp.tp_debug_drop_load(1)
        blk.run(check=False, sync=False)
        assert tp.tp_sync_status(check=False) == 6
    finally:
        tp.tp_set_wait_timeout_ns(0)
        tp.tp_debug_drop_load(-1)
    blk.run()
    ref = O.mlp_backward_sharded(_vals(inp["X"]), _vals(inp["W1"]), _vals(inp["b1"]),
                                 _vals(inp["W2"]), _vals(inp["dZ"]), p, "gelu_tanh",
                                 hidden_round="bf16")
    assert O.rel_err(host_f32(blk.dX), ref["dX"]) <= TOL


@pytest.mark.parametrize("T,d,k,p,act", [(300, 256, 512, 2, "gelu_tanh"), (129, 512, 1024, 4, "swiglu")])
def test_backward_recompute_matches_explicit(T, d, k, p, act):
    """tp_mlp_block_backward_recompute rebuilds H (and the up projection) and
    Y with the same column-layer kernels, so its gradients have the same bits
    as the explicit call on tp_column_linear's outputs."""
    inp = _inputs(T, d, k, act, seed=T + k)
    blk = DeviceBackward(inp, T, d, k, p, act)
    blk.run()
    want = blk.grads()
    t = blk.t
    out = {name: torch.full_like(v, float("nan")) for name, v in
           (("dX", blk.dX), ("dW1", blk.dW1), ("db1", blk.db1), ("dW2", blk.dW2), ("db2", blk.db2))}
    if blk.dWu is not None:
        out["dW_up"] = torch.full_like(blk.dWu, float("nan"))
    n = tp.tp_mlp_block_backward_recompute_workspace_size(T, d, k, p, blk.act)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    tp.tp_mlp_block_backward_recompute(t["X"], t["W1"], t["W_up"], t["b1"], t["W2"], t["dZ"],
                                       out["dX"], out["dW1"], out.get("dW_up"), out["db1"],
                                       out["dW2"], out["db2"], ws, n, T, d, k, p, blk.act)
    tp.tp_sync_status()
    for name, v in out.items():
        got = host_f32(v)
        assert np.array_equal(got.view(np.uint32), want[name].view(np.uint32)), name


def _r256(n):
    return -(-n // 256) * 256


@pytest.mark.parametrize("T,d,k,p,act", [(2048, 2048, 4096, 4, "swiglu"),
                                         (1800, 2048, 4096, 4, "gelu_tanh")])
def test_dx_fold_beside_its_gemm_is_the_fixed_order_fold(T, d, k, p, act):
    """On shapes whose dX partials run on CTA-pair tiles the dX fold runs
    beside that GEMM: dX must have the bits of tp_reduce_partials applied to
    the partials the call left in its workspace, and the workspace's region
    counters must read 16 p (the layout: dH, dU for SwiGLU, the partials,
    the bias-gradient scratch, the counters)."""
    inp = _inputs(T, d, k, act, seed=5)
    blk = DeviceBackward(inp, T, d, k, p, act)
    blk.ws.fill_(0x7F)
    blk.run()
    off = _r256(T * k * 2) * (2 if act == "swiglu" else 1)
    part = blk.ws[off:off + p * T * d * 4].view(torch.float32).view(p, T, d)
    Z = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")
    tp.tp_reduce_partials(part, None, Z, T, d, p)
    tp.tp_sync_status()
    assert np.array_equal(host_f32(Z).view(np.uint32), host_f32(blk.dX).view(np.uint32))
    if not region_fold_enabled():
        return
    scratch = _r256(-(-T // 128) * max(k, d) * 4)
    cnt_off = off + _r256(p * T * d * 4) + scratch
    m_regions = -(-T // 256)
    cnt = blk.ws[cnt_off:cnt_off + 4 * m_regions * -(-d // 128)].cpu().numpy().view(np.int32)
    assert cnt[0] == 16 * p
    assert set(np.unique(cnt).tolist()) <= {0, 16 * p}
