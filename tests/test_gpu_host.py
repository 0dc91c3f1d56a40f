"""GPU parity of tp_mlp_block_host (X and Z in host memory, the token rows
pipelined in chunks through copy-in, the block and copy-out).

The block is row-wise, so the chunked call must give exactly the bits of the
device call on all rows (same kernels, same per-element order); that is
checked bit for bit, and the device call itself is checked against the
oracle, as in the other parity tests."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
import workloads as W
from gpu_util import DeviceBlock, bits, host_f32
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu


def _host_x(inp, pinned):
    if inp.X.dtype == np.uint16:
        t = torch.from_numpy(np.ascontiguousarray(inp.X).view(np.int16)).view(torch.bfloat16)
    else:
        t = torch.from_numpy(np.ascontiguousarray(inp.X))
    return t.pin_memory() if pinned else t.clone()


def _run_host(blk, Xh, flags=tp.TP_FLAG_NONE, pinned=True, stream=None):
    Zh = torch.full((blk.T, blk.d), float("nan"), dtype=torch.float32)
    if pinned:
        Zh = Zh.pin_memory()
    n = tp.tp_mlp_block_host_workspace_size(blk.T, blk.d, blk.k, blk.p, blk.dtype, blk.act, flags)
    ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
    tp.tp_mlp_block_host(Xh, blk.W1, blk.Wu, blk.b1, blk.W2, blk.b2, Zh, ws, n, blk.T, blk.d,
                         blk.k, blk.p, blk.dtype, blk.act, flags, stream=stream)
    torch.cuda.synchronize()
    tp.tp_sync_status()
    return Zh.numpy().copy()


CASES = [
    # T, d, k, p, act, bias
    (1024, 768, 3072, 2, "gelu_tanh", True),     # GPT-2 width: four chunks of 256 rows
    (300, 256, 512, 2, "gelu_tanh", True),       # two chunks, the second ragged (44 rows)
    (1, 128, 256, 1, "swiglu", False),           # one row, one chunk
    (1000, 1024, 4096, 4, "swiglu", False),      # four chunks of 256, last of 232
    (257, 512, 2048, 8, "relu", True),           # 256 + 1
]


@pytest.mark.parametrize("T,d,k,p,act,bias", CASES)
@pytest.mark.parametrize("pinned", [True, False])
def test_host_call_matches_device_call(T, d, k, p, act, bias, pinned):
    inp = W.make_inputs(W.Workload("t", T, d, k, p, act, "bf16", bias, bias, ""), seed=T + d)
    blk = DeviceBlock(inp, T, d, k, p, act)
    blk.block()
    blk.sync()
    want = host_f32(blk.Z)
    got = _run_host(blk, _host_x(inp, pinned), pinned=pinned)
    assert np.array_equal(bits(got), bits(want))
    ref = O.mlp_sharded(inp.values("X"), inp.values("W1"), inp.values("b1"),
                        inp.values("W2"), inp.b2, p, act, W_up=inp.values("W_up"))["Z"]
    assert O.rel_err(got, ref) <= 1e-2


def test_host_call_flags_pass_through():
    """Split-K and the single-launch block run per chunk as well."""
    T, d, k, p = 700, 512, 2048, 4
    inp = W.make_inputs(W.Workload("t", T, d, k, p, "gelu_tanh", "bf16", True, True, ""), seed=5)
    blk = DeviceBlock(inp, T, d, k, p, "gelu_tanh")
    Xh = _host_x(inp, True)
    for flags in (tp.TP_FLAG_FUSED_LAUNCH, tp.TP_FLAG_SPLITK_FUSED,
                  tp.TP_FLAG_SPLITK_FUSED | tp.TP_FLAG_FUSED_LAUNCH):
        Zd = torch.full_like(blk.Z, float("nan"))
        blk.block(flags, Z=Zd)
        blk.sync()
        assert np.array_equal(bits(_run_host(blk, Xh, flags)), bits(host_f32(Zd))), flags


def test_host_call_fp32_toy():
    """The pages' fp32 shape (4 tokens) through the host call."""
    w = W.WORKLOADS["toy"]
    inp = W.make_inputs(w)
    blk = DeviceBlock(inp, w.T, w.d, w.k, w.p, w.act)
    blk.block()
    blk.sync()
    got = _run_host(blk, _host_x(inp, True))
    assert np.array_equal(bits(got), bits(host_f32(blk.Z)))


def test_host_call_in_a_graph_and_on_a_side_stream():
    """Captured into a CUDA graph from a side stream (pinned buffers) and
    replayed: the helper streams fork from and join into the capturing
    stream, so every replay writes the same Z into the host buffer."""
    w = W.WORKLOADS["gpt2"]
    inp = W.make_inputs(w)
    blk = DeviceBlock(inp, w.T, w.d, w.k, w.p, w.act)
    blk.block()
    blk.sync()
    want = bits(host_f32(blk.Z))
    Xh = _host_x(inp, True)
    Zh = torch.full((w.T, w.d), float("nan"), dtype=torch.float32).pin_memory()
    n = tp.tp_mlp_block_host_workspace_size(w.T, w.d, w.k, w.p, blk.dtype, blk.act)
    ws = torch.empty(n, dtype=torch.uint8, device="cuda")
    s = torch.cuda.Stream()

    def call(stream):
        tp.tp_mlp_block_host(Xh, blk.W1, blk.Wu, blk.b1, blk.W2, blk.b2, Zh, ws, n, w.T, w.d,
                             w.k, w.p, blk.dtype, blk.act, stream=stream)

    with torch.cuda.stream(s):
        call(s)                      # uncaptured first call creates the helper streams
    s.synchronize()
    assert np.array_equal(bits(Zh.numpy()), want)
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g, stream=s):
        call(torch.cuda.current_stream())
    for _ in range(3):
        Zh.fill_(float("nan"))
        g.replay()
        torch.cuda.synchronize()
        assert np.array_equal(bits(Zh.numpy()), want)
    tp.tp_sync_status()
