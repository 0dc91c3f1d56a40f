"""tp_mlp_block_noalloc: the block for callers that cannot allocate device
memory (a plugin whose host framework owns the whole device memory pool, or
a hot loop that cannot afford cudaMalloc's device synchronisation).  Its
scratch is a fixed 16 MiB array inside the library instead of a caller
workspace.

Checked through the C ABI against the existing entry point, tp_mlp_block with
a caller workspace, on two calls in a row (the second call reuses the scratch
the first one left behind).  Both entry points run the same kernels on the
same inputs, so the outputs must be identical bit for bit; that also catches
a wrong offset or an overlap inside the scratch.  Every flag that changes the
scratch layout is covered: the default (hidden shards then partials), split-K
(hidden shards only), the single persistent launch (tile counters at the end
of the scratch, which must start at zero on every call) and the fold in the
row layer's epilogue.  This file is collected last so that a run stopping at
its first failure has already run every other test; it also passes alone in
a fresh process."""

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
import workloads as W
from gpu_util import DeviceBlock, bits, host_f32

pytestmark = pytest.mark.gpu

SCRATCH_BYTES = 16 << 20


def _noalloc(blk, flags=tp.TP_FLAG_NONE):
    Z = torch.full_like(blk.Z, float("nan"))
    tp.tp_mlp_block_noalloc(blk.X, blk.W1, blk.Wu, blk.b1, blk.W2, blk.b2, Z, blk.T, blk.d, blk.k,
                            blk.p, blk.dtype, blk.act, flags)
    return Z


def _reference(blk, flags=tp.TP_FLAG_NONE):
    Z = torch.full_like(blk.Z, float("nan"))
    blk.block(flags, Z=Z)
    return Z


def _same_bits(got, want):
    g, w = host_f32(got), host_f32(want)
    assert not np.isnan(g).any()
    assert np.array_equal(bits(g), bits(w)), float(np.max(np.abs(g - w)))


@pytest.mark.parametrize("name,flags", [
    ("gpt2", tp.TP_FLAG_NONE),
    ("toy", tp.TP_FLAG_NONE),
    ("gpt2", tp.TP_FLAG_SPLITK_FUSED),
    ("gpt2", tp.TP_FLAG_FUSED_LAUNCH),
    ("gpt2", tp.TP_FLAG_ROW_FOLD),
], ids=["gpt2", "toy", "gpt2-splitk", "gpt2-fused-launch", "gpt2-row-fold"])
def test_bit_identical_to_workspace_entry_point_two_calls_in_a_row(name, flags):
    w = W.WORKLOADS[name]
    first = W.make_inputs(w, seed=42)
    second = W.make_inputs(w, seed=43)
    blocks = [DeviceBlock(x, w.T, w.d, w.k, w.p, w.act) for x in (first, second)]
    need = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, w.p, blocks[0].dtype, blocks[0].act,
                                          flags)
    assert 0 < need <= SCRATCH_BYTES
    outs = [_noalloc(b, flags) for b in blocks]   # two calls in a row, same scratch
    refs = [_reference(b, flags) for b in blocks]
    tp.tp_sync_status()
    for got, want in zip(outs, refs):
        _same_bits(got, want)
    # the two inputs differ, so the second call really recomputed
    assert not np.array_equal(host_f32(outs[0]), host_f32(outs[1]))
    # and a third call on the first inputs, after the second call's leftovers
    _same_bits(_noalloc(blocks[0], flags), refs[0])
    tp.tp_sync_status()


def test_rejects_problems_larger_than_the_scratch():
    w = W.WORKLOADS["wide"]   # needs ~400 MB of scratch
    X = torch.zeros(8, device="cuda")
    Z = torch.zeros(8, device="cuda")
    st = tp.tp_mlp_block_noalloc(X, X, None, None, X, None, Z, w.T, w.d, w.k, w.p, tp.TP_BF16,
                                 tp.TP_ACT_GELU_TANH, check=False)
    assert st == 7
    assert "16777216" in tp.tp_last_error_detail()
    assert tp.tp_mlp_block_noalloc(X, X, None, None, X, None, Z, 4, 64, 250, 4, tp.TP_BF16,
                                   tp.TP_ACT_GELU_TANH, check=False) == 2
