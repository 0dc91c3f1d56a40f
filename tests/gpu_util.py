"""Helpers for the GPU parity tests: host arrays -> device tensors, device
results -> host arrays, and a run of the whole block through the C ABI.
The oracle is called by the tests themselves, never from here."""

import numpy as np
import torch

import megatron_tensor_sharded_b200 as tp


def dev(a, device="cuda"):
    """numpy float32 or bf16-bit (uint16) array -> device tensor."""
    if a is None:
        return None
    if a.dtype == np.uint16:
        return torch.from_numpy(np.ascontiguousarray(a).view(np.int16)).view(torch.bfloat16).to(device)
    return torch.from_numpy(np.ascontiguousarray(a)).to(device)


def host_f32(t):
    """device tensor (bf16 or fp32) -> numpy float32 values."""
    return t.detach().float().cpu().numpy()


def bits(a):
    return np.ascontiguousarray(a, dtype=np.float32).view(np.uint32)


def pairs_enabled():
    """CTA-pair tiles are in use (the library's TP_DISABLE_PAIR=1 turns them
    off, and with them the one-launch Q, K, V and the fold beside the row
    layer)."""
    import os
    return os.environ.get("TP_DISABLE_PAIR", "") != "1"


def region_fold_enabled():
    """The fold beside the row layer is in use (TP_DISABLE_REGION_FOLD=1 and
    single-CTA tiles turn it off)."""
    import os
    return pairs_enabled() and os.environ.get("TP_DISABLE_REGION_FOLD", "") != "1"


def row_chain_enabled():
    """The row layer folds the partials in its own epilogue where the fold
    beside it would run (TP_DISABLE_ROW_CHAIN=1 keeps the fold beside it)."""
    import os
    return region_fold_enabled() and os.environ.get("TP_DISABLE_ROW_CHAIN", "") != "1"


class DeviceBlock:
    """Device copies of one workload instance plus output buffers."""

    def __init__(self, inp, T, d, k, p, act):
        self.T, self.d, self.k, self.p, self.s = T, d, k, p, k // p
        self.act = tp.ACT[act]
        self.dtype = tp.DTYPE[inp.dtype]
        self.X, self.W1, self.Wu = dev(inp.X), dev(inp.W1), dev(inp.W_up)
        self.b1, self.W2, self.b2 = dev(inp.b1), dev(inp.W2), dev(inp.b2)
        hdt = torch.bfloat16 if inp.dtype == "bf16" else torch.float32
        self.Y = torch.full((p, T, self.s), float("nan"), dtype=hdt, device="cuda")
        self.P = torch.full((p, T, d), float("nan"), dtype=torch.float32, device="cuda")
        self.Z = torch.full((T, d), float("nan"), dtype=torch.float32, device="cuda")

    def column(self):
        tp.tp_column_linear(self.X, self.W1, self.Wu, self.b1, self.Y, self.T, self.d, self.k,
                            self.p, self.dtype, self.act)

    def row(self):
        tp.tp_row_linear(self.Y, self.W2, self.P, self.T, self.k, self.d, self.p, self.dtype)

    def reduce(self):
        tp.tp_reduce_partials(self.P, self.b2, self.Z, self.T, self.d, self.p)

    def block(self, flags=tp.TP_FLAG_NONE, Z=None):
        Z = self.Z if Z is None else Z
        n = tp.tp_mlp_block_workspace_size(self.T, self.d, self.k, self.p, self.dtype, self.act, flags)
        ws = torch.empty(max(n, 256), dtype=torch.uint8, device="cuda")
        tp.tp_mlp_block(self.X, self.W1, self.Wu, self.b1, self.W2, self.b2, Z, ws, n, self.T,
                        self.d, self.k, self.p, self.dtype, self.act, flags)
        return ws

    def sync(self):
        tp.tp_sync_status()
