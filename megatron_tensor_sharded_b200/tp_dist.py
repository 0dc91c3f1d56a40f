"""The tensor-parallel MLP block on p GPUs, one process per GPU.

Shard i lives on GPU i, as the pages lay the method out: X is replicated,
W1's column block i (and W_up's, for SwiGLU), b1's slice i and W2's row block
i are local; each GPU runs the column-parallel layer and the row-parallel
layer on its own shard (tp_column_linear and tp_row_linear with one local
shard), and the p full-shape partials are summed across GPUs by one
all-reduce, the output bias added after it (day-41 post, "Simulating row
parallel linear"; "Building GPT from Scratch -- Part 9", "Implementation
Sketch": ColumnParallelLinear needs no communication, RowParallelLinear
all-reduces its partial outputs and then adds the bias).

The all-reduce is deterministic and bit-identical to the single-GPU
fixed-order fold (tp_reduce_partials): GPU r owns the token-row slab r of Z,
folds that slab of P_0, ..., P_{p-1} in shard order in one of this library's
kernels, and the folded slabs are gathered on every GPU.  Two exchanges:

* ``"nccl"``: an all-to-all of row slabs (GPU r receives slab r of every
  partial), the fold (tp_reduce_partials on the received [p][rows][d]
  block), an all-gather of the folded slabs.
* ``"peer"``: every GPU maps its peers' partial and output buffers once
  (CUDA IPC, tp_ipc_export / tp_ipc_import); a step is a stream-ordered
  barrier, one tp_reduce_partials_gather launch that reads slab r of every
  partial over NVLink and writes the folded slab into every GPU's Z (the
  reduce-scatter and the all-gather in one pass), and a second barrier.

Plumbing (process groups, the all-to-all, the all-gather, the barriers) is
torch.distributed; every arithmetic step is a kernel of this library.  The
``fold`` argument of :func:`fixed_order_all_reduce` exists so that the
exchange logic can be exercised on host tensors with a host fold in tests;
the product path passes none and uses the CUDA fold.
"""

from __future__ import annotations

from typing import Callable, List, Optional, Sequence, Tuple

import megatron_tensor_sharded_b200 as tp


def row_slabs(T: int, world: int) -> List[Tuple[int, int]]:
    """(row0, rows) of the token-row slab each rank owns: contiguous, in rank
    order, ceil(T / world) rows each except at the end (a rank may own none
    when T < world)."""
    if world < 1 or T < 0:
        raise ValueError(f"T={T}, world={world}")
    m = -(-T // world) if T else 0
    out = []
    for r in range(world):
        r0 = min(T, r * m)
        out.append((r0, max(0, min(T, r0 + m) - r0)))
    return out


def shard_weights(W1, W_up, b1, W2, rank: int, world: int):
    """Rank `rank`'s blocks of the full weights (row-major [in, out]):
    W1[:, i s:(i+1) s] (and W_up's), b1[i s:(i+1) s], W2[i s:(i+1) s, :],
    s = k / world, each made contiguous.  The divisibility rule is the
    walkthrough's: k must split evenly over the GPUs."""
    k = W1.shape[1]
    if k % world != 0:
        raise ValueError(f"{k} features cannot be split evenly over {world} shards")
    s = k // world
    c0, c1 = rank * s, (rank + 1) * s
    return (W1[:, c0:c1].contiguous(),
            None if W_up is None else W_up[:, c0:c1].contiguous(),
            None if b1 is None else b1[c0:c1].contiguous(),
            W2[c0:c1, :].contiguous())


def _cuda_fold(parts, b2, out, rows: int, d: int, p: int) -> None:
    tp.tp_reduce_partials(parts, b2, out, rows, d, p)


def fixed_order_all_reduce(P_local, b2, Z, group=None, fold: Optional[Callable] = None) -> None:
    """Z = ((P_0 + P_1) + ...) + P_{p-1} (+ b2) over the ranks of `group`,
    P_r being this rank's [T][d] fp32 partial: the ``"nccl"`` exchange.

    All-to-all of row slabs, the fold of this rank's slab in rank order,
    all-gather of the slabs (padded to equal length).  `fold(parts, b2, out,
    rows, d, p)` folds parts [p][rows][d] into out [rows][d]; None = the
    library's CUDA fold."""
    import torch
    import torch.distributed as dist

    fold = _cuda_fold if fold is None else fold
    world = dist.get_world_size(group)
    rank = dist.get_rank(group)
    T, d = P_local.shape
    slabs = row_slabs(T, world)
    m = slabs[0][1]
    rows = slabs[rank][1]
    recv = torch.empty((world * rows, d), dtype=P_local.dtype, device=P_local.device)
    dist.all_to_all_single(recv, P_local.contiguous(), output_split_sizes=[rows] * world,
                           input_split_sizes=[r for _, r in slabs], group=group)
    mine = torch.zeros((m, d), dtype=P_local.dtype, device=P_local.device)
    if rows:
        fold(recv.view(world, rows, d), b2, mine, rows, d, world)
    gathered = torch.empty((world * m, d), dtype=P_local.dtype, device=P_local.device)
    dist.all_gather_into_tensor(gathered, mine, group=group)
    Z.copy_(gathered[:T])


def peer_tables(rank: int, world: int, p_ptrs: Sequence[int], z_ptrs: Sequence[int], T: int):
    """Arguments of this rank's tp_reduce_partials_gather call in the
    ``"peer"`` exchange: the partials in shard (rank) order, every rank's Z as
    a destination, and this rank's slab."""
    if len(p_ptrs) != world or len(z_ptrs) != world:
        raise ValueError("one partial and one output buffer per rank")
    row0, rows = row_slabs(T, world)[rank]
    return list(p_ptrs), list(z_ptrs), row0, rows


class PeerAllReduce:
    """The ``"peer"`` exchange over buffers mapped once: this rank's P and Z
    ([T_max][d] fp32 each, from cudaMalloc-backed allocations) are exported,
    the handles exchanged, the peers' buffers imported."""

    def __init__(self, P, Z, group=None):
        import torch.distributed as dist

        self.group = group
        self.world = dist.get_world_size(group)
        self.rank = dist.get_rank(group)
        self.P, self.Z = P, Z
        mine = (tp.tp_ipc_export(P).to_bytes(), tp.tp_ipc_export(Z).to_bytes())
        allh: list = [None] * self.world
        dist.all_gather_object(allh, mine, group=group)
        self.imported = []
        self.p_ptrs, self.z_ptrs = [], []
        for r, (hp, hz) in enumerate(allh):
            if r == self.rank:
                self.p_ptrs.append(P.data_ptr())
                self.z_ptrs.append(Z.data_ptr())
                continue
            for h, dst in ((hp, self.p_ptrs), (hz, self.z_ptrs)):
                handle = tp.IpcHandle.from_bytes(h)
                dst.append(tp.tp_ipc_import(handle))
                self.imported.append(handle)

    def _barrier(self):
        """Stream-ordered barrier: over NCCL a one-element all-reduce on the
        current stream, which completes on a rank only once every rank has
        reached it; over other backends (gloo: ranks sharing one GPU in the
        tests) the stream is drained first and the barrier runs on the host."""
        import torch
        import torch.distributed as dist

        if dist.get_backend(self.group) == "nccl":
            flag = torch.zeros(1, dtype=torch.int32, device=self.P.device)
            dist.all_reduce(flag, group=self.group)
        else:
            torch.cuda.current_stream(self.P.device).synchronize()
            dist.barrier(group=self.group)

    def __call__(self, b2, T: int, d: int) -> None:
        parts, outs, row0, rows = peer_tables(self.rank, self.world, self.p_ptrs, self.z_ptrs, T)
        self._barrier()
        tp.tp_reduce_partials_gather(parts, b2, outs, row0, rows, d)
        self._barrier()

    def close(self) -> None:
        for h in self.imported:
            tp.tp_ipc_release(h)
        self.imported = []


class TensorParallelMLP:
    """This rank's part of the p-GPU block (bf16 weights, fp32 partials and
    output).  `W1_local` [d][s], `W_up_local` [d][s] (SwiGLU) or None,
    `b1_local` [s] or None, `W2_local` [s][d], `b2` [d] fp32 or None: the
    rank's blocks (see :func:`shard_weights`).  `forward(X)` returns Z [T][d],
    the same on every rank."""

    def __init__(self, W1_local, W_up_local, b1_local, W2_local, b2, act: int,
                 T_max: int, group=None, exchange: str = "nccl"):
        import torch
        import torch.distributed as dist

        if exchange not in ("nccl", "peer"):
            raise ValueError(exchange)
        self.group = group
        self.world = dist.get_world_size(group) if dist.is_initialized() else 1
        self.d, self.s = W1_local.shape
        self.W1, self.Wu, self.b1, self.W2, self.b2 = W1_local, W_up_local, b1_local, W2_local, b2
        self.act = act
        self.dtype = tp.TP_BF16 if W1_local.dtype == torch.bfloat16 else tp.TP_F32
        dev = W1_local.device
        self.Y = torch.empty((T_max, self.s), dtype=W1_local.dtype, device=dev)
        self.P = torch.empty((T_max, self.d), dtype=torch.float32, device=dev)
        self.Z = torch.empty((T_max, self.d), dtype=torch.float32, device=dev)
        self.T_max = T_max
        self.exchange = exchange
        self.peer = PeerAllReduce(self.P, self.Z, group) if exchange == "peer" and self.world > 1 else None

    def forward(self, X):
        T = X.shape[0]
        if T > self.T_max:
            raise ValueError(f"T={T} > T_max={self.T_max}")
        d, s = self.d, self.s
        tp.tp_column_linear(X, self.W1, self.Wu, self.b1, self.Y, T, d, s, 1, self.dtype, self.act)
        tp.tp_row_linear(self.Y, self.W2, self.P, T, s, d, 1, self.dtype)
        if self.world == 1:
            tp.tp_reduce_partials(self.P, self.b2, self.Z, T, d, 1)
        elif self.peer is not None:
            self.peer(self.b2, T, d)
        else:
            fixed_order_all_reduce(self.P[:T], self.b2, self.Z[:T], self.group)
        return self.Z[:T]

    def close(self) -> None:
        if self.peer is not None:
            self.peer.close()
            self.peer = None
