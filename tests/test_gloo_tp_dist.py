"""The p-GPU all-reduce of the partials, exercised on CPU ranks (gloo).

Each rank holds its own full-shape partial P_r; the "nccl" exchange of
megatron_tensor_sharded_b200.tp_dist (all-to-all of row slabs, a fold of the
rank's slab in rank order, all-gather of the slabs) must give every rank the
oracle's fixed-order fold of all the partials, bit for bit.  On the host the
fold step is the oracle's (the CUDA fold is checked against the same oracle
by the GPU tests); what runs here is the exchange: which rows go where, in
which order the shards meet, and the padding of uneven slabs.

Also the host-side pieces of the "peer" exchange (slabs, pointer tables) and
the weight sharding."""

import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

from megatron_tensor_sharded_b200 import tp_dist
from oracle import tp_oracle as O


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _partials(world, T, d, seed):
    """The partials of every rank, with values chosen so that the fold order
    matters: large cancelling terms, ties at 2^24, signed zeros."""
    rng = np.random.default_rng(seed)
    P = (rng.standard_normal((world, T, d)) * rng.choice([1.0, 1e8, 1e-3], size=(world, T, d)))
    P = P.astype(np.float32)
    if T and d >= 3:
        P[:, 0, 0] = [16777216.0 if j == 0 else 1.0 for j in range(world)]
        P[:, 0, 1] = -0.0
        P[:, 0, 2] = [1e8 if j % 2 == 0 else -1e8 for j in range(world)]
    return P


def _host_fold(parts, b2, out, rows, d, p):
    """Oracle fold of the received [p][rows][d] block into out[:rows]."""
    z = O.reduce_partials_fixed_order(parts.numpy(), None if b2 is None else b2.numpy())
    out[:rows].copy_(torch.from_numpy(z))


def _worker(rank, world, port, cases, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        res = {}
        for name, (T, d, with_b2, seed) in cases.items():
            P = _partials(world, T, d, seed)
            b2 = np.random.default_rng(seed + 1).standard_normal(d).astype(np.float32) if with_b2 else None
            Z = torch.full((T, d), float("nan"))
            tp_dist.fixed_order_all_reduce(torch.from_numpy(P[rank].copy()),
                                           None if b2 is None else torch.from_numpy(b2), Z,
                                           fold=_host_fold)
            res[name] = Z.numpy().copy()
        out[rank] = res
        dist.barrier()
    finally:
        dist.destroy_process_group()


CASES = {
    "even": (8, 12, False, 1),
    "ragged_rows": (7, 12, True, 2),
    "fewer_rows_than_ranks": (1, 5, True, 3),
    "no_rows": (0, 4, False, 4),
    "odd_width": (13, 3, True, 5),
}


@pytest.mark.parametrize("world", [2, 3])
def test_all_reduce_is_the_fixed_order_fold_on_every_rank(world):
    port = _free_port()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(world, port, CASES, out), nprocs=world, join=True)
    for name, (T, d, with_b2, seed) in CASES.items():
        P = _partials(world, T, d, seed)
        b2 = np.random.default_rng(seed + 1).standard_normal(d).astype(np.float32) if with_b2 else None
        want = O.reduce_partials_fixed_order(P, b2)
        for r in range(world):
            got = out[r][name]
            assert got.shape == (T, d)
            assert np.array_equal(got.view(np.uint32), want.view(np.uint32)), (name, r)


def test_row_slabs_partition_the_rows_in_rank_order():
    for T in range(0, 40):
        for world in range(1, 9):
            slabs = tp_dist.row_slabs(T, world)
            assert len(slabs) == world
            nxt = 0
            for r0, rows in slabs:
                assert rows >= 0 and r0 == min(T, nxt)
                nxt = r0 + rows
            assert nxt == T
            m = -(-T // world)
            assert all(rows <= m for _, rows in slabs)
    with pytest.raises(ValueError):
        tp_dist.row_slabs(4, 0)


def test_peer_tables_keep_shard_order_and_give_every_rank_its_slab():
    world, T = 4, 10
    p_ptrs = [1000 + 16 * r for r in range(world)]
    z_ptrs = [5000 + 16 * r for r in range(world)]
    covered = []
    for rank in range(world):
        parts, outs, row0, rows = tp_dist.peer_tables(rank, world, p_ptrs, z_ptrs, T)
        assert parts == p_ptrs          # P_0 .. P_{p-1}: the fold order
        assert sorted(outs) == sorted(z_ptrs)
        covered += list(range(row0, row0 + rows))
    assert covered == list(range(T))
    with pytest.raises(ValueError):
        tp_dist.peer_tables(0, world, p_ptrs[:3], z_ptrs, T)


def test_shard_weights_are_the_column_and_row_blocks():
    d, k, world = 6, 12, 3
    W1 = torch.arange(d * k, dtype=torch.float32).reshape(d, k)
    Wu = -W1
    b1 = torch.arange(k, dtype=torch.float32)
    W2 = torch.arange(k * d, dtype=torch.float32).reshape(k, d)
    s = k // world
    for r in range(world):
        w1, wu, bb, w2 = tp_dist.shard_weights(W1, Wu, b1, W2, r, world)
        assert torch.equal(w1, W1[:, r * s:(r + 1) * s]) and w1.is_contiguous()
        assert torch.equal(wu, Wu[:, r * s:(r + 1) * s])
        assert torch.equal(bb, b1[r * s:(r + 1) * s])
        assert torch.equal(w2, W2[r * s:(r + 1) * s, :]) and w2.is_contiguous()
    with pytest.raises(ValueError):
        tp_dist.shard_weights(W1[:, :11], None, None, W2[:11], 0, 2)
