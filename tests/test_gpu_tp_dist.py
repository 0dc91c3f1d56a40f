"""The p-GPU version of the block, checked on one GPU.

Ranks whose kernels wait on each other cannot share one GPU, so the p ranks
are emulated the way the pages' own walkthrough simulates them: p separate
buffers on one device.  Each emulated rank runs the column and row layers on
its own weight blocks (one local shard), and tp_reduce_partials_gather is
then called once per rank, as that rank would call it, with the p partial
buffers in shard order and every rank's output as a destination.  Every
output must equal the single-GPU fixed-order fold bit for bit, and the
block must match the oracle within the bf16 tolerance.

Also: the gather-fold on its own against tp_reduce_partials (vector and
scalar paths, slabs, ragged widths, b2), its argument checks, the
single-rank TensorParallelMLP, and CUDA IPC between two processes on the
same GPU (the second process maps the first one's buffer and folds from it;
the processes only wait for each other on the host)."""

import os
import subprocess
import sys
import textwrap

import numpy as np
import pytest
import torch

import megatron_tensor_sharded_b200 as tp
from megatron_tensor_sharded_b200 import tp_dist
import workloads as W
from gpu_util import bits, dev, host_f32
from oracle import tp_oracle as O

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _fold_ref(P, b2, T, d, p):
    Z = torch.full((T, d), float("nan"), device="cuda")
    tp.tp_reduce_partials(P, b2, Z, T, d, p)
    return Z


@pytest.mark.parametrize("p,T,d,with_b2", [
    (1, 5, 64, False), (2, 33, 256, True), (3, 17, 1000, True), (8, 64, 8192, False),
    (8, 19, 1001, True), (16, 9, 128, True), (5, 7, 6, False),
])
def test_gather_fold_is_the_fixed_order_fold(p, T, d, with_b2):
    g = torch.Generator(device="cuda").manual_seed(1000 * p + T)
    parts = [torch.randn(T, d, device="cuda", generator=g) for _ in range(p)]
    b2 = torch.randn(d, device="cuda", generator=g) if with_b2 else None
    want = host_f32(_fold_ref(torch.stack(parts), b2, T, d, p))
    outs = [torch.full((T, d), float("nan"), device="cuda") for _ in range(3)]
    for r0, rows in tp_dist.row_slabs(T, p):
        tp.tp_reduce_partials_gather(parts, b2, outs, r0, rows, d)
    tp.tp_sync_status()
    for o in outs:
        assert np.array_equal(bits(host_f32(o)), bits(want))
    # the oracle agrees too
    P = np.stack([host_f32(x) for x in parts])
    ref = O.reduce_partials_fixed_order(P, None if b2 is None else host_f32(b2))
    assert np.array_equal(bits(want), bits(ref))


def test_gather_fold_touches_only_the_slab():
    T, d, p = 12, 64, 2
    parts = [torch.randn(T, d, device="cuda") for _ in range(p)]
    out = torch.full((T, d), 7.0, device="cuda")
    tp.tp_reduce_partials_gather(parts, None, [out], 4, 3, d)
    tp.tp_sync_status()
    o = host_f32(out)
    assert np.all(o[:4] == 7.0) and np.all(o[7:] == 7.0)
    assert not np.any(o[4:7] == 7.0)


def test_gather_fold_argument_checks():
    x = torch.zeros(8, 8, device="cuda")
    y = torch.zeros(8, 8, device="cuda")
    call = lambda parts, outs, r0=0, rows=8, d=8: tp.tp_reduce_partials_gather(  # noqa: E731
        parts, None, outs, r0, rows, d, check=False)
    assert call([], [y]) == 1
    assert call([x] * 17, [y]) == 1
    assert call([x], []) == 1
    assert call([x], [x]) == 1                       # output overlaps a partial
    assert call([x], [y], r0=-1) == 1
    assert call([x.data_ptr() + 2], [y]) == 3        # misaligned
    assert call([x], [y], rows=0) == 0               # nothing to do


def _emulated_ranks(name, p, seed=42):
    """Column + row layers of each emulated rank on its own weight blocks."""
    w = W.WORKLOADS[name]
    inp = W.make_inputs(w, seed=seed)
    X, W1, Wu, b1, W2 = dev(inp.X), dev(inp.W1), dev(inp.W_up), dev(inp.b1), dev(inp.W2)
    b2 = dev(inp.b2)
    s = w.k // p
    P = []
    for r in range(p):
        w1, wu, bb, w2 = tp_dist.shard_weights(W1, Wu, b1, W2, r, p)
        Y = torch.empty(w.T, s, dtype=torch.bfloat16, device="cuda")
        Pr = torch.empty(w.T, w.d, device="cuda")
        tp.tp_column_linear(X, w1, wu, bb, Y, w.T, w.d, s, 1, tp.TP_BF16, tp.ACT[w.act])
        tp.tp_row_linear(Y, w2, Pr, w.T, s, w.d, 1, tp.TP_BF16)
        P.append(Pr)
    return w, inp, (X, W1, Wu, b1, W2, b2), P


@pytest.mark.parametrize("name,p", [("gpt2", 2), ("gpt2", 4), ("wide", 4), ("llama", 8)])
def test_emulated_p_gpu_block(name, p):
    w, inp, (X, W1, Wu, b1, W2, b2), P = _emulated_ranks(name, p)
    Z = [torch.full((w.T, w.d), float("nan"), device="cuda") for _ in range(p)]
    for r, (r0, rows) in enumerate(tp_dist.row_slabs(w.T, p)):
        parts, outs, row0, nrows = tp_dist.peer_tables(r, p, P, Z, w.T)
        tp.tp_reduce_partials_gather(parts, b2, outs, row0, nrows, w.d)
    tp.tp_sync_status()
    fold = host_f32(_fold_ref(torch.stack(P), b2, w.T, w.d, p))
    for z in Z:
        assert np.array_equal(bits(host_f32(z)), bits(fold))
    # the same block on one GPU with p simulated shards
    ws_n = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, p, tp.TP_BF16, tp.ACT[w.act])
    ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
    Z1 = torch.empty(w.T, w.d, device="cuda")
    tp.tp_mlp_block(X, W1, Wu, b1, W2, b2, Z1, ws, ws_n, w.T, w.d, w.k, p, tp.TP_BF16,
                    tp.ACT[w.act])
    tp.tp_sync_status()
    z0 = host_f32(Z[0])
    assert np.array_equal(bits(z0), bits(host_f32(Z1)))
    # and the oracle (sampled rows at the large sizes)
    rows = np.arange(w.T) if w.T * w.k <= 1024 * 3072 else np.arange(0, w.T, 97)
    want = O.mlp_sharded(inp.values("X")[rows], inp.values("W1"), inp.values("b1"),
                         inp.values("W2"), inp.values("b2"), p, w.act,
                         W_up=inp.values("W_up"))["Z"]
    assert O.rel_err(z0[rows], want) <= 1e-2


def _init_single_rank_group(tmp_path):
    import torch.distributed as dist
    if dist.is_initialized():
        return False
    store = dist.FileStore(str(tmp_path / "store"), 1)
    dist.init_process_group("nccl", store=store, rank=0, world_size=1,
                            device_id=torch.device("cuda", 0))
    return True


def test_single_rank_exchanges_and_block(tmp_path):
    """World size 1 over NCCL: both exchanges reduce to the one-shard fold,
    and TensorParallelMLP to tp_mlp_block with p = 1, bit for bit."""
    import torch.distributed as dist
    created = _init_single_rank_group(tmp_path)
    try:
        T, d = 300, 512
        P = torch.randn(T, d, device="cuda")
        b2 = torch.randn(d, device="cuda")
        want = host_f32(_fold_ref(P, b2, T, d, 1))
        Z = torch.full((T, d), float("nan"), device="cuda")
        tp_dist.fixed_order_all_reduce(P, b2, Z)
        torch.cuda.synchronize()
        assert np.array_equal(bits(host_f32(Z)), bits(want))
        Z2 = torch.full((T, d), float("nan"), device="cuda")
        peer = tp_dist.PeerAllReduce(P, Z2)
        peer(b2, T, d)
        peer.close()
        torch.cuda.synchronize()
        assert np.array_equal(bits(host_f32(Z2)), bits(want))

        w = W.WORKLOADS["gpt2"]
        inp = W.make_inputs(w, seed=7)
        X, W1, b1, W2, b2 = dev(inp.X), dev(inp.W1), dev(inp.b1), dev(inp.W2), dev(inp.b2)
        ws_n = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, 1, tp.TP_BF16, tp.TP_ACT_GELU_TANH)
        ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
        Z1 = torch.empty(w.T, w.d, device="cuda")
        tp.tp_mlp_block(X, W1, None, b1, W2, b2, Z1, ws, ws_n, w.T, w.d, w.k, 1, tp.TP_BF16,
                        tp.TP_ACT_GELU_TANH)
        for exchange in ("nccl", "peer"):
            m = tp_dist.TensorParallelMLP(W1, None, b1, W2, b2, tp.TP_ACT_GELU_TANH, w.T,
                                          exchange=exchange)
            Zm = host_f32(m.forward(X))
            m.close()
            tp.tp_sync_status()
            assert np.array_equal(bits(Zm), bits(host_f32(Z1))), exchange
    finally:
        if created:
            dist.destroy_process_group()


_EXPORTER = textwrap.dedent("""
    import sys, time, torch
    sys.path.insert(0, {root!r})
    import megatron_tensor_sharded_b200 as tp
    torch.cuda.set_device(0)
    P = torch.arange(4 * 64, dtype=torch.float32, device="cuda").reshape(4, 64) * 0.5
    torch.cuda.synchronize()
    h0 = tp.tp_ipc_export(P)
    h = tp.tp_ipc_export(P[1:])          # a buffer that starts 256 bytes further in
    assert h.offset == h0.offset + 64 * 4 and h.bytes[:] == h0.bytes[:]
    sys.stdout.write(h.to_bytes().hex() + "\\n")
    sys.stdout.flush()
    sys.stdin.readline()                 # wait until the importer is done
""")


def test_ipc_export_import_between_processes():
    proc = subprocess.Popen([sys.executable, "-c", _EXPORTER.format(root=ROOT)],
                            stdin=subprocess.PIPE, stdout=subprocess.PIPE, text=True)
    try:
        line = proc.stdout.readline().strip()
        assert line, "exporter printed no handle"
        h = tp.IpcHandle.from_bytes(bytes.fromhex(line))
        assert h.offset % 256 == 0 and h.size >= h.offset + 3 * 64 * 4
        addr = tp.tp_ipc_import(h)
        addr2 = tp.tp_ipc_import(h)       # the same allocation: one mapping
        assert addr == addr2
        out = torch.full((3, 64), float("nan"), device="cuda")
        tp.tp_reduce_partials_gather([addr], None, [out], 0, 3, 64)
        tp.tp_sync_status()
        want = (np.arange(4 * 64, dtype=np.float32).reshape(4, 64) * 0.5)[1:]
        assert np.array_equal(host_f32(out), want)
        tp.tp_ipc_release(h)
        tp.tp_ipc_release(h)
        with pytest.raises(tp.TPError):
            tp.tp_ipc_release(h)
    finally:
        proc.stdin.write("done\n")
        proc.stdin.flush()
        proc.wait(timeout=60)
    assert proc.returncode == 0


def _two_rank_worker(rank, world, port, out):
    """One of two processes on the same GPU: gloo for the host-side
    plumbing (handle exchange and the stream-ordered barriers, which for a
    CUDA tensor wait for the stream's earlier kernels), CUDA IPC for the peer
    mappings.  No kernel of one process waits on the other's."""
    import datetime
    import torch.distributed as dist
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    torch.cuda.set_device(0)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    try:
        res = {}
        # the block: each process runs its own shard, the peer exchange sums
        w = W.WORKLOADS["gpt2"]
        inp = W.make_inputs(w, seed=11)
        X, W1, b1, W2, b2 = dev(inp.X), dev(inp.W1), dev(inp.b1), dev(inp.W2), dev(inp.b2)
        w1, _, bb, w2 = tp_dist.shard_weights(W1, None, b1, W2, rank, world)
        m = tp_dist.TensorParallelMLP(w1, None, bb, w2, b2, tp.TP_ACT_GELU_TANH, w.T,
                                      exchange="peer")
        Z = host_f32(m.forward(X)).copy()
        torch.cuda.synchronize()
        dist.barrier()          # both processes are done reading each other's buffers
        m.close()
        ws_n = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, world, tp.TP_BF16, tp.TP_ACT_GELU_TANH)
        ws = torch.empty(ws_n, dtype=torch.uint8, device="cuda")
        Z1 = torch.empty(w.T, w.d, device="cuda")
        tp.tp_mlp_block(X, W1, None, b1, W2, b2, Z1, ws, ws_n, w.T, w.d, w.k, world, tp.TP_BF16,
                        tp.TP_ACT_GELU_TANH)
        tp.tp_sync_status()
        res["block_same_bits"] = bool(np.array_equal(bits(Z), bits(host_f32(Z1))))
        # the exchange alone on ragged sizes: rank r's partial drawn from seed r
        T, d = 301, 1000
        g = torch.Generator(device="cuda").manual_seed(100 + rank)
        P = torch.randn(T, d, device="cuda", generator=g)
        Zx = torch.full((T, d), float("nan"), device="cuda")
        bx = torch.randn(d, device="cuda", generator=torch.Generator(device="cuda").manual_seed(7))
        peer = tp_dist.PeerAllReduce(P, Zx)
        peer(bx, T, d)
        torch.cuda.synchronize()
        dist.barrier()
        peer.close()
        Ps = [torch.randn(T, d, device="cuda",
                          generator=torch.Generator(device="cuda").manual_seed(100 + r))
              for r in range(world)]
        want = _fold_ref(torch.stack(Ps), bx, T, d, world)
        tp.tp_sync_status()
        res["exchange_same_bits"] = bool(np.array_equal(bits(host_f32(Zx)), bits(host_f32(want))))
        out[rank] = res
    finally:
        dist.destroy_process_group()


def test_two_processes_on_one_gpu_peer_exchange():
    """The "peer" exchange with world size 2, the two ranks being two
    processes on the same GPU: every rank's output has the bits of the
    single-GPU block with p = 2, and the exchange alone of the fixed-order
    fold of both partials (+ b2)."""
    import socket
    import torch.multiprocessing as mp
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    mgr = mp.get_context("spawn").Manager()   # never fork a process that has used CUDA
    out = mgr.dict()
    mp.spawn(_two_rank_worker, args=(2, port, out), nprocs=2, join=True)
    for r in range(2):
        assert out[r] == {"block_same_bits": True, "exchange_same_bits": True}, (r, out[r])
