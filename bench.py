"""Benchmark of the sharded Megatron MLP block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gpt2|toy|wide|decode|llama]
                    [--mode partials|splitk] [--impl tp|reference]

One step = one pass of the whole hot path over one batch of synthetic input:
tp_mlp_block, i.e. the column-parallel GEMM + activation (all p shards), the
row-parallel GEMM to p fp32 partials and the fixed-order partial-sum
reduction (one persistent launch on the bf16 path).  The step is captured
once as a CUDA graph and replayed; CUDA events on the launching stream
bracket each replay.  A second loop times the same block as the three
separate C-ABI calls, with events between them, for the per-kernel
breakdown (column GEMM, row GEMM, reduction GB/s).  L2 is flushed (a 256 MiB
write) before every step, outside the events.

With N > 1 (torchrun) every rank runs an independent replica on its own GPU:
the block is single-GPU by design (the p shards are simulated on one device),
so there is no data-path collective; the step time is the max over ranks and
`value` counts the work of all ranks ("scaling": "weak").

`--impl reference` times the CPU oracle (float64 numpy) on the host cores on a
bounded token-row sample of the same workload, in the same metric.
"""

from __future__ import annotations

import argparse
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "sharded-MLP TFLOP/s & % BF16 tensor peak; partial-sum reduce HBM GB/s"
UNIT = "TFLOP/s"
FALLBACK_PEAKS = {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0}
L2_FLUSH_BYTES = 256 << 20


# ----------------------------------------------------------------------------- helpers

def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        with open(path) as f:
            d = json.load(f)
        return {k: float(d[k]) for k in FALLBACK_PEAKS}, "measured"
    except Exception:
        return dict(FALLBACK_PEAKS), "fallback"


def whole_job_value(units_per_step_per_rank: float, n_ranks: int, ms_per_step_max: float) -> float:
    """Aggregate throughput: the work of all ranks over the slowest rank's time."""
    return units_per_step_per_rank * n_ranks / (ms_per_step_max * 1e-3)


def reduce_max(values, dist=None, device=None):
    """Element-wise max of a list of floats over all ranks (identity without a group)."""
    if dist is None or not dist.is_initialized() or dist.get_world_size() == 1:
        return list(values)
    import torch
    t = torch.tensor(list(values), dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return t.cpu().tolist()


def reduce_bytes(w: WL.Workload) -> int:
    """Algorithmic HBM bytes of the reduction: read p partials, write Z (+ b2)."""
    return (w.p + 1) * w.T * w.d * 4 + (w.d * 4 if w.has_b2 else 0)


def column_flops(w: WL.Workload) -> int:
    return 2 * w.T * w.d * w.k * (2 if w.act == "swiglu" else 1)


def row_flops(w: WL.Workload) -> int:
    return 2 * w.T * w.k * w.d


def column_bytes(w: WL.Workload) -> int:
    e = 2 if w.dtype == "bf16" else 4
    nw = 2 if w.act == "swiglu" else 1
    return e * (w.T * w.d + nw * w.d * w.k + w.T * w.k + (w.k if w.has_b1 else 0))


def row_bytes(w: WL.Workload) -> int:
    e = 2 if w.dtype == "bf16" else 4
    return e * (w.T * w.k + w.k * w.d) + 4 * w.p * w.T * w.d


def block_bytes(w: WL.Workload) -> int:
    """Minimum HBM bytes of one block step: read X, the weights and biases
    once, write Z.  (The hidden shards and partials of this design add
    2*T*k*e + 2*p*T*d*4 bytes on top when they leave L2.)"""
    e = 2 if w.dtype == "bf16" else 4
    nw = 2 if w.act == "swiglu" else 1
    return (e * (w.T * w.d + nw * w.d * w.k + w.k * w.d + (w.k if w.has_b1 else 0))
            + 4 * w.T * w.d + (4 * w.d if w.has_b2 else 0))


def blas_threads() -> int:
    try:
        from threadpoolctl import threadpool_info
        n = [i.get("num_threads", 0) for i in threadpool_info() if i.get("user_api") == "blas"]
        if n:
            return int(max(n))
    except Exception:
        pass
    return os.cpu_count() or 1


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region."""

    QUERY = ("index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.path = os.path.join(ROOT, "gpurun_out", f"clocks_gpu{gpu_index}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", "100"],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        time.sleep(0.3)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.2)
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        rows = []
        for line in open(self.path):
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 9:
                continue
            try:
                rows.append((float(parts[1]), float(parts[2]), float(parts[3]) if parts[3] not in ("[N/A]", "N/A") else 0.0, parts[5:9]))
            except ValueError:
                continue
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows for i, v in enumerate(r[3]) if v.lower() == "active"})
        loaded = [r for r in rows if r[2] > 0.5 * max(x[2] for x in rows)] or rows
        return {"sm_mhz": statistics.median(r[0] for r in loaded), "sm_max_mhz": max(r[1] for r in rows),
                "reasons": reasons, "samples": len(rows)}


def ncu_traffic(kernel_key: str):
    """dram bytes per launch from the committed ncu summary table, if it was
    taken on the current kernel sources (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except Exception:
        return None
    ent = table.get(kernel_key)
    if not ent:
        return None
    h = hashlib.sha256()
    try:
        for src in ent["sources"]:
            with open(os.path.join(ROOT, "megatron_tensor_sharded_b200", "csrc", src), "rb") as f:
                h.update(f.read())
    except (OSError, KeyError):
        return None
    if h.hexdigest()[:16] != ent.get("source_sha"):
        return None
    return ent.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- CPU oracle arm

def oracle_sample_rows(w: WL.Workload, target_flops: float = 4e10) -> int:
    per_row = w.gemm_flops() / w.T
    return int(max(1, min(w.T, target_flops // per_row)))


def time_oracle(w: WL.Workload, inp: WL.Inputs, rows: int, min_seconds: float, max_reps: int):
    """Time the oracle (as it stands) on the first `rows` token rows; returns
    (seconds per rep, reps)."""
    from oracle import tp_oracle as O
    X = inp.values("X")[:rows]
    args = (inp.values("W1"), inp.values("b1"), inp.values("W2"), inp.values("b2"))
    Wu = inp.values("W_up")
    reps, t0 = 0, time.perf_counter()
    while True:
        O.mlp_sharded(X, args[0], args[1], args[2], args[3], w.p, w.act, W_up=Wu)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            return el / reps, reps


def run_reference(a, w: WL.Workload, rank: int, world: int):
    if rank != 0:
        return 0
    inp = WL.make_inputs(w)
    rows = oracle_sample_rows(w)
    flops = w.gemm_flops() * rows / w.T
    for _ in range(a.warmup):
        time_oracle(w, inp, rows, 0.0, 1)
    times = []
    for _ in range(a.steps):
        t, _ = time_oracle(w, inp, rows, 0.0, 1)
        times.append(t)
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    sample = f"first {rows} of {w.T} token rows per step, full weights, p={w.p}"
    line = {
        "impl": "reference", "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "k": w.k, "p": w.p, "act": w.act,
                   "sample_rows": rows, "parallelism": "replicas" if world > 1 else "single"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": sample},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


# ----------------------------------------------------------------------------- GPU arm

def run_tp(a, w: WL.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    import megatron_tensor_sharded_b200 as tp

    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    inp = WL.make_inputs(w)

    def dev(x):
        if x is None:
            return None
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(x).to(device)

    X, W1, Wu, b1, W2 = dev(inp.X), dev(inp.W1), dev(inp.W_up), dev(inp.b1), dev(inp.W2)
    b2 = dev(inp.b2)
    dtype = tp.DTYPE[w.dtype]
    act = tp.ACT[w.act]
    hdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
    Y = torch.empty((w.p, w.T, w.s), dtype=hdt, device=device)
    P = torch.empty((w.p, w.T, w.d), dtype=torch.float32, device=device)
    Z = torch.empty((w.T, w.d), dtype=torch.float32, device=device)
    flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
    stream = torch.cuda.current_stream(device)
    flags = tp.TP_FLAG_SPLITK_FUSED if a.mode == "splitk" else tp.TP_FLAG_NONE
    if a.mode == "fused":
        flags = tp.TP_FLAG_FUSED_LAUNCH
    nbytes = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, w.p, dtype, act, flags)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def block_step(st):
        tp.tp_mlp_block(X, W1, Wu, b1, W2, b2, Z, ws, nbytes, w.T, w.d, w.k, w.p, dtype, act,
                        flags, stream=st)

    def calls_step(st, ev):
        ev[0].record(st)
        tp.tp_column_linear(X, W1, Wu, b1, Y, w.T, w.d, w.k, w.p, dtype, act, stream=st)
        ev[1].record(st)
        tp.tp_row_linear(Y, W2, P, w.T, w.k, w.d, w.p, dtype, stream=st)
        ev[2].record(st)
        tp.tp_reduce_partials(P, b2, Z, w.T, w.d, w.p, stream=st)
        ev[3].record(st)

    def capture(fn):
        """Warm up eagerly, then capture one step as a CUDA graph; returns
        (graph, kernels of this library per step)."""
        for _ in range(a.warmup):
            flush.zero_()
            fn(stream)
        tp.tp_sync_status(stream)
        if a.no_graph:
            return None, None
        g = torch.cuda.CUDAGraph()
        n0 = tp.tp_kernel_launch_count()
        with torch.cuda.graph(g):
            fn(torch.cuda.current_stream())
        per_step = tp.tp_kernel_launch_count() - n0
        for _ in range(a.warmup):
            flush.zero_()
            g.replay()
        torch.cuda.synchronize(device)
        return g, per_step

    # ---- the timed region: K steps of the block, one graph replay each
    g_block, k_block = capture(block_step)
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    step_ms = []
    with ClockSampler(local_rank) as clocks:
        barrier()
        torch.cuda.synchronize(device)
        n0 = tp.tp_kernel_launch_count()
        t_wall = time.perf_counter()
        for _ in range(a.steps):
            flush.zero_()
            e0.record(stream)
            if g_block is not None:
                g_block.replay()
            else:
                block_step(stream)
            e1.record(stream)
            torch.cuda.synchronize(device)
            step_ms.append(e0.elapsed_time(e1))
        t_wall = time.perf_counter() - t_wall
        launches = tp.tp_kernel_launch_count() - n0
        if g_block is not None:
            launches = k_block * a.steps
        barrier()
    tp.tp_sync_status(stream)
    ms_step, launches = reduce_max([statistics.mean(step_ms), float(launches)],
                                   dist if world > 1 else None, device)

    # ---- per-kernel breakdown of the same block as three separate calls
    kernels = None
    if a.mode == "partials" and not a.no_breakdown:
        evs = [torch.cuda.Event(enable_timing=True, external=not a.no_graph) for _ in range(4)]
        g_calls, _ = capture(lambda st: calls_step(st, evs))
        col_ms, row_ms, red_ms, sum_ms = [], [], [], []
        barrier()
        for _ in range(a.steps):
            flush.zero_()
            if g_calls is not None:
                g_calls.replay()
            else:
                calls_step(stream, evs)
            torch.cuda.synchronize(device)
            col_ms.append(evs[0].elapsed_time(evs[1]))
            row_ms.append(evs[1].elapsed_time(evs[2]))
            red_ms.append(evs[2].elapsed_time(evs[3]))
            sum_ms.append(evs[0].elapsed_time(evs[3]))
        barrier()
        tp.tp_sync_status(stream)
        kernels = dict(zip(["column", "row", "reduce", "sum"],
                           reduce_max([statistics.mean(x) for x in (col_ms, row_ms, red_ms, sum_ms)],
                                      dist if world > 1 else None, device)))

    # ---- end to end through the public block call, inputs from pinned host memory
    e2e = None
    if not a.no_e2e:
        Xh = X.cpu().pin_memory()
        Zh = torch.empty(Z.shape, dtype=Z.dtype).pin_memory()
        Xd = torch.empty_like(X)

        def e2e_step():
            Xd.copy_(Xh, non_blocking=True)
            tp.tp_mlp_block(Xd, W1, Wu, b1, W2, b2, Z, ws, nbytes, w.T, w.d, w.k, w.p, dtype, act,
                            flags, stream=stream)
            Zh.copy_(Z, non_blocking=True)

        for _ in range(a.warmup):
            flush.zero_()
            e2e_step()
        torch.cuda.synchronize(device)
        barrier()
        t_e2e = []
        for _ in range(a.steps):
            flush.zero_()
            e0.record(stream)
            e2e_step()
            e1.record(stream)
            torch.cuda.synchronize(device)
            t_e2e.append(e0.elapsed_time(e1))
        barrier()
        tp.tp_sync_status(stream)
        e_ms = reduce_max([statistics.mean(t_e2e)], dist if world > 1 else None, device)[0]
        e2e = {"value": whole_job_value(w.gemm_flops(), world, e_ms) / 1e12, "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": Xh.numel() * Xh.element_size(),
               "d2h_bytes_per_step": Zh.numel() * Zh.element_size(),
               "call": "tp_mlp_block, X host->device and Z device->host inside the timed step"}

    peaks, peak_src = load_peaks()
    value = whole_job_value(w.gemm_flops(), world, ms_step) / 1e12
    kernel_name = {"partials": "tp_mlp_block: column GEMM -> row GEMM -> fixed-order fold (PDL-chained)",
                   "splitk": "tp_mlp_block split-K: column GEMM -> row GEMM accumulating all shards",
                   "fused": "tc_block_kernel (both GEMM layers, one launch) -> fold"}[a.mode]
    # Roofline side: tensor peak unless the step's arithmetic intensity
    # (FLOPs per minimum HBM byte) is below the measured ridge point.
    intensity = w.gemm_flops() / block_bytes(w)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if w.dtype == "bf16" and intensity >= ridge:
        achieved = w.gemm_flops() / (ms_step * 1e-3) / 1e12
        peak = peaks["bf16_tflops"]
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
                "frac": achieved / peak, "traffic": ncu_traffic(f"{w.name}/{a.mode}"),
                "kernel": kernel_name,
                "duration": "block step time (graph replay, CUDA events on the launching stream)",
                "traffic_scope": "dram bytes of all kernels of one step (ncu)",
                "peak_source": f"{peak_src} bf16 dense (burst)"}
    else:
        achieved = block_bytes(w) / (ms_step * 1e-3) / 1e9
        peak = peaks["hbm_gbs"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s",
                "frac": achieved / peak, "traffic": ncu_traffic(f"{w.name}/{a.mode}"),
                "kernel": kernel_name, "bytes_per_step": block_bytes(w),
                "duration": "block step time (graph replay, CUDA events on the launching stream)",
                "peak_source": f"{peak_src} hbm copy"}
    roof["intensity_flop_per_byte"] = intensity
    roof["ridge_flop_per_byte"] = ridge

    breakdown = None
    if kernels is not None:
        def tfl(f, ms):
            return f / (ms * 1e-3) / 1e12
        breakdown = {
            "column": {"ms": kernels["column"], "TFLOP/s": tfl(column_flops(w), kernels["column"]),
                       "frac_bf16_peak": tfl(column_flops(w), kernels["column"]) / peaks["bf16_tflops"]},
            "row": {"ms": kernels["row"], "TFLOP/s": tfl(row_flops(w), kernels["row"]),
                    "frac_bf16_peak": tfl(row_flops(w), kernels["row"]) / peaks["bf16_tflops"]},
            "reduce": {"ms": kernels["reduce"], "GB/s": reduce_bytes(w) / (kernels["reduce"] * 1e-3) / 1e9,
                       "frac_hbm": reduce_bytes(w) / (kernels["reduce"] * 1e-3) / 1e9 / peaks["hbm_gbs"],
                       "bytes": reduce_bytes(w)},
            "step_ms": kernels["sum"],
            "how": "the three C-ABI calls as one graph, external timing events between them",
        }

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "k": w.k, "p": w.p, "act": w.act,
                   "mode": a.mode, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "launch": "eager" if g_block is None else "cuda-graph replay of tp_mlp_block",
                   "l2": "flushed before every step (256 MiB write, outside the timed events)"},
        "pct_bf16_peak": 100.0 * value / (peaks["bf16_tflops"] * world) if w.dtype == "bf16" else None,
        "reduce": None if breakdown is None else breakdown["reduce"],
        "unfused_breakdown": breakdown,
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rows = min(w.T, oracle_sample_rows(w))
        sec, reps = time_oracle(w, inp, rows, min_seconds=10.0, max_reps=1000)
        line["cpu_baseline"] = {"value": w.gemm_flops() * rows / w.T / sec / 1e12, "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": f"first {rows} of {w.T} token rows, {reps} reps, float64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def main(argv=None):
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=20)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["tp", "reference"], default="tp")
    ap.add_argument("--workload", choices=sorted(WL.WORKLOADS), default="gpt2")
    ap.add_argument("--mode", choices=["partials", "splitk", "fused"], default="partials")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of graph replay")
    ap.add_argument("--no-breakdown", action="store_true", help="skip the per-kernel loop")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != a.gpus:
        ap.error(f"--gpus {a.gpus} but WORLD_SIZE={world}")
    w = WL.WORKLOADS[a.workload]
    if a.impl == "reference":
        return run_reference(a, w, rank, world)
    return run_tp(a, w, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
