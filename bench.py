"""Benchmark of the sharded Megatron MLP block on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--workload gpt2|toy|wide|decode|llama]
                    [--mode partials|splitk] [--impl tp|reference]
    python bench.py --workload attn_wide|attn_llama     (the attention block)
    python bench.py --workload block_wide|block_llama   (the transformer block)
    python bench.py --workload wide --mode backward     (the MLP block's backward pass)

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

The attention workloads time tp_attn_block the same way (one graph replay per
step: column Q, K, V projections, attention of every shard's heads,
row-parallel output projection, fold), with a per-call breakdown; the CPU
oracle runs on a causal prefix of the tokens (with a causal mask the first n
rows of the block depend only on the first n tokens).

The transformer-block workloads time tp_transformer_block (LayerNorm,
attention block with the residual folded into its reduction and the second
LayerNorm fused behind it, MLP block, reduction with the residual), with a
breakdown over the public calls run one after another.
"""

from __future__ import annotations

import argparse
import dataclasses
import datetime
import hashlib
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

import numpy as np  # noqa: E402

import workloads as WL  # noqa: E402

METRIC = "sharded-MLP TFLOP/s & % BF16 tensor peak; partial-sum reduce HBM GB/s"
ATTN_METRIC = "tensor-parallel attention block TFLOP/s & % BF16 tensor peak"
BLOCK_METRIC = "tensor-parallel transformer block TFLOP/s & % BF16 tensor peak"
BWD_METRIC = "sharded-MLP backward TFLOP/s & % BF16 tensor peak"
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
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed
    region: sampling starts (and its first line is waited for) before the
    region, every sample carries nvidia-smi's timestamp, and the summary keeps
    the samples taken between entering and leaving the context."""

    QUERY = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
             "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
             "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")
    PERIOD_MS = 20

    def __init__(self, gpu_index: int):
        self.gpu_index = gpu_index
        self.proc = None
        self.t0 = self.t1 = None
        # raw samples: $TP_BENCH_CLOCK_DIR if set (kept for inspection), else a
        # temporary directory
        out_dir = os.environ.get("TP_BENCH_CLOCK_DIR") or tempfile.gettempdir()
        self.path = os.path.join(out_dir, f"tp_bench_clocks_gpu{gpu_index}_{os.getpid()}.csv")

    def __enter__(self):
        try:
            os.makedirs(os.path.dirname(self.path), exist_ok=True)
            self.f = open(self.path, "w")
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu_index}", f"--query-gpu={self.QUERY}",
                 "--format=csv,noheader,nounits", "-lms", str(self.PERIOD_MS)],
                stdout=self.f, stderr=subprocess.DEVNULL)
        except Exception:
            self.proc = None
        # nvidia-smi takes a moment to start: wait (up to 3 s) for its first
        # line, so that the timed region is sampled from its start
        deadline = time.time() + 3.0
        while self.proc is not None and time.time() < deadline:
            self.f.flush()
            if os.path.getsize(self.path) > 0 or self.proc.poll() is not None:
                break
            time.sleep(0.01)
        self.t0 = time.time()
        return self

    def __exit__(self, *exc):
        self.t1 = time.time()
        if self.proc is not None:
            time.sleep(2.5 * self.PERIOD_MS / 1000.0)   # the sample in flight at t1
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except Exception:
                self.proc.kill()
            self.f.close()

    @staticmethod
    def parse(lines):
        """(unix time or None, sm MHz, max sm MHz, power W, [4 reason flags])
        per well-formed line of the query above."""
        import datetime
        rows = []
        for line in lines:
            parts = [x.strip() for x in line.split(",")]
            if len(parts) < 10:
                continue
            try:
                ts = datetime.datetime.strptime(parts[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
            except ValueError:
                ts = None
            try:
                rows.append((ts, float(parts[2]), float(parts[3]),
                             float(parts[4]) if parts[4] not in ("[N/A]", "N/A") else 0.0,
                             parts[6:10]))
            except ValueError:
                continue
        return rows

    @staticmethod
    def summarise(rows, t0=None, t1=None):
        """Median SM clock of the loaded samples inside [t0, t1] (all samples
        when none falls inside), the maximum clock, and every throttle reason
        seen in that window."""
        if not rows:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["no samples"]}
        window = "timed region"
        if t0 is not None and t1 is not None:
            slack = 0.03
            inside = [r for r in rows if r[0] is not None and t0 - slack <= r[0] <= t1 + slack]
            if inside:
                rows_w = inside
            else:
                rows_w, window = rows, "whole sampling (no sample inside the timed region)"
        else:
            rows_w = rows
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        reasons = sorted({names[i] for r in rows_w for i, v in enumerate(r[4]) if v.lower() == "active"})
        loaded = [r for r in rows_w if r[3] > 0.5 * max(x[3] for x in rows_w)] or rows_w
        return {"sm_mhz": statistics.median(r[1] for r in loaded),
                "sm_max_mhz": max(r[2] for r in rows), "reasons": reasons,
                "samples": len(rows_w), "window": window}

    def summary(self):
        if self.proc is None or not os.path.exists(self.path):
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        with open(self.path) as f:
            rows = self.parse(f)
        return self.summarise(rows, self.t0, self.t1)


def source_digest(files) -> str:
    """Digest of the kernels' device sources with comments and whitespace
    removed, so that a traffic figure stays tied to the code it was measured
    on, not to its comments."""
    import re
    h = hashlib.sha256()
    for src in files:
        with open(os.path.join(ROOT, "megatron_tensor_sharded_b200", "csrc", src)) as f:
            text = f.read()
        text = re.sub(r"/\*.*?\*/", " ", text, flags=re.S)
        text = re.sub(r"//[^\n]*", " ", text)
        h.update(" ".join(text.split()).encode())
    return h.hexdigest()[:16]


def ncu_traffic(kernel_key: str):
    """dram bytes per launch from the committed ncu summary table, if it was
    taken on the current kernel code (else None)."""
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    try:
        with open(path) as f:
            table = json.load(f)
    except Exception:
        return None
    ent = table.get(kernel_key)
    if not ent:
        return None
    try:
        digest = source_digest(ent["sources"])
    except (OSError, KeyError):
        return None
    if digest != ent.get("source_sha"):
        return None
    return ent.get("dram_bytes_per_launch")


# ----------------------------------------------------------------------------- CPU oracle arm

def oracle_sample_rows(w: WL.Workload, target_flops: float = 4e10) -> int:
    per_row = w.gemm_flops() / w.T
    return int(max(1, min(w.T, target_flops // per_row)))


def time_oracle(w: WL.Workload, inp: WL.Inputs, rows: int, min_seconds: float, max_reps: int,
                want_z: bool = False):
    """Time the oracle (as it stands) on the first `rows` token rows; returns
    (seconds per rep, reps), plus the oracle's Z rows with `want_z`."""
    from oracle import tp_oracle as O
    X = inp.values("X")[:rows]
    args = (inp.values("W1"), inp.values("b1"), inp.values("W2"), inp.values("b2"))
    Wu = inp.values("W_up")
    reps, t0 = 0, time.perf_counter()
    while True:
        z = O.mlp_sharded(X, args[0], args[1], args[2], args[3], w.p, w.act, W_up=Wu)["Z"]
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            return (el / reps, reps, z) if want_z else (el / reps, reps)


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


def attn_flops_prefix(w: WL.AttnWorkload, n: int) -> dict:
    """Algorithmic FLOPs of the block on the first n tokens."""
    return dataclasses.replace(w, T=n).flops()


def attn_oracle_rows(w: WL.AttnWorkload, target_flops: float = 3e10) -> int:
    n = 16
    while n < w.T and attn_flops_prefix(w, min(w.T, 2 * n))["total"] <= target_flops:
        n *= 2
    return min(n, w.T)


def time_attn_oracle(w: WL.AttnWorkload, inp, rows: int, min_seconds: float, max_reps: int):
    from oracle import tp_oracle as O
    X = inp.values("X")[:rows]
    args = (inp.values("Wq"), inp.values("Wk"), inp.values("Wv"), inp.values("Wo"), inp.bo)
    reps, t0 = 0, time.perf_counter()
    while True:
        O.attention_sharded(X, *args, w.p, w.n_heads, w.n_kv_heads, w.head_dim, w.causal)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            return el / reps, reps


def attn_config(w: WL.AttnWorkload, world: int) -> dict:
    return {"workload": w.name, "T": w.T, "d": w.d, "n_heads": w.n_heads,
            "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "p": w.p, "causal": w.causal,
            "parallelism": f"replicas{world}" if world > 1 else "single"}


def run_reference_attn(a, w: WL.AttnWorkload, rank: int, world: int):
    if rank != 0:
        return 0
    inp = WL.make_attn_inputs(w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim)
    rows = attn_oracle_rows(w)
    flops = attn_flops_prefix(w, rows)["total"]
    for _ in range(a.warmup):
        time_attn_oracle(w, inp, rows, 0.0, 1)
    times = [time_attn_oracle(w, inp, rows, 0.0, 1)[0] for _ in range(a.steps)]
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    cfg = attn_config(w, world)
    cfg["sample_rows"] = rows
    line = {
        "impl": "reference", "metric": ATTN_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"causal prefix: first {rows} of {w.T} tokens per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def block_flops_prefix(w: WL.BlockWorkload, n: int) -> dict:
    return dataclasses.replace(w, T=n).flops()


def block_oracle_rows(w: WL.BlockWorkload, target_flops: float = 3e10) -> int:
    n = 8
    while n < w.T and block_flops_prefix(w, min(w.T, 2 * n))["total"] <= target_flops:
        n *= 2
    return min(n, w.T)


def time_block_oracle(w: WL.BlockWorkload, inp, rows: int, min_seconds: float, max_reps: int):
    from oracle import tp_oracle as O
    X = inp.X[:rows]
    prm = inp.value_dict()
    reps, t0 = 0, time.perf_counter()
    while True:
        O.transformer_block_sharded(X, prm, w.p, w.n_heads, w.n_kv_heads, w.head_dim, w.act,
                                    w.causal)
        reps += 1
        el = time.perf_counter() - t0
        if el >= min_seconds or reps >= max_reps:
            return el / reps, reps


def block_config(w: WL.BlockWorkload, world: int) -> dict:
    return {"workload": w.name, "T": w.T, "d": w.d, "n_heads": w.n_heads,
            "n_kv_heads": w.n_kv_heads, "head_dim": w.head_dim, "k": w.k, "p": w.p, "act": w.act,
            "causal": w.causal, "parallelism": f"replicas{world}" if world > 1 else "single"}


def run_reference_block(a, w: WL.BlockWorkload, rank: int, world: int):
    if rank != 0:
        return 0
    inp = WL.make_block_inputs(w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, w.k, w.act)
    rows = block_oracle_rows(w)
    flops = block_flops_prefix(w, rows)["total"]
    for _ in range(a.warmup):
        time_block_oracle(w, inp, rows, 0.0, 1)
    times = [time_block_oracle(w, inp, rows, 0.0, 1)[0] for _ in range(a.steps)]
    ms = 1e3 * sum(times) / len(times)
    value = flops / (ms * 1e-3) / 1e12
    cfg = block_config(w, world)
    cfg["sample_rows"] = rows
    line = {
        "impl": "reference", "metric": BLOCK_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic", "config": cfg,
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"causal prefix: first {rows} of {w.T} tokens per step"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


class Harness:
    """Warm-up, CUDA-graph capture and the timed loop of the attention,
    transformer-block and backward arms."""

    def __init__(self, a, torch, tp, device, barrier):
        self.a, self.torch, self.tp, self.device, self.barrier = a, torch, tp, device, barrier
        self.stream = torch.cuda.current_stream(device)
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)

    def capture(self, fn, graph: bool):
        """Warm up eagerly, then (with `graph`) capture one step; returns
        (graph or None, library kernels per step or None)."""
        torch, tp = self.torch, self.tp
        for _ in range(self.a.warmup):
            self.flush.zero_()
            fn(self.stream)
        tp.tp_sync_status(self.stream)
        if not graph:
            return None, None
        g = torch.cuda.CUDAGraph()
        n0 = tp.tp_kernel_launch_count()
        with torch.cuda.graph(g):
            fn(torch.cuda.current_stream())
        per_step = tp.tp_kernel_launch_count() - n0
        for _ in range(self.a.warmup):
            self.flush.zero_()
            g.replay()
        torch.cuda.synchronize(self.device)
        return g, per_step

    def time_steps(self, fn, graph: bool = True, events=None):
        """K timed steps, L2 flushed before each (outside the events).  Returns
        the step times (ms), or with `events` (recorded inside the step) the
        per-step lists of their successive intervals; plus the library
        launches in the timed region and its wall time."""
        torch, tp = self.torch, self.tp
        g, per_step = self.capture(fn, graph and not self.a.no_graph)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        out = []
        self.barrier()
        torch.cuda.synchronize(self.device)
        n0 = tp.tp_kernel_launch_count()
        t_wall = time.perf_counter()
        for _ in range(self.a.steps):
            self.flush.zero_()
            e0.record(self.stream)
            if g is not None:
                g.replay()
            else:
                fn(self.stream)
            e1.record(self.stream)
            torch.cuda.synchronize(self.device)
            if events is None:
                out.append(e0.elapsed_time(e1))
            else:
                out.append([events[i].elapsed_time(events[i + 1]) for i in range(len(events) - 1)])
        t_wall = time.perf_counter() - t_wall
        launches = tp.tp_kernel_launch_count() - n0
        if g is not None:
            launches = per_step * self.a.steps
        self.barrier()
        tp.tp_sync_status(self.stream)
        return out, launches, t_wall


# ----------------------------------------------------------------------------- GPU arm

def clocks_capped(clk: dict) -> bool:
    """True when the SM clocks of a timed loop were held below their
    maximum: a median clock (of the samples inside the loop) under 90% of
    the maximum, the power-capped regime of the sustained GEMM figure.  A
    loop that touched the power cap but kept its median clock near the
    maximum is compared with the burst figure."""
    if not clk or clk.get("sm_mhz") is None or not clk.get("sm_max_mhz"):
        return False
    return clk["sm_mhz"] < 0.9 * clk["sm_max_mhz"]


def tensor_peak(peaks: dict, peak_src: str, clk: dict):
    """The bf16 denominator for a loop: the burst figure when the loop ran at
    (near) full clocks, the sustained (power-capped) figure when it did not."""
    if clocks_capped(clk):
        return peaks["bf16_tflops_sustained"], f"{peak_src} bf16 dense (sustained, power-capped loop)"
    return peaks["bf16_tflops"], f"{peak_src} bf16 dense (burst)"


def traffic_entry(key: str) -> dict:
    """roofline.traffic and where it comes from: the committed ncu table,
    keyed by workload/kernel and by a digest of the kernels' device code."""
    v = ncu_traffic(key)
    if v is None:
        return {"traffic": None,
                "traffic_source": f"none: no ncu figure for {key} on the current kernel code"}
    path = os.path.join(ROOT, "profiles", "ncu_traffic.json")
    with open(path) as f:
        ent = json.load(f)[key]
    return {"traffic": v,
            "traffic_source": f"profiles/ncu_traffic.json[{key}] (cold-cache ncu capture, "
                              f"device-code digest {ent['source_sha']})"}


class MlpBench:
    """Device buffers of one MLP workload and the timed loops over them: the
    block step (one CUDA-graph replay of tp_mlp_block) and the same block as
    the three separate C-ABI calls with events between them."""

    def __init__(self, a, torch, tp, w: WL.Workload, inp: WL.Inputs, device, mode: str, barrier,
                 dist, world: int):
        self.a, self.torch, self.tp, self.w, self.device = a, torch, tp, w, device
        self.barrier, self.dist, self.world = barrier, dist, world
        self.inp = inp

        def dev(x):
            if x is None:
                return None
            if x.dtype == np.uint16:
                return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
            return torch.from_numpy(x).to(device)

        self.X, self.W1, self.Wu, self.b1 = dev(inp.X), dev(inp.W1), dev(inp.W_up), dev(inp.b1)
        self.W2, self.b2 = dev(inp.W2), dev(inp.b2)
        self.dtype = tp.DTYPE[w.dtype]
        self.act = tp.ACT[w.act]
        hdt = torch.bfloat16 if w.dtype == "bf16" else torch.float32
        self.Y = torch.empty((w.p, w.T, w.s), dtype=hdt, device=device)
        self.P = torch.empty((w.p, w.T, w.d), dtype=torch.float32, device=device)
        self.Z = torch.empty((w.T, w.d), dtype=torch.float32, device=device)
        self.flush = torch.empty(L2_FLUSH_BYTES // 4, dtype=torch.float32, device=device)
        self.stream = torch.cuda.current_stream(device)
        self.mode = mode
        self.flags = {"partials": tp.TP_FLAG_NONE, "splitk": tp.TP_FLAG_SPLITK_FUSED,
                      "fused": tp.TP_FLAG_FUSED_LAUNCH, "fold": tp.TP_FLAG_ROW_FOLD}[mode]
        self.nbytes = tp.tp_mlp_block_workspace_size(w.T, w.d, w.k, w.p, self.dtype, self.act,
                                                     self.flags)
        self.ws = torch.empty(self.nbytes, dtype=torch.uint8, device=device)
        self.evs = None

    def block_step(self, st):
        w, tp = self.w, self.tp
        tp.tp_mlp_block(self.X, self.W1, self.Wu, self.b1, self.W2, self.b2, self.Z, self.ws,
                        self.nbytes, w.T, w.d, w.k, w.p, self.dtype, self.act, self.flags,
                        stream=st)

    def calls_step(self, st):
        w, tp, ev = self.w, self.tp, self.evs
        ev[0].record(st)
        tp.tp_column_linear(self.X, self.W1, self.Wu, self.b1, self.Y, w.T, w.d, w.k, w.p,
                            self.dtype, self.act, stream=st)
        ev[1].record(st)
        tp.tp_row_linear(self.Y, self.W2, self.P, w.T, w.k, w.d, w.p, self.dtype, stream=st)
        ev[2].record(st)
        tp.tp_reduce_partials(self.P, self.b2, self.Z, w.T, w.d, w.p, stream=st)
        ev[3].record(st)

    def capture(self, fn):
        """Warm up eagerly, then capture one step as a CUDA graph; returns
        (graph, kernels of this library per step)."""
        torch, tp = self.torch, self.tp
        for _ in range(self.a.warmup):
            self.flush.zero_()
            fn(self.stream)
        tp.tp_sync_status(self.stream)
        if self.a.no_graph:
            return None, None
        g = torch.cuda.CUDAGraph()
        n0 = tp.tp_kernel_launch_count()
        with torch.cuda.graph(g):
            fn(torch.cuda.current_stream())
        per_step = tp.tp_kernel_launch_count() - n0
        for _ in range(self.a.warmup):
            self.flush.zero_()
            g.replay()
        torch.cuda.synchronize(self.device)
        return g, per_step

    def rmax(self, vals):
        return reduce_max(vals, self.dist if self.world > 1 else None, self.device)

    def time_block(self, gpu_index: int, flush: bool = True):
        """K steps of the block, one graph replay each, L2 flushed before each
        step outside the events.  Returns (ms per step max over ranks, library
        launches in the timed region, clock summary, wall seconds)."""
        torch, tp = self.torch, self.tp
        if not hasattr(self, "g_block"):
            self.g_block, self.k_block = self.capture(self.block_step)
        e0 = torch.cuda.Event(enable_timing=True)
        e1 = torch.cuda.Event(enable_timing=True)
        step_ms = []
        with ClockSampler(gpu_index) as clocks:
            self.barrier()
            torch.cuda.synchronize(self.device)
            n0 = tp.tp_kernel_launch_count()
            t_wall = time.perf_counter()
            for _ in range(self.a.steps):
                if flush:
                    self.flush.zero_()
                e0.record(self.stream)
                if self.g_block is not None:
                    self.g_block.replay()
                else:
                    self.block_step(self.stream)
                e1.record(self.stream)
                torch.cuda.synchronize(self.device)
                step_ms.append(e0.elapsed_time(e1))
            t_wall = time.perf_counter() - t_wall
            launches = tp.tp_kernel_launch_count() - n0
            if self.g_block is not None:
                launches = self.k_block * self.a.steps
            self.barrier()
        tp.tp_sync_status(self.stream)
        ms, launches = self.rmax([statistics.mean(step_ms), float(launches)])
        return ms, int(launches), clocks.summary(), t_wall

    def time_calls(self, gpu_index: int):
        """The block as the three C-ABI calls (one graph), events between them:
        per-layer times (max over ranks) and the loop's clock summary."""
        torch, tp = self.torch, self.tp
        self.evs = [torch.cuda.Event(enable_timing=True, external=not self.a.no_graph)
                    for _ in range(4)]
        g_calls, _ = self.capture(self.calls_step)
        col, row, red, tot = [], [], [], []
        with ClockSampler(gpu_index) as clocks:
            self.barrier()
            for _ in range(self.a.steps):
                self.flush.zero_()
                if g_calls is not None:
                    g_calls.replay()
                else:
                    self.calls_step(self.stream)
                torch.cuda.synchronize(self.device)
                ev = self.evs
                col.append(ev[0].elapsed_time(ev[1]))
                row.append(ev[1].elapsed_time(ev[2]))
                red.append(ev[2].elapsed_time(ev[3]))
                tot.append(ev[0].elapsed_time(ev[3]))
            self.barrier()
        tp.tp_sync_status(self.stream)
        vals = self.rmax([statistics.mean(x) for x in (col, row, red, tot)])
        return dict(zip(["column", "row", "reduce", "sum"], vals)), clocks.summary()


def layer_figures(w: WL.Workload, kernels: dict, clk: dict, peaks: dict, peak_src: str) -> dict:
    """Per-layer throughput of the three-call loop against the peak that fits
    that loop's clocks, with the clock record and time x median SM MHz."""
    peak, src = tensor_peak(peaks, peak_src, clk)

    def tfl(f, ms):
        return f / (ms * 1e-3) / 1e12

    mhz = clk.get("sm_mhz")
    out = {}
    bf16 = w.dtype == "bf16"
    for name, fl in (("column", column_flops(w)), ("row", row_flops(w))):
        ms = kernels[name]
        out[name] = {"ms": ms, "TFLOP/s": tfl(fl, ms),
                     "frac_bf16_peak": tfl(fl, ms) / peak if bf16 else None,
                     "frac_bf16_burst": tfl(fl, ms) / peaks["bf16_tflops"] if bf16 else None,
                     "ms_x_mhz": None if mhz is None else ms * mhz}
    rb = reduce_bytes(w)
    gbs = rb / (kernels["reduce"] * 1e-3) / 1e9
    out["reduce"] = {"ms": kernels["reduce"], "GB/s": gbs, "frac_hbm": gbs / peaks["hbm_gbs"],
                     "bytes": rb, "ms_x_mhz": None if mhz is None else kernels["reduce"] * mhz}
    out["step_ms"] = kernels["sum"]
    out["peak"] = {"bf16_tflops": peak, "source": src, "hbm_gbs": peaks["hbm_gbs"]}
    out["clocks"] = clk
    out["how"] = ("the three C-ABI calls as one graph, external timing events between them, "
                  "L2 flushed before each step; clocks sampled over this loop alone")
    return out


def step_roofline(w: WL.Workload, ms: float, clk: dict, peaks: dict, peak_src: str) -> dict:
    """Whole-step roofline: tensor side unless the step's arithmetic intensity
    (FLOPs per minimum HBM byte) is below the measured ridge point."""
    intensity = w.gemm_flops() / block_bytes(w)
    ridge = peaks["bf16_tflops"] * 1e12 / (peaks["hbm_gbs"] * 1e9)
    if w.dtype == "bf16" and intensity >= ridge:
        peak, src = tensor_peak(peaks, peak_src, clk)
        ach = w.gemm_flops() / (ms * 1e-3) / 1e12
        r = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
             "frac": ach / peak, "peak_source": src}
    else:
        ach = block_bytes(w) / (ms * 1e-3) / 1e9
        r = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
             "frac": ach / peaks["hbm_gbs"], "bytes_per_step": block_bytes(w),
             "peak_source": f"{peak_src} hbm copy"}
    r["intensity_flop_per_byte"] = intensity
    r["ridge_flop_per_byte"] = ridge
    return r


def measure_e2e(a, torch, tp, B: "MlpBench", w: WL.Workload, world: int, barrier) -> dict:
    """The block through tp_mlp_block_host: X copied in from pinned host
    memory and Z copied back inside every timed step (plus the same copies
    run one after the other around tp_mlp_block, for comparison)."""
    device = B.device
    e0 = torch.cuda.Event(enable_timing=True)
    e1 = torch.cuda.Event(enable_timing=True)
    stream = B.stream
    Xh = B.X.cpu().pin_memory()
    Zh = torch.empty(B.Z.shape, dtype=B.Z.dtype).pin_memory()
    n_host = tp.tp_mlp_block_host_workspace_size(w.T, w.d, w.k, w.p, B.dtype, B.act, B.flags)
    ws_host = torch.empty(max(n_host, 256), dtype=torch.uint8, device=device)
    Xd = torch.empty_like(B.X)

    def e2e_step():
        tp.tp_mlp_block_host(Xh, B.W1, B.Wu, B.b1, B.W2, B.b2, Zh, ws_host, n_host, w.T, w.d,
                             w.k, w.p, B.dtype, B.act, B.flags, stream=stream)

    def serial_step():
        Xd.copy_(Xh, non_blocking=True)
        tp.tp_mlp_block(Xd, B.W1, B.Wu, B.b1, B.W2, B.b2, B.Z, B.ws, B.nbytes, w.T, w.d, w.k,
                        w.p, B.dtype, B.act, B.flags, stream=stream)
        Zh.copy_(B.Z, non_blocking=True)

    def time_e2e(fn):
        for _ in range(a.warmup):
            B.flush.zero_()
            fn()
        torch.cuda.synchronize(device)
        barrier()
        t = []
        for _ in range(a.steps):
            B.flush.zero_()
            e0.record(stream)
            fn()
            e1.record(stream)
            torch.cuda.synchronize(device)
            t.append(e0.elapsed_time(e1))
        barrier()
        tp.tp_sync_status(stream)
        return B.rmax([statistics.mean(t)])[0]

    e_ms = time_e2e(e2e_step)
    s_ms = time_e2e(serial_step)
    e2e = {"value": whole_job_value(w.gemm_flops(), world, e_ms) / 1e12, "unit": UNIT,
           "ms_per_step": e_ms, "h2d_bytes_per_step": Xh.numel() * Xh.element_size(),
           "d2h_bytes_per_step": Zh.numel() * Zh.element_size(),
           "call": "tp_mlp_block_host: X read from and Z written to pinned host memory, the "
                   "token rows pipelined in chunks through copy-in, the block and copy-out",
           "serial_copies": {"value": whole_job_value(w.gemm_flops(), world, s_ms) / 1e12,
                             "ms_per_step": s_ms,
                             "how": "copy X in, tp_mlp_block on all rows, copy Z out, one "
                                    "after the other"}}

    return e2e


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

    peaks, peak_src = load_peaks()
    inp = WL.make_inputs(w)
    B = MlpBench(a, torch, tp, w, inp, device, a.mode, barrier, dist, world)

    # ---- the timed region: K steps of the block, one graph replay each
    ms_step, launches, clocks, t_wall = B.time_block(local_rank)

    # ---- the same graph replayed without the L2 flush (operands L2-resident
    # when they fit): a labelled second figure, not the metric
    l2_resident = None
    if B.g_block is not None:
        w_ms, _, _, _ = B.time_block(local_rank, flush=False)
        l2_resident = {"ms_per_step": w_ms, "value": whole_job_value(w.gemm_flops(), world, w_ms) / 1e12,
                       "unit": UNIT, "how": "graph replay without the L2 flush between steps"}

    # ---- per-kernel breakdown of the same block as three separate calls
    breakdown = None
    if a.mode == "partials" and not a.no_breakdown:
        kernels, kclk = B.time_calls(local_rank)
        breakdown = layer_figures(w, kernels, kclk, peaks, peak_src)

    # ---- end to end through the public block call with host buffers: X read
    # from, and Z written to, pinned host memory inside the timed step
    e2e = None if a.no_e2e else measure_e2e(a, torch, tp, B, w, world, barrier)

    value = whole_job_value(w.gemm_flops(), world, ms_step) / 1e12
    kernel_name = {"partials": "tp_mlp_block: column GEMM -> row GEMM with the fixed-order fold "
                               "(PDL-chained; on CTA-pair row tiles the row GEMM's epilogue folds "
                               "shard by shard into Z, else a fold kernel follows)",
                   "fold": "tp_mlp_block row-fold: column GEMM -> row GEMM folding the p partials "
                           "in its epilogue (bit-identical to partials + fold)",
                   "splitk": "tp_mlp_block split-K: column GEMM -> row GEMM accumulating all shards",
                   "fused": "tc_block_kernel (both GEMM layers, one launch) -> fold"}[a.mode]
    roof = step_roofline(w, ms_step, clocks, peaks, peak_src)
    roof.update(traffic_entry(f"{w.name}/{a.mode}"))
    roof.update({"kernel": kernel_name,
                 "duration": "block step time (graph replay, CUDA events on the launching stream)",
                 "traffic_scope": "dram bytes of all kernels of one step (ncu)"})

    # The dominant kernel (largest share of the separately timed layers):
    # algorithmic FLOPs (or bytes) per launch over its CUDA-event duration,
    # against the peak that fits the clocks of the loop it was timed in.
    if breakdown is not None:
        ridge = roof["ridge_flop_per_byte"]
        cand = {
            "column": (column_flops(w), column_bytes(w), breakdown["column"]["ms"],
                       "tc_gemm_kernel/tc_gemm_pair_kernel, column layer (all shards)"),
            "row": (row_flops(w), row_bytes(w), breakdown["row"]["ms"],
                    "tc_gemm_kernel/tc_gemm_pair_kernel, row layer to partials (all shards)"),
            "reduce": (0, reduce_bytes(w), breakdown["reduce"]["ms"],
                       "reduce_vec_kernel, fixed-order fold"),
        }
        name = max(cand, key=lambda n: cand[n][2])
        fl_k, by_k, ms_k, desc = cand[name]
        if w.dtype == "bf16" and fl_k > 0 and fl_k / by_k >= ridge:
            peak, src = breakdown["peak"]["bf16_tflops"], breakdown["peak"]["source"]
            ach = fl_k / (ms_k * 1e-3) / 1e12
            kroof = {"bound": "tensor", "achieved": ach, "peak": peak, "unit": "TFLOP/s",
                     "frac": ach / peak, "frac_of_burst": ach / peaks["bf16_tflops"],
                     "flops_per_launch": fl_k, "peak_source": src}
        else:
            ach = by_k / (ms_k * 1e-3) / 1e9
            kroof = {"bound": "hbm", "achieved": ach, "peak": peaks["hbm_gbs"], "unit": "GB/s",
                     "frac": ach / peaks["hbm_gbs"], "bytes_per_launch": by_k,
                     "peak_source": f"{peak_src} hbm copy"}
        kroof.update(traffic_entry(f"{w.name}/{name}"))
        kroof.update({"kernel": f"{name}: {desc}",
                      "duration": "average launch duration, CUDA events on the launching stream "
                                  "around the layer's call inside a replayed graph",
                      "launch_ms": ms_k, "loop_clocks": breakdown["clocks"], "step": roof})
        roof = kroof

    line = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": w.dtype, "data": "synthetic",
        "config": {"workload": w.name, "T": w.T, "d": w.d, "k": w.k, "p": w.p, "act": w.act,
                   "mode": a.mode, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "launch": "eager" if B.g_block is None else "cuda-graph replay of tp_mlp_block",
                   "l2": "flushed before every step (256 MiB write, outside the timed events)"},
        "pct_bf16_peak": 100.0 * value / (peaks["bf16_tflops"] * world) if w.dtype == "bf16" else None,
        "reduce": None if breakdown is None else breakdown["reduce"],
        "unfused_breakdown": breakdown,
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clocks,
        "e2e": e2e,
        "l2_resident": l2_resident,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rows = min(w.T, oracle_sample_rows(w))
        sec, reps, z_ref = time_oracle(w, inp, rows, min_seconds=10.0, max_reps=1000, want_z=True)
        line["cpu_baseline"] = {"value": w.gemm_flops() * rows / w.T / sec / 1e12, "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": f"first {rows} of {w.T} token rows, {reps} reps, float64"}
        # the timed steps' own output on the same rows against the oracle
        # (each output row depends only on its own input row)
        from oracle import tp_oracle as O
        tol = 1e-2 if w.dtype == "bf16" else 1e-5
        err = O.rel_err(B.Z[:rows].cpu().numpy(), z_ref)
        line["cpu_baseline"]["parity"] = {
            "rows": rows, "measure": "max|gpu - oracle| / max|oracle|", "value": err,
            "tolerance": tol, "ok": bool(err <= tol),
            "of": "the device Z the timed calls wrote (each of them writes the same bits)"}
        try:   # the same oracle on one host thread
            from threadpoolctl import threadpool_limits
            with threadpool_limits(limits=1):
                rows1 = max(1, rows // 8)
                sec1, reps1 = time_oracle(w, inp, rows1, min_seconds=3.0, max_reps=100)
            line["cpu_baseline"]["single_thread"] = {
                "value": w.gemm_flops() * rows1 / w.T / sec1 / 1e12, "unit": UNIT, "cores": 1,
                "sample": f"first {rows1} of {w.T} token rows, {reps1} reps, float64"}
        except Exception as exc:  # threadpoolctl missing or BLAS not controllable
            line["cpu_baseline"]["single_thread"] = {"unavailable": str(exc)[:120]}

    # ---- the other MLP workloads, each measured the same way in this process
    # (block step + three-call breakdown), for the per-workload table
    if world == 1 and not a.no_configs and a.mode == "partials":
        del B, inp
        torch.cuda.empty_cache()
        table = {}
        for name in [n for n in CONFIG_ORDER if n != w.name]:
            wc = WL.WORKLOADS[name]
            try:
                Bc = MlpBench(a, torch, tp, wc, WL.make_inputs(wc), device, "partials", barrier,
                              dist, world)
                ms_c, _, clk_c, _ = Bc.time_block(local_rank)
                kern_c, kclk_c = Bc.time_calls(local_rank)
                lay = layer_figures(wc, kern_c, kclk_c, peaks, peak_src)
                table[name] = {
                    "T": wc.T, "d": wc.d, "k": wc.k, "p": wc.p, "act": wc.act, "dtype": wc.dtype,
                    "ms_per_step": ms_c,
                    "TFLOP/s": wc.gemm_flops() / (ms_c * 1e-3) / 1e12,
                    "step_roofline": step_roofline(wc, ms_c, clk_c, peaks, peak_src),
                    "clocks": clk_c,
                    "column": lay["column"], "row": lay["row"], "reduce": lay["reduce"],
                    "layer_loop_clocks": kclk_c, "layer_peak": lay["peak"]}
            except Exception as exc:   # the table is an extra: it never costs the headline line
                table[name] = {"error": f"{type(exc).__name__}: {str(exc)[:200]}"}
            Bc = None
            torch.cuda.empty_cache()
        line["configs"] = table
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


# The workloads of the per-workload table, smallest first.
CONFIG_ORDER = ["toy", "gpt2", "decode", "wide", "llama"]


def run_tp_attn(a, w: WL.AttnWorkload, rank: int, world: int, local_rank: int):
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

    grp = dist if world > 1 else None
    inp = WL.make_attn_inputs(w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim)

    def dev(x):
        if x is None:
            return None
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(x).to(device)

    X, Wq, Wk, Wv, Wo, bo = (dev(inp.X), dev(inp.Wq), dev(inp.Wk), dev(inp.Wv), dev(inp.Wo),
                             dev(inp.bo))
    T, d, h, hkv, dh, p, causal = w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, w.p, w.causal
    Z = torch.empty((T, d), dtype=torch.float32, device=device)
    nbytes = tp.tp_attn_block_workspace_size(T, d, h, hkv, dh, p)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)
    # separate buffers for the per-call breakdown
    Qs = torch.empty((p, T, h // p * dh), dtype=torch.bfloat16, device=device)
    Ks = torch.empty((p, T, hkv // p * dh), dtype=torch.bfloat16, device=device)
    Vs = torch.empty_like(Ks)
    Os = torch.empty_like(Qs)
    Ps = torch.empty((p, T, d), dtype=torch.float32, device=device)
    ident = tp.TP_ACT_IDENTITY
    H = Harness(a, torch, tp, device, barrier)

    def block_step(st):
        tp.tp_attn_block(X, Wq, Wk, Wv, Wo, bo, Z, ws, nbytes, T, d, h, hkv, dh, p, causal,
                         stream=st)

    evs = [torch.cuda.Event(enable_timing=True, external=not a.no_graph) for _ in range(5)]

    def calls_step(st):
        evs[0].record(st)
        tp.tp_column_linear(X, Wq, None, None, Qs, T, d, h * dh, p, tp.TP_BF16, ident, stream=st)
        tp.tp_column_linear(X, Wk, None, None, Ks, T, d, hkv * dh, p, tp.TP_BF16, ident, stream=st)
        tp.tp_column_linear(X, Wv, None, None, Vs, T, d, hkv * dh, p, tp.TP_BF16, ident, stream=st)
        evs[1].record(st)
        tp.tp_attention_heads(Qs, Ks, Vs, Os, T, p, h, hkv, dh, causal, stream=st)
        evs[2].record(st)
        tp.tp_row_linear(Os, Wo, Ps, T, h * dh, d, p, tp.TP_BF16, stream=st)
        evs[3].record(st)
        tp.tp_reduce_partials(Ps, bo, Z, T, d, p, stream=st)
        evs[4].record(st)

    with ClockSampler(local_rank) as clocks:
        step_ms, launches, t_wall = H.time_steps(block_step)
    ms_step, launches = reduce_max([statistics.mean(step_ms), float(launches)], grp, device)

    fl = w.flops()
    peaks, peak_src = load_peaks()
    breakdown = None
    if not a.no_breakdown:
        parts, _, _ = H.time_steps(calls_step, events=evs)
        qkv_ms, att_ms, out_ms, red_ms = reduce_max([statistics.mean(col) for col in zip(*parts)],
                                                    grp, device)
        red_bytes = (p + 1) * T * d * 4 + (d * 4 if bo is not None else 0)

        def tf(f, ms):
            return f / (ms * 1e-3) / 1e12
        breakdown = {
            "qkv": {"ms": qkv_ms, "TFLOP/s": tf(fl["qkv"], qkv_ms)},
            "attention": {"ms": att_ms, "TFLOP/s": tf(fl["attention"], att_ms)},
            "out": {"ms": out_ms, "TFLOP/s": tf(fl["out"], out_ms)},
            "reduce": {"ms": red_ms, "GB/s": red_bytes / (red_ms * 1e-3) / 1e9, "bytes": red_bytes},
            "how": "the six C-ABI calls as one graph, external timing events between them",
        }
        for k in ("qkv", "attention", "out"):
            breakdown[k]["frac_bf16_peak"] = breakdown[k]["TFLOP/s"] / peaks["bf16_tflops"]

    e2e = None
    if not a.no_e2e:
        Xh = X.cpu().pin_memory()
        Zh = torch.empty(Z.shape, dtype=Z.dtype).pin_memory()
        Xd = torch.empty_like(X)

        def e2e_step(st):
            Xd.copy_(Xh, non_blocking=True)
            tp.tp_attn_block(Xd, Wq, Wk, Wv, Wo, bo, Z, ws, nbytes, T, d, h, hkv, dh, p, causal,
                             stream=st)
            Zh.copy_(Z, non_blocking=True)

        t_e2e, _, _ = H.time_steps(e2e_step, graph=False)
        e_ms = reduce_max([statistics.mean(t_e2e)], grp, device)[0]
        e2e = {"value": whole_job_value(fl["total"], world, e_ms) / 1e12, "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": Xh.numel() * Xh.element_size(),
               "d2h_bytes_per_step": Zh.numel() * Zh.element_size(),
               "call": "tp_attn_block, X host->device and Z device->host inside the timed step"}

    value = whole_job_value(fl["total"], world, ms_step) / 1e12
    achieved = fl["total"] / (ms_step * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "traffic": ncu_traffic(f"{w.name}/block"),
            "kernel": "tp_attn_block: QKV column GEMMs -> tc_attn_kernel -> row GEMM with the "
                      "fixed-order fold in its epilogue (CTA-pair tiles; else -> fold)",
            "duration": "block step time (graph replay, CUDA events on the launching stream)",
            "peak_source": f"{peak_src} bf16 dense (burst)",
            "flops_per_step": fl}
    if breakdown is not None:
        # the attention kernel, the row's own hot kernel: FLOPs per launch over
        # its event-timed duration
        att_ms = breakdown["attention"]["ms"]
        ach = fl["attention"] / (att_ms * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"],
                "flops_per_launch": fl["attention"], "traffic": ncu_traffic(f"{w.name}/attention"),
                "kernel": "tc_attn_kernel (all shards and heads, one launch)",
                "duration": "average launch duration, CUDA events on the launching stream around "
                            "tp_attention_heads inside a replayed graph",
                "launch_ms": att_ms, "peak_source": f"{peak_src} bf16 dense (burst)", "step": roof}
    line = {
        "metric": ATTN_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(attn_config(w, world),
                       launch="eager" if a.no_graph else "cuda-graph replay of tp_attn_block",
                       l2="flushed before every step (256 MiB write, outside the timed events)"),
        "pct_bf16_peak": 100.0 * value / (peaks["bf16_tflops"] * world),
        "breakdown": breakdown,
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rows = attn_oracle_rows(w)
        sec, reps = time_attn_oracle(w, inp, rows, min_seconds=10.0, max_reps=1000)
        line["cpu_baseline"] = {"value": attn_flops_prefix(w, rows)["total"] / sec / 1e12,
                                "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"causal prefix: first {rows} of {w.T} tokens, {reps} reps, "
                                          "float64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def run_tp_block(a, w: WL.BlockWorkload, rank: int, world: int, local_rank: int):
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

    grp = dist if world > 1 else None
    H = Harness(a, torch, tp, device, barrier)
    inp = WL.make_block_inputs(w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, w.k, w.act)

    def dev(x):
        if x is None:
            return None
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(x).to(device)

    T, d, h, hkv, dh, k, p = w.T, w.d, w.n_heads, w.n_kv_heads, w.head_dim, w.k, w.p
    act, causal = tp.ACT[w.act], w.causal
    X = dev(inp.X)
    t = {name: dev(v) for name, v in inp.prm.items()}
    prm = tp.block_params(**t)
    out = torch.empty((T, d), dtype=torch.float32, device=device)
    nbytes = tp.tp_transformer_block_workspace_size(T, d, h, hkv, dh, k, p)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def block_step(st):
        tp.tp_transformer_block(X, prm, out, ws, nbytes, T, d, h, hkv, dh, k, p, act, causal,
                                stream=st)

    with ClockSampler(local_rank) as clocks:
        step_ms, launches, t_wall = H.time_steps(block_step)
    ms_step, launches = reduce_max([statistics.mean(step_ms), float(launches)], grp, device)
    fl = w.flops()
    peaks, peak_src = load_peaks()

    breakdown = None
    if not a.no_breakdown:
        A = torch.empty((T, d), dtype=torch.bfloat16, device=device)
        Hs = torch.empty((T, d), dtype=torch.float32, device=device)
        Qs = torch.empty((p, T, h // p * dh), dtype=torch.bfloat16, device=device)
        Ks = torch.empty((p, T, hkv // p * dh), dtype=torch.bfloat16, device=device)
        Vs = torch.empty_like(Ks)
        Os = torch.empty_like(Qs)
        Ys = torch.empty((p, T, k // p), dtype=torch.bfloat16, device=device)
        Ps = torch.empty((p, T, d), dtype=torch.float32, device=device)
        Zs = torch.empty((T, d), dtype=torch.float32, device=device)
        names = ["ln1", "qkv", "attention", "out_proj", "fold1", "ln2", "mlp_column", "mlp_row",
                 "fold2"]
        evs = [torch.cuda.Event(enable_timing=True, external=not a.no_graph)
               for _ in range(len(names) + 1)]
        ident, bf = tp.TP_ACT_IDENTITY, tp.TP_BF16

        def calls_step(st):
            evs[0].record(st)
            tp.tp_layer_norm(X, t["ln1_gamma"], t["ln1_beta"], A, T, d, stream=st)
            evs[1].record(st)
            tp.tp_column_linear(A, t["Wq"], None, None, Qs, T, d, h * dh, p, bf, ident, stream=st)
            tp.tp_column_linear(A, t["Wk"], None, None, Ks, T, d, hkv * dh, p, bf, ident, stream=st)
            tp.tp_column_linear(A, t["Wv"], None, None, Vs, T, d, hkv * dh, p, bf, ident, stream=st)
            evs[2].record(st)
            tp.tp_attention_heads(Qs, Ks, Vs, Os, T, p, h, hkv, dh, causal, stream=st)
            evs[3].record(st)
            tp.tp_row_linear(Os, t["Wo"], Ps, T, h * dh, d, p, bf, stream=st)
            evs[4].record(st)
            tp.tp_reduce_partials_residual(Ps, t["bo"], X, Hs, T, d, p, stream=st)
            evs[5].record(st)
            tp.tp_layer_norm(Hs, t["ln2_gamma"], t["ln2_beta"], A, T, d, stream=st)
            evs[6].record(st)
            tp.tp_column_linear(A, t["W1"], t["W_up"], t["b1"], Ys, T, d, k, p, bf, act, stream=st)
            evs[7].record(st)
            tp.tp_row_linear(Ys, t["W2"], Ps, T, k, d, p, bf, stream=st)
            evs[8].record(st)
            tp.tp_reduce_partials_residual(Ps, t["b2"], Hs, Zs, T, d, p, stream=st)
            evs[9].record(st)

        parts, _, _ = H.time_steps(calls_step, events=evs)
        means = reduce_max([statistics.mean(col) for col in zip(*parts)], grp, device)
        af = w.attn().flops()
        mlp_col = 2 * T * d * k * (2 if w.act == "swiglu" else 1)
        flops_of = {"qkv": af["qkv"], "attention": af["attention"], "out_proj": af["out"],
                    "mlp_column": mlp_col, "mlp_row": 2 * T * k * d}
        bytes_of = {"ln1": T * d * 6, "ln2": T * d * 6, "fold1": (p + 2) * T * d * 4,
                    "fold2": (p + 2) * T * d * 4}
        breakdown = {"how": "the public calls one after another as one graph, external timing "
                            "events between them (unfused: the block fuses fold1 with ln2)"}
        for name, ms in zip(names, means):
            ent = {"ms": ms}
            if name in flops_of:
                ent["TFLOP/s"] = flops_of[name] / (ms * 1e-3) / 1e12
                ent["frac_bf16_peak"] = ent["TFLOP/s"] / peaks["bf16_tflops"]
            else:
                ent["GB/s"] = bytes_of[name] / (ms * 1e-3) / 1e9
                ent["frac_hbm"] = ent["GB/s"] / peaks["hbm_gbs"]
            breakdown[name] = ent
        breakdown["sum_ms"] = sum(means)

    e2e = None
    if not a.no_e2e:
        Xh = X.cpu().pin_memory()
        Oh = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        Xd = torch.empty_like(X)

        def e2e_step(st):
            Xd.copy_(Xh, non_blocking=True)
            tp.tp_transformer_block(Xd, prm, out, ws, nbytes, T, d, h, hkv, dh, k, p, act, causal,
                                    stream=st)
            Oh.copy_(out, non_blocking=True)

        t_e2e, _, _ = H.time_steps(e2e_step, graph=False)
        e_ms = reduce_max([statistics.mean(t_e2e)], grp, device)[0]
        e2e = {"value": whole_job_value(fl["total"], world, e_ms) / 1e12, "unit": UNIT,
               "ms_per_step": e_ms, "h2d_bytes_per_step": Xh.numel() * Xh.element_size(),
               "d2h_bytes_per_step": Oh.numel() * Oh.element_size(),
               "call": "tp_transformer_block, X host->device and out device->host inside the "
                       "timed step"}

    value = whole_job_value(fl["total"], world, ms_step) / 1e12
    achieved = fl["total"] / (ms_step * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "traffic": ncu_traffic(f"{w.name}/block"),
            "kernel": "tp_transformer_block: LN -> QKV GEMMs -> tc_attn_kernel -> Wo GEMM -> "
                      "fold+residual+LN -> MLP GEMMs, the row GEMM folding + b2 + residual in "
                      "its epilogue (CTA-pair tiles; else -> fold+residual)",
            "duration": "block step time (graph replay, CUDA events on the launching stream)",
            "peak_source": f"{peak_src} bf16 dense (burst)", "flops_per_step": fl}
    if breakdown is not None:
        # the dominant single kernel launch (the Q, K, V GEMMs are three launches)
        per_launch = {n: breakdown[n]["ms"] / (3 if n == "qkv" else 1)
                      for n in ("qkv", "attention", "out_proj", "mlp_column", "mlp_row")}
        name = max(per_launch, key=per_launch.get)
        fl_k = flops_of[name] / (3 if name == "qkv" else 1)
        ach = fl_k / (per_launch[name] * 1e-3) / 1e12
        roof = {"bound": "tensor", "achieved": ach, "peak": peaks["bf16_tflops"],
                "unit": "TFLOP/s", "frac": ach / peaks["bf16_tflops"], "flops_per_launch": fl_k,
                "traffic": ncu_traffic(f"{w.name}/{name}"), "kernel": name,
                "duration": "average launch duration, CUDA events on the launching stream around "
                            "the call inside a replayed graph",
                "launch_ms": per_launch[name], "peak_source": f"{peak_src} bf16 dense (burst)",
                "step": roof}
    line = {
        "metric": BLOCK_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": dict(block_config(w, world),
                       launch="eager" if a.no_graph else "cuda-graph replay of tp_transformer_block",
                       l2="flushed before every step (256 MiB write, outside the timed events)"),
        "pct_bf16_peak": 100.0 * value / (peaks["bf16_tflops"] * world),
        "breakdown": breakdown,
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        rows = block_oracle_rows(w)
        sec, reps = time_block_oracle(w, inp, rows, min_seconds=10.0, max_reps=1000)
        line["cpu_baseline"] = {"value": block_flops_prefix(w, rows)["total"] / sec / 1e12,
                                "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                                "sample": f"causal prefix: first {rows} of {w.T} tokens, {reps} "
                                          "reps, float64"}
    if rank == 0:
        print(json.dumps(line), flush=True)
    if world > 1:
        dist.destroy_process_group()
    return 0


def backward_flops(w: WL.Workload, T=None) -> int:
    """GEMM FLOPs of the backward pass: dY = dZ W2^T, dW2 = Y^T dZ, dW1 = X^T dH,
    dX = dH W1^T (SwiGLU: dW_up and dU W_up^T as well), 2*T*d*k each."""
    T = w.T if T is None else T
    return 2 * T * w.d * w.k * (6 if w.act == "swiglu" else 4)


def backward_inputs(w: WL.Workload, seed: int = 42):
    """The forward inputs of the workload plus an upstream gradient dZ
    (bf16, standard normal), drawn after them."""
    inp = WL.make_inputs(w, seed)
    rng = np.random.default_rng(seed + 1)
    dZ = WL.f32_to_bf16_bits(rng.standard_normal((w.T, w.d), dtype=np.float32))
    return inp, dZ


def run_reference_backward(a, w: WL.Workload, rank: int, world: int):
    if rank != 0:
        return 0
    from oracle import tp_oracle as O
    inp, dZ = backward_inputs(w)
    rows = int(max(1, min(w.T, 3e10 // (backward_flops(w) / w.T))))
    X = inp.values("X")[:rows]
    dz = WL.bf16_bits_to_f32(dZ)[:rows]
    args = (inp.values("W1"), inp.values("b1"), inp.values("W2"), dz, w.p, w.act)

    def once():
        t0 = time.perf_counter()
        O.mlp_backward_sharded(X, *args, W_up=inp.values("W_up"))
        return time.perf_counter() - t0

    for _ in range(a.warmup):
        once()
    ms = 1e3 * statistics.mean(once() for _ in range(a.steps))
    value = backward_flops(w, rows) / (ms * 1e-3) / 1e12
    line = {
        "impl": "reference", "metric": BWD_METRIC, "value": value, "unit": UNIT, "n_gpus": world,
        "steps": a.steps, "warmup": a.warmup, "ms_per_step": ms, "higher_is_better": True,
        "scaling": "weak", "vs_baseline": None, "dtype": "f64", "data": "synthetic",
        "config": {"workload": w.name, "mode": "backward", "T": w.T, "d": w.d, "k": w.k, "p": w.p,
                   "act": w.act, "sample_rows": rows,
                   "parallelism": f"replicas{world}" if world > 1 else "single"},
        "cpu_baseline": {"value": value, "unit": UNIT, "cores": blas_threads(), "kind": "oracle",
                         "sample": f"first {rows} of {w.T} token rows per step, full weights"},
        "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }
    print(json.dumps(line), flush=True)
    return 0


def run_tp_backward(a, w: WL.Workload, rank: int, world: int, local_rank: int):
    import torch
    import torch.distributed as dist
    import megatron_tensor_sharded_b200 as tp

    if w.dtype != "bf16":
        raise SystemExit("the backward pass is provided for the bf16 workloads")
    torch.cuda.set_device(local_rank)
    device = torch.device("cuda", local_rank)
    if world > 1:
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    def barrier():
        if world > 1:
            dist.barrier()

    grp = dist if world > 1 else None
    H = Harness(a, torch, tp, device, barrier)
    inp, dZh = backward_inputs(w)

    def dev(x):
        if x is None:
            return None
        if x.dtype == np.uint16:
            return torch.from_numpy(x.view(np.int16)).view(torch.bfloat16).to(device)
        return torch.from_numpy(x).to(device)

    T, d, k, p = w.T, w.d, w.k, w.p
    act, bf = tp.ACT[w.act], tp.TP_BF16
    X, W1, Wu, b1, W2 = dev(inp.X), dev(inp.W1), dev(inp.W_up), dev(inp.b1), dev(inp.W2)
    dZ = dev(dZh)
    sh = (p, T, k // p)
    Hp = torch.empty(sh, dtype=torch.bfloat16, device=device)
    Hu = torch.empty(sh, dtype=torch.bfloat16, device=device) if w.act == "swiglu" else None
    Y = torch.empty(sh, dtype=torch.bfloat16, device=device)
    ident = tp.TP_ACT_IDENTITY
    tp.tp_column_linear(X, W1, None, b1, Hp, T, d, k, p, bf, ident)
    if Hu is not None:
        tp.tp_column_linear(X, Wu, None, None, Hu, T, d, k, p, bf, ident)
    tp.tp_column_linear(X, W1, Wu, b1, Y, T, d, k, p, bf, act)
    f32 = dict(dtype=torch.float32, device=device)
    dX, dW1, db1 = torch.empty((T, d), **f32), torch.empty((d, k), **f32), torch.empty(k, **f32)
    dWu = torch.empty((d, k), **f32) if Hu is not None else None
    dW2, db2 = torch.empty((k, d), **f32), torch.empty(d, **f32)
    nbytes = tp.tp_mlp_block_backward_workspace_size(T, d, k, p, act)
    ws = torch.empty(nbytes, dtype=torch.uint8, device=device)

    def step(st, dz=dZ):
        tp.tp_mlp_block_backward(X, W1, Wu, W2, Hp, Hu, Y, dz, dX, dW1, dWu, db1, dW2, db2, ws,
                                 nbytes, T, d, k, p, act, stream=st)

    with ClockSampler(local_rank) as clocks:
        step_ms, launches, t_wall = H.time_steps(step)
    ms_step, launches = reduce_max([statistics.mean(step_ms), float(launches)], grp, device)
    fl = backward_flops(w)
    peaks, peak_src = load_peaks()

    e2e = None
    if not a.no_e2e:
        dZpin = dZ.cpu().pin_memory()
        dXh = torch.empty((T, d), dtype=torch.float32).pin_memory()
        dZd = torch.empty_like(dZ)

        def e2e_step(st):
            dZd.copy_(dZpin, non_blocking=True)
            step(st, dZd)
            dXh.copy_(dX, non_blocking=True)

        t_e2e, _, _ = H.time_steps(e2e_step, graph=False)
        e_ms = reduce_max([statistics.mean(t_e2e)], grp, device)[0]
        e2e = {"value": whole_job_value(fl, world, e_ms) / 1e12, "unit": UNIT, "ms_per_step": e_ms,
               "h2d_bytes_per_step": dZpin.numel() * dZpin.element_size(),
               "d2h_bytes_per_step": dXh.numel() * dXh.element_size(),
               "call": "tp_mlp_block_backward, dZ host->device and dX device->host inside the "
                       "timed step (weight gradients stay on the device)"}

    value = whole_job_value(fl, world, ms_step) / 1e12
    achieved = fl / (ms_step * 1e-3) / 1e12
    roof = {"bound": "tensor", "achieved": achieved, "peak": peaks["bf16_tflops"],
            "unit": "TFLOP/s", "frac": achieved / peaks["bf16_tflops"],
            "traffic": ncu_traffic(f"{w.name}/backward"),
            "kernel": "tp_mlp_block_backward: dH GEMM (act' epilogue) -> dW2, dW1 GEMMs -> "
                      "bias-gradient column sums -> dX partial GEMM -> fold",
            "duration": "backward step time (graph replay, CUDA events on the launching stream)",
            "peak_source": f"{peak_src} bf16 dense (burst)"}
    line = {
        "metric": BWD_METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": a.steps,
        "warmup": a.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": w.name, "mode": "backward", "T": T, "d": d, "k": k, "p": p,
                   "act": w.act, "parallelism": f"replicas{world}" if world > 1 else "single",
                   "launch": "eager" if a.no_graph else "cuda-graph replay of tp_mlp_block_backward",
                   "l2": "flushed before every step (256 MiB write, outside the timed events)"},
        "pct_bf16_peak": 100.0 * value / (peaks["bf16_tflops"] * world),
        "roofline": roof,
        "gpu_launches": int(launches),
        "clocks": clocks.summary(),
        "e2e": e2e,
        "wall_s_timed_region": t_wall,
    }
    if rank == 0 and world == 1 and not a.no_cpu_baseline:
        from oracle import tp_oracle as O
        rows = int(max(1, min(T, 3e10 // (fl / T))))
        Xs = inp.values("X")[:rows]
        dzs = WL.bf16_bits_to_f32(dZh)[:rows]
        reps, t0 = 0, time.perf_counter()
        while time.perf_counter() - t0 < 10.0 and reps < 1000:
            O.mlp_backward_sharded(Xs, inp.values("W1"), inp.values("b1"), inp.values("W2"), dzs,
                                   p, w.act, W_up=inp.values("W_up"))
            reps += 1
        sec = (time.perf_counter() - t0) / reps
        line["cpu_baseline"] = {"value": backward_flops(w, rows) / sec / 1e12, "unit": UNIT,
                                "cores": blas_threads(), "kind": "oracle",
                                "sample": f"first {rows} of {T} token rows, {reps} reps, float64"}
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
    ap.add_argument("--workload", choices=sorted(WL.WORKLOADS) + sorted(WL.ATTN_WORKLOADS)
                    + sorted(WL.BLOCK_WORKLOADS), default="llama")
    ap.add_argument("--mode", choices=["partials", "fold", "splitk", "fused", "backward"],
                    default="partials")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-graph", action="store_true", help="launch eagerly instead of graph replay")
    ap.add_argument("--no-breakdown", action="store_true", help="skip the per-kernel loop")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-configs", action="store_true",
                    help="skip the per-workload table of the other MLP workloads")
    ap.add_argument("--tokens", type=int, default=None,
                    help="MLP workloads: another token count T (same widths and shards)")
    a = ap.parse_args(argv)
    if a.warmup < 3:
        ap.error("--warmup must be >= 3")
    rank = int(os.environ.get("RANK", "0"))
    world = int(os.environ.get("WORLD_SIZE", "1"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if world != a.gpus:
        ap.error(f"--gpus {a.gpus} but WORLD_SIZE={world}")
    if a.workload in WL.BLOCK_WORKLOADS:
        w = WL.BLOCK_WORKLOADS[a.workload]
        if a.impl == "reference":
            return run_reference_block(a, w, rank, world)
        return run_tp_block(a, w, rank, world, local_rank)
    if a.workload in WL.ATTN_WORKLOADS:
        w = WL.ATTN_WORKLOADS[a.workload]
        if a.impl == "reference":
            return run_reference_attn(a, w, rank, world)
        return run_tp_attn(a, w, rank, world, local_rank)
    w = WL.WORKLOADS[a.workload]
    if a.tokens is not None:
        if a.tokens < 1:
            ap.error("--tokens must be >= 1")
        w = dataclasses.replace(w, T=a.tokens, name=f"{w.name}_T{a.tokens}")
    if a.mode == "backward":
        if a.impl == "reference":
            return run_reference_backward(a, w, rank, world)
        return run_tp_backward(a, w, rank, world, local_rank)
    if a.impl == "reference":
        return run_reference(a, w, rank, world)
    return run_tp(a, w, rank, world, local_rank)


if __name__ == "__main__":
    sys.exit(main())
