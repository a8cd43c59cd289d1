"""Benchmark of the fused MLA decode epilogue on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-sweep] [--no-cpu-baseline] [--split-policy]

One step is one call of the epilogue (the whole hot path) on one batch of
the workload.  Default workload: the large batch, T=8192 tokens, H=16 heads,
RoPE and e4m3 query and cache rows, the one configuration with T >= 4096
(where the bandwidth target applies) and the largest that fits one GPU.
Inputs are device-resident when a timed region starts; consecutive calls
rotate over input sets whose total is more than twice the L2, and L2 is
written over before every timed region, so every call reads HBM.  The K
calls are replayed from CUDA graphs on one stream, timed with CUDA events on
that stream; the K-call region is timed REPLAYS times and the median is
reported.  The bare-launch floor is an empty kernel with the same grid,
block and launch attributes, timed the same way.

Printed: one JSON line (rank 0) with the metric in microseconds per call,
achieved HBM GB/s against the measured copy bandwidth, the launch floor, the
decode sizes T = 1 .. 64 standalone and behind the synthetic producer with
programmatic dependent launch (against an empty dependent kernel), the
launch-to-end latency of isolated calls, a sweep over the other workload
sizes, the end-to-end time through the Python API with pinned host buffers,
the CPU oracle as a baseline and the SM clocks seen under load.
``--impl reference`` times the CPU oracle instead (the only reference
implementation this operation has here).
"""

from __future__ import annotations

import argparse
import csv
import datetime as _dt
import json
import os
import statistics
import subprocess
import sys
import tempfile
import time

import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
if ROOT not in sys.path:
    sys.path.insert(0, ROOT)

from mla_decode_attention_10_b200 import workloads as W  # noqa: E402

METRIC = "µs/call and achieved HBM GB/s (fraction of ~8 TB/s) vs T for MLA epilogue"
UNIT = "µs/call"
HEADLINE = "batch_t8192_h16_pdl_fp8"
FALLBACK_HBM_GBS = 6650.0
NOMINAL_HBM_GBS = 8000.0
REPLAYS = 11          # timed regions per headline measurement (median reported)
CONTEXT_REPLAYS = 5   # timed regions per context measurement
DECODE_T = (1, 2, 4, 8, 16, 32, 64)
IMPLEMENTATION = "CUDA sm_100a kernels through the C ABI (libmla_epilogue.so)"

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the epilogue kernel, from ncu captures of `bench.py --steps 3 --warmup 3
# --no-sweep --no-cpu-baseline --workload <name>` (summaries in profiles/).
# Keyed by a hash of the kernel sources they were taken on: a changed kernel
# reports null until it is captured again.
KERNEL_SOURCES = ("mla_decode_attention_10_b200/csrc/mla_epilogue.cu",
                  "mla_decode_attention_10_b200/csrc/mla_rows.cu",
                  "mla_decode_attention_10_b200/csrc/epilogue_device.cuh",
                  "mla_decode_attention_10_b200/csrc/latent_math.cuh", "include/mla_epilogue.h")
TRAFFIC_SOURCE_HASH = "c179ba93f29fcdba"
TRAFFIC_BYTES = {
    "batch_t8192_h16_pdl_fp8": 163964672 + 49944320,
    "split_boundary_t64_h16_rope": 1279232 + 0,
    "prefill_t1024_h128_strided": 152633344 + 101662464,
}
L2_BYTES = 126 * 2 ** 20
# The weight-streaming producer (decode sizes): the weights a projection
# producing q for 16 heads reads, and the pool its calls rotate over.
GEMM_WEIGHT_BYTES = 9 * 2 ** 20
GEMM_WEIGHT_POOL_BYTES = 32 * GEMM_WEIGHT_BYTES
GRAPH_CALLS = 500
# ---------------------------------------------------------------------------------------
# ranks
# ---------------------------------------------------------------------------------------

def rank_info():
    return (int(os.environ.get("RANK", "0")), int(os.environ.get("WORLD_SIZE", "1")),
            int(os.environ.get("LOCAL_RANK", "0")))


def max_over_ranks(value: float, device) -> float:
    """Max of a per-rank float over the process group (identity without one)."""
    import torch.distributed as dist
    if not (dist.is_available() and dist.is_initialized()) or dist.get_world_size() == 1:
        return value
    t = torch.tensor([value], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def barrier(device):
    import torch.distributed as dist
    if dist.is_available() and dist.is_initialized():
        if dist.get_backend() == "nccl":
            dist.barrier(device_ids=[device.index])
        else:
            dist.barrier()


def job_us_per_call(max_ms: float, steps: int, world: int) -> float:
    """Whole-job microseconds per call: every rank makes `steps` calls in at
    most `max_ms`, so the job completes world*steps calls in that time."""
    return max_ms * 1e3 / (steps * world)


# ---------------------------------------------------------------------------------------
# clocks
# ---------------------------------------------------------------------------------------

class ClockSampler:
    """nvidia-smi sampled every 100 ms in the background (read-only queries)."""

    FIELDS = ("timestamp,index,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        try:
            self.gpu = f"GPU-{torch.cuda.get_device_properties(gpu_index).uuid}"
        except Exception:
            self.gpu = str(gpu_index)
        self.proc = None
        self.path = None

    def __enter__(self):
        fd, self.path = tempfile.mkstemp(suffix=".csv")
        os.close(fd)
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", f"--id={self.gpu}", f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=open(self.path, "w"), stderr=subprocess.DEVNULL)
        except (OSError, FileNotFoundError):
            self.proc = None
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()

    def samples(self):
        out = []
        if not self.path or not os.path.exists(self.path):
            return out
        for row in csv.reader(open(self.path)):
            if len(row) < 10:
                continue
            try:
                ts = _dt.datetime.strptime(row[0].strip(), "%Y/%m/%d %H:%M:%S.%f").timestamp()
                out.append(dict(t=ts, sm=float(row[2]), sm_max=float(row[3]), power=float(row[4]),
                                hw=row[6].strip(), hw_thermal=row[7].strip(), sw_thermal=row[8].strip(),
                                sw_power=row[9].strip()))
            except ValueError:
                continue
        return out

    def summary(self, t0: float, t1: float):
        s = self.samples()
        inside = [x for x in s if t0 <= x["t"] <= t1]
        window = "timed region"
        if not inside:
            inside = [x for x in s if x["power"] > 0 and t0 - 3.0 <= x["t"] <= t1 + 1.0]
            window = "load of the same graphs within 3 s before the timed region (region too short to sample)"
        if not inside:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": [], "samples": 0, "window": "no samples"}
        reasons = set()
        for x in inside:
            for k, name in (("hw", "hw_slowdown"), ("hw_thermal", "hw_thermal_slowdown"),
                            ("sw_thermal", "sw_thermal_slowdown"), ("sw_power", "sw_power_cap")):
                if x[k].lower().startswith("active"):
                    reasons.add(name)
        return {"sm_mhz": statistics.median(x["sm"] for x in inside),
                "sm_max_mhz": max(x["sm_max"] for x in inside),
                "reasons": sorted(reasons), "samples": len(inside), "window": window}


# ---------------------------------------------------------------------------------------
# device timing
# ---------------------------------------------------------------------------------------

def capture(step_fn, first: int, n: int, stream) -> torch.cuda.CUDAGraph:
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(stream):
        with torch.cuda.graph(g, stream=stream):
            for i in range(n):
                step_fn(first + i)
    return g


def graph_plan(steps: int):
    """Graphs of at most GRAPH_CALLS calls covering `steps` calls."""
    full, rest = divmod(steps, GRAPH_CALLS)
    return [GRAPH_CALLS] * full + ([rest] if rest else [])


class GraphRunner:
    def __init__(self, step_fn, steps: int, stream):
        self.stream = stream
        self.graphs = []
        first = 0
        for n in graph_plan(steps):
            self.graphs.append(capture(step_fn, first, n, stream))
            first += n

    def replay(self):
        for g in self.graphs:
            g.replay()


def timed(runner: GraphRunner, device, flush: bool = True) -> float:
    """ms for one replay of all graphs, bracketed by barrier + synchronize, max over ranks."""
    s = runner.stream
    if flush:
        flush_l2()
    barrier(device)
    torch.cuda.synchronize()
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    with torch.cuda.stream(s):
        e0.record(s)
        runner.replay()
        e1.record(s)
    torch.cuda.synchronize()
    barrier(device)
    return max_over_ranks(e0.elapsed_time(e1), device)


def kernel_source_hash() -> str:
    import hashlib
    h = hashlib.sha256()
    for f in KERNEL_SOURCES:
        with open(os.path.join(ROOT, f), "rb") as fh:
            h.update(fh.read())
    return h.hexdigest()[:16]


def traffic_for(name: str):
    """Captured DRAM bytes per launch for `name`, or None (not captured, or the kernel changed since)."""
    if name not in TRAFFIC_BYTES or kernel_source_hash() != TRAFFIC_SOURCE_HASH:
        return None
    return TRAFFIC_BYTES[name]


def measured_hbm_gbs():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    try:
        v = float(json.load(open(p))["hbm_gbs"])
        return v, "measured (MEASURED_PEAKS.json hbm_gbs: torch copy, read+write bytes)"
    except (OSError, KeyError, ValueError):
        return FALLBACK_HBM_GBS, "fallback 6.65 TB/s (no MEASURED_PEAKS.json)"


# ---------------------------------------------------------------------------------------
# workloads on the device
# ---------------------------------------------------------------------------------------

def named_variant(name: str, seed_offset: int) -> W.Workload:
    """The named workload's recipe with its seed shifted (fresh values, same shapes)."""
    return W.named(name, seed_offset)


class DeviceSets:
    """Input sets of one workload on the device, each a complete set of call
    arguments, so that consecutive calls read different memory.

    Sizes whose one call already touches more than 2x L2 get two full copies
    of the named workload.  Smaller ones get S sets cut from device pools
    drawn with a seeded CUDA generator (same shapes and distributions as the
    named recipe, contiguous layouts), S chosen so that S calls touch more
    than 2x L2; the RoPE table and the cache are shared by all sets (each
    call writes its own T slots)."""

    def __init__(self, name: str):
        self.name = name
        self.w0 = w0 = named_variant(name, 0)
        self.bytes_per_call = w0.algorithmic_bytes()
        self.sets = []
        if self.bytes_per_call > 2 * L2_BYTES or w0.producer or not w0.q_nope.is_contiguous():
            table = w0.cos_sin.to("cuda") if w0.cos_sin is not None else None
            for k in range(2):
                w = w0 if k == 0 else named_variant(name, k)
                w.cos_sin = None
                d = w.to("cuda")
                d.cos_sin = table
                q_out = torch.empty((w.T, w.H, W.ROW), dtype=w.q_out_dtype(), device="cuda")
                src = (d.q_nope.contiguous().clone(), d.q_pe.contiguous().clone()) if w.producer else None
                self.sets.append((d, q_out, src))
            self.touched = 2 * self.bytes_per_call
            return
        S = max(2, -(-2 * L2_BYTES // self.bytes_per_call))
        self._pool(w0, S)

    def _pool(self, w0, S):
        T, H = w0.T, w0.H
        g = torch.Generator(device="cuda").manual_seed(1234 + T)
        std = float(w0.q_nope.float().std()) if w0.q_nope.numel() > 1 else 1.0
        std = 2.0 if std > 1.5 else 1.0

        def randn(*shape):
            return (torch.randn(*shape, generator=g, device="cuda") * std).to(torch.bfloat16)

        qn, qp, kv, kp = randn(S, T, H, W.NOPE), randn(S, T, H, W.PE), randn(S, T, W.NOPE), randn(S, T, W.PE)
        cap = w0.num_blocks * w0.block_size
        if S * T <= cap:
            slots = torch.randperm(cap, generator=g, device="cuda")[:S * T].view(S, T)
        else:
            slots = torch.argsort(torch.rand(S, cap, generator=g, device="cuda"), dim=1)[:, :T]
        slots = slots.to(torch.int64).contiguous()
        pos = None
        table = None
        if w0.flags & W.FLAG_ROPE:
            rows = w0.cos_sin.shape[0]
            pos = torch.randint(0, rows, (S, T), generator=g, device="cuda", dtype=torch.int32)
            table = w0.cos_sin.to("cuda")
        cache = w0.cache.to("cuda")
        qs = w0.q_scale.to("cuda") if w0.q_scale is not None else None
        ks = w0.kv_scale.to("cuda") if w0.kv_scale is not None else None
        q_out = torch.empty((S, T, H, W.ROW), dtype=w0.q_out_dtype(), device="cuda")
        self._keep = (qn, qp, kv, kp, slots, pos, q_out)
        for k in range(S):
            d = W.Workload(name=w0.name, T=T, H=H, block_size=w0.block_size, num_blocks=w0.num_blocks,
                           flags=w0.flags, q_nope=qn[k], q_pe=qp[k], kv_c=kv[k], k_pe=kp[k],
                           slot_mapping=slots[k], cache=cache, positions=None if pos is None else pos[k],
                           cos_sin=table, q_scale=qs, kv_scale=ks)
            self.sets.append((d, q_out[k], None))
        self.touched = S * self.bytes_per_call


def flush_l2():
    """Write a buffer of twice the L2 size (outside any timed region)."""
    buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device="cuda")
    buf.fill_(1)
    torch.cuda.synchronize()
    del buf


# ---------------------------------------------------------------------------------------
# our implementation
# ---------------------------------------------------------------------------------------

def interleaved_medians(runners: dict, device, calls: int, reps: int) -> dict:
    """Median µs per call of each runner over `reps` timed regions, the runners
    taking turns within every repetition, so that a drift of the clocks
    between repetitions lands on all of them alike."""
    times = {k: [] for k in runners}
    for _ in range(reps):
        for k, r in runners.items():
            times[k].append(job_us_per_call(timed(r, device), calls, 1))
    return {k: statistics.median(v) for k, v in times.items()}


def median_us(runner, device, calls: int, reps: int, world: int = 1, flush: bool = True) -> float:
    """Median over `reps` timed regions of one replay each, as whole-job
    microseconds per call (each region's time is the max over ranks)."""
    return statistics.median(job_us_per_call(timed(runner, device, flush), calls, world) for _ in range(reps))


class Harness:
    """Step functions on one stream: the epilogue on a workload's device sets,
    the synthetic producer, the empty kernel with the epilogue's grid."""

    def __init__(self, E, stream):
        self.E = E
        self.stream = stream

    def epilogue(self, ds, extra=0):
        E, stream = self.E, self.stream

        def f(i):
            d, q_out, _ = ds.sets[i % len(ds.sets)]
            rc = E.launch_workload(d, q_out, extra_flags=extra, stream=stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_epilogue_launch")
        return f

    def empty(self, w0, flags):
        E, stream = self.E, self.stream
        plan = E.mla_epilogue_plan(w0.T, w0.H, w0.flags)

        def f(i):
            rc = E.mla_harness_empty(plan.blocks, plan.threads_per_block, flags, stream.cuda_stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_harness_empty")
        return f, plan

    def producer(self, ds):
        """The producer writes set i's q_nope / q_pe (from its staged copy, or
        from the next set's values when the sets carry none: the values do not
        matter for timing)."""
        E, stream, S = self.E, self.stream, len(ds.sets)

        def f(i):
            d, _, src = ds.sets[i % S]
            if src is None:
                nxt = ds.sets[(i + 1) % S][0]
                src = (nxt.q_nope, nxt.q_pe)
            rc = E.mla_harness_produce(src[0].data_ptr(), src[1].data_ptr(), d.q_nope.data_ptr(), d.q_nope.stride(0),
                                       d.q_nope.stride(1), d.q_pe.data_ptr(), d.q_pe.stride(0), d.q_pe.stride(1),
                                       d.T, d.H, 0, stream.cuda_stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_harness_produce")
        return f

    def producer_after_weights(self, ds, pool, sink):
        """The producer that first streams GEMM_WEIGHT_BYTES of weights: call i
        reads window i of `pool` (more than 2x L2 in all), so its weights come
        from DRAM as a projection's would between layers."""
        E, stream, S = self.E, self.stream, len(ds.sets)
        windows = pool.numel() * pool.element_size() // GEMM_WEIGHT_BYTES

        def f(i):
            d, _, src = ds.sets[i % S]
            if src is None:
                nxt = ds.sets[(i + 1) % S][0]
                src = (nxt.q_nope, nxt.q_pe)
            wptr = pool.data_ptr() + (i % windows) * GEMM_WEIGHT_BYTES
            rc = E.mla_harness_produce_after_weights(
                src[0].data_ptr(), src[1].data_ptr(), d.q_nope.data_ptr(), d.q_nope.stride(0), d.q_nope.stride(1),
                d.q_pe.data_ptr(), d.q_pe.stride(0), d.q_pe.stride(1), wptr, GEMM_WEIGHT_BYTES, sink.data_ptr(),
                d.T, d.H, 0, stream.cuda_stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_harness_produce_after_weights")
        return f

    def runner(self, step, calls, warmup=3):
        warm = GraphRunner(step, max(warmup, 1), self.stream)
        warm.replay()
        torch.cuda.synchronize()
        del warm
        r = GraphRunner(step, calls, self.stream)
        r.replay()  # the first replay uploads the graphs
        torch.cuda.synchronize()
        return r


def then(*fns):
    def f(i):
        for g in fns:
            g(i)
    return f


def behind_producer(hx, ds, device, calls, reps, prod=None, prefix=""):
    """Per call: the synthetic producer writes the query inputs, then X is
    launched as its programmatic dependent (PDL).  X is the epilogue, the
    empty kernel (same grid) and the empty kernel that executes
    griddepcontrol.wait; each increment is X's cost over the producer alone.
    The floor of a dependent launch is the empty kernel that waits: one that
    does not wait runs beside the producer and is not a dependent at all.
    `prod` replaces the plain producer (keys then start with `prefix`)."""
    E = hx.E
    prod = prod or hx.producer(ds)
    empty, _ = hx.empty(ds.w0, E.MLA_FLAG_PDL)
    empty_wait, _ = hx.empty(ds.w0, E.MLA_FLAG_PDL | E.MLA_HARNESS_EMPTY_WAIT)
    steps = {"producer_us": prod,
             "producer_epilogue_pdl_us": then(prod, hx.epilogue(ds, E.MLA_FLAG_PDL)),
             "producer_epilogue_no_pdl_us": then(prod, hx.epilogue(ds)),
             "producer_empty_pdl_us": then(prod, empty),
             "producer_empty_wait_pdl_us": then(prod, empty_wait)}
    runners = {key: hx.runner(fn, calls) for key, fn in steps.items()}
    out = {k: round(v, 4) for k, v in interleaved_medians(runners, device, calls, reps).items()}
    del runners
    p = out["producer_us"]
    inc = out["producer_epilogue_pdl_us"] - p
    inc_wait = out["producer_empty_wait_pdl_us"] - p
    inc_empty = out["producer_empty_pdl_us"] - p
    out["epilogue_increment_pdl_us"] = round(inc, 4)
    out["epilogue_increment_no_pdl_us"] = round(out["producer_epilogue_no_pdl_us"] - p, 4)
    out["empty_wait_increment_us"] = round(inc_wait, 4)
    out["empty_increment_us"] = round(inc_empty, 4)
    out["floor_ratio_behind_producer"] = round(inc / inc_wait, 3) if inc_wait > 0 else None
    return {prefix + k: v for k, v in out.items()}


def standalone(hx, ds, device, calls, reps, peak):
    """The epilogue alone on cold inputs against the empty kernel of the same
    grid; `calls` None: 20 calls per region for sizes above 32 MiB, else 200."""
    w0 = ds.w0
    if calls is None:
        calls = 20 if ds.bytes_per_call > 32 * 2 ** 20 else 200
    fstep, plan = hx.empty(w0, 0)
    m = interleaved_medians({"epilogue": hx.runner(hx.epilogue(ds), calls), "empty": hx.runner(fstep, calls)},
                            device, calls, reps)
    us, floor_us = m["epilogue"], m["empty"]
    gbs = w0.algorithmic_bytes() / (us * 1e-6) / 1e9
    return {"workload": ds.name, "T": w0.T, "H": w0.H, "flags": flag_names(w0.flags), "mode": mode_name(hx.E, plan),
            "grid": [plan.blocks, plan.threads_per_block], "bytes_per_call": w0.algorithmic_bytes(),
            "traffic": traffic_for(ds.name), "us_per_call": round(us, 4), "gbs": round(gbs, 1),
            "frac": round(gbs / peak, 4), "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4),
            "launch_floor_us": round(floor_us, 4), "floor_ratio": round(us / floor_us, 3), "calls": calls,
            "sets": len(ds.sets), "l2": f"{ds.touched / 2 ** 20:.0f} MiB touched per rotation"}


def mode_name(E, plan):
    return {E.MLA_MODE_SPLIT: "split", E.MLA_MODE_ROWS: "rows"}[plan.mode]


def decode_floors(hx, device, peak, calls=200, reps=7):
    """T = 1 .. 64 (the decode sweep workload: H=16, RoPE, e4m3): standalone
    with cold inputs (`floor_ratio`: against an empty kernel of the same
    grid), and behind two producers with PDL: the plain one, which only
    copies q, and `gemm_`, which first streams GEMM_WEIGHT_BYTES of weights
    as the projection that produces q would.  `floor_ratio_behind_producer`
    is the epilogue's increment over the producer against the increment of
    an empty dependent that waits, `increment_over_launch_floor` the same
    increment against one bare launch of an empty kernel (the median over the
    sizes, `launch_floor_median_us`)."""
    out = []
    pool = torch.ones(GEMM_WEIGHT_POOL_BYTES // 4, dtype=torch.int32, device=device)
    sink = torch.zeros(1, dtype=torch.int32, device=device)
    for T in DECODE_T:
        ds = DeviceSets(f"decode_sweep_t{T}_h16_rope_fp8")
        row = standalone(hx, ds, device, calls, reps, peak)
        row.update(behind_producer(hx, ds, device, calls, reps))
        row.update(behind_producer(hx, ds, device, calls, reps, hx.producer_after_weights(ds, pool, sink), "gemm_"))
        out.append(row)
        del ds
        torch.cuda.empty_cache()
    del pool, sink
    # the epilogue's cost behind each producer against one bare launch: the
    # median over these sizes of the empty kernel's time (the grids differ
    # little; a replay of the empty kernel now and then runs a third faster,
    # and one such reading should not decide a ratio it was not timed with)
    floor = statistics.median(r["launch_floor_us"] for r in out)
    for r in out:
        r["launch_floor_median_us"] = round(floor, 4)
        r["increment_over_launch_floor"] = round(r["epilogue_increment_pdl_us"] / floor, 3)
        r["gemm_increment_over_launch_floor"] = round(r["gemm_epilogue_increment_pdl_us"] / floor, 3)
    return out


def launch_to_end(hx, device, names=("decode_sweep_t1_h16_rope_fp8", "decode_sweep_t4_h16_rope_fp8",
                                     "decode_sweep_t64_h16_rope_fp8"), iters=1000, sleep_cycles=400_000):
    """Device time from an event recorded just before one isolated launch to
    one recorded just after it, for the epilogue and for the empty kernel of
    the same grid: median (and 10th / 90th percentile) of `iters` launches.
    Before each event pair, outside it, the stream writes twice the L2 (cold
    inputs) and then sleeps on the GPU for about 200 us, so the host has
    queued the launch and the closing event before the opening event
    executes: the pair holds the device-side launch, the kernel and its
    completion, not host overhead."""
    E, stream = hx.E, hx.stream
    buf = torch.empty(2 * L2_BYTES // 4, dtype=torch.int32, device=device)
    out = []
    for name in names:
        ds = DeviceSets(name)
        epi = hx.epilogue(ds)
        empty, plan = hx.empty(ds.w0, 0)
        row = {"workload": name, "T": ds.w0.T, "H": ds.w0.H, "mode": mode_name(E, plan), "launches": iters}
        for key, fn in (("epilogue", epi), ("empty", empty)):
            times = []
            for base in range(0, iters, 100):
                pairs = []
                with torch.cuda.stream(stream):
                    for i in range(base, min(iters, base + 100)):
                        buf.fill_(i)
                        torch.cuda._sleep(sleep_cycles)
                        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
                        e0.record(stream)
                        fn(i)
                        e1.record(stream)
                        pairs.append((e0, e1))
                torch.cuda.synchronize()
                times += [a.elapsed_time(b) * 1e3 for a, b in pairs]
            times.sort()
            row[key] = {"median_us": round(statistics.median(times), 3),
                        "p10_us": round(times[len(times) // 10], 3), "p90_us": round(times[9 * len(times) // 10], 3)}
        row["ratio"] = round(row["epilogue"]["median_us"] / row["empty"]["median_us"], 3)
        out.append(row)
        del ds
    del buf
    torch.cuda.empty_cache()
    return out


def producer_consumer_chain(hx, ds, device, calls, reps):
    """Per step: the synthetic producer writes a set's q_nope / q_pe, the
    epilogue runs on that set, and the synthetic consumer reads its q_out and
    cache rows; timed with the epilogue and the consumer launched as
    programmatic dependents (PDL) and without."""
    E, stream = hx.E, hx.stream
    w0 = ds.w0
    scores = torch.empty(w0.T * w0.H, dtype=torch.float32, device=device)
    cflags = (E.MLA_FLAG_Q_FP8 if w0.q_fp8 else 0) | (E.MLA_FLAG_KV_FP8 if w0.kv_fp8 else 0)
    prod = hx.producer(ds)

    def consume(pdl):
        def f(i):
            d, q_out, _ = ds.sets[i % len(ds.sets)]
            rc = E.mla_harness_consume(q_out.data_ptr(), d.cache.data_ptr(), d.slot_mapping.data_ptr(), d.T, d.H,
                                       d.num_blocks * d.block_size, cflags | pdl, scores.data_ptr(),
                                       stream.cuda_stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_harness_consume")
        return f

    out = {"workload": ds.name}
    for key, fn in (("producer_us", prod),
                    ("chain_pdl_us", then(prod, hx.epilogue(ds, E.MLA_FLAG_PDL), consume(E.MLA_FLAG_PDL))),
                    ("chain_no_pdl_us", then(prod, hx.epilogue(ds), consume(0)))):
        r = hx.runner(fn, calls)
        out[key] = round(median_us(r, device, calls, reps), 3)
        del r
    out["pdl_saves_us"] = round(out["chain_no_pdl_us"] - out["chain_pdl_us"], 3)
    out["steps"] = calls
    return out


def split_policy(args):
    """The split / rows crossover: both kernels forced on the same cold
    inputs (RoPE, Q and KV e4m3, std 2, random-byte cache) across T for
    H in {8, 16, 32, 128}; one JSON line per (T, H)."""
    from mla_decode_attention_10_b200 import epilogue as E
    device = torch.device("cuda", 0)
    torch.cuda.set_device(device)
    stream = torch.cuda.Stream(device)
    peak, _ = measured_hbm_gbs()

    def forced(force):
        class Forced(Harness):
            def epilogue(self, ds, extra=0):
                return Harness.epilogue(self, ds, extra | force)

            def empty(self, w0, flags):
                plan = E.mla_epilogue_plan(w0.T, w0.H, w0.flags | force)

                def f(i):
                    rc = E.mla_harness_empty(plan.blocks, plan.threads_per_block, flags, stream.cuda_stream)
                    if rc != E.MLA_OK:
                        raise E.MlaError(rc, "mla_harness_empty")
                return f, plan
        return Forced(E, stream)

    grid = {8: (128, 256, 384, 512, 768), 16: (128, 192, 256, 384, 512), 32: (64, 96, 128, 192, 256),
            128: (16, 24, 32, 48, 64)}
    for H, Ts in grid.items():
        for T in Ts:
            name = f"split_policy_t{T}_h{H}"
            W.RECIPES[name] = dict(T=T, H=H, flags=W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=0,
                                   num_blocks=max(64, 4 * T), std=2.0, rope_rows=32768, scale=0.05,
                                   cache_fill="random", recipe=f"T={T} H={H}, RoPE, Q/KV e4m3, std 2")
            ds = DeviceSets(name)
            row = {"T": T, "H": H, "rows": T * (H + 1)}
            for mode, force in (("split", E.MLA_FLAG_FORCE_SPLIT), ("rows", E.MLA_FLAG_FORCE_ROWS)):
                row[mode + "_us"] = standalone(forced(force), ds, device, 200, 7, peak)["us_per_call"]
            row["plan"] = "split" if E.mla_epilogue_plan(T, H, 0).mode == E.MLA_MODE_SPLIT else "rows"
            print(json.dumps(row), flush=True)
            del ds
            torch.cuda.empty_cache()


def common_config(name: str):
    """The `config` both arms print (plus their own `implementation`)."""
    w = W.RECIPES[name]
    return {"workload": name, "T": w["T"], "H": w["H"], "flags": flag_names(w["flags"]), "recipe": w["recipe"]}


def run_ours(args, rank, world, local_rank):
    from mla_decode_attention_10_b200 import epilogue as E

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    E.lib()  # fail loudly if the CUDA library is missing
    stream = torch.cuda.Stream(device)
    hx = Harness(E, stream)
    peak, peak_note = measured_hbm_gbs()

    # ---- headline workload: K calls per timed region, REPLAYS regions, median
    ds = DeviceSets(args.workload)
    w0 = ds.w0
    runner = hx.runner(hx.epilogue(ds), args.steps, args.warmup)
    fstep, plan = hx.empty(w0, 0)
    frunner = hx.runner(fstep, args.steps, args.warmup)
    for _ in range(args.warmup):
        runner.replay()
    torch.cuda.synchronize()
    # burst: the same regions right after warm-up, before the GPU has reached
    # its sustained power state (context; the headline is the sustained figure)
    burst_ms = statistics.median(timed(runner, device) for _ in range(REPLAYS))

    with ClockSampler(local_rank) as clk:
        # a short soak of the same graphs so that clocks are sampled under this load
        t_soak = time.time()
        while time.time() - t_soak < 1.5:
            runner.replay()
            torch.cuda.synchronize()
        t0 = time.time()
        region_ms = [timed(runner, device) for _ in range(REPLAYS)]
        t1 = time.time()
        time.sleep(0.25)
    clocks = clk.summary(t0, t1)
    ms = statistics.median(region_ms)
    floor_us = median_us(frunner, device, args.steps, REPLAYS)
    del frunner

    l2_note = (f"inputs larger than L2: {len(ds.sets)} rotating input sets touching {ds.touched / 2 ** 20:.0f} MiB "
               "(> 2x L2); L2 written over before every timed region")
    us = job_us_per_call(ms, args.steps, world)
    per_call_us_rank = ms * 1e3 / args.steps
    gbs = w0.algorithmic_bytes() / (per_call_us_rank * 1e-6) / 1e9
    spread = [round(x * 1e3 / args.steps, 4) for x in sorted(region_ms)]

    # the same calls launched as programmatic dependents of the synthetic producer
    headline_pdl = behind_producer(hx, ds, device, min(args.steps, GRAPH_CALLS), CONTEXT_REPLAYS) if w0.producer \
        else None
    del runner

    # ---- end to end through the Python API: pinned host inputs -> call -> q_out to host
    e2e = run_e2e(args, w0, stream, device, world)
    del ds
    torch.cuda.empty_cache()

    # ---- context: decode sizes, launch-to-end latency, other sizes, PDL chain, absorbed query rows
    context, context_errors = {}, []

    def ctx(key, fn):
        try:
            context[key] = fn()
        except Exception as exc:  # noqa: BLE001 -- context only: report, keep the line
            context_errors.append(f"{key}: {type(exc).__name__}: {str(exc).splitlines()[0][:200]}")
        torch.cuda.empty_cache()

    if not args.no_sweep:
        ctx("decode_floors", lambda: decode_floors(hx, device, peak))
        ctx("launch_to_end", lambda: launch_to_end(hx, device))
        ctx("sweep", lambda: [standalone(hx, DeviceSets(n), device, None, CONTEXT_REPLAYS, peak)
                              for n in sweep_names(args.workload)])
        ctx("producer_epilogue_consumer",
            lambda: producer_consumer_chain(hx, DeviceSets("split_boundary_t64_h16_rope"), device, 200,
                                            CONTEXT_REPLAYS))
        ctx("absorbed_query", lambda: absorb_measure(E, stream, device, peak))

    config = dict(common_config(args.workload), implementation=IMPLEMENTATION)
    line = {
        "metric": METRIC, "value": round(us, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": config,
        "timing": {"mode": mode_name(E, plan), "grid": [plan.blocks, plan.threads_per_block],
                   "regions": REPLAYS, "region_us_per_call_sorted": spread,
                   "l2": l2_note,
                   "method": f"median of {REPLAYS} timed regions, each one replay of CUDA graphs holding the "
                             f"{args.steps} calls (<= {GRAPH_CALLS} per graph) on one stream, CUDA events on that "
                             "stream, barrier + synchronize around each region, after 1.5 s of the same load "
                             "(sustained power state; the clocks are sampled there)",
                   "burst_us_per_call": round(job_us_per_call(burst_ms, args.steps, world), 4),
                   "burst_note": "the same regions right after warm-up, before the soak",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "gbs": round(gbs, 1),
        "launch_floor_us": round(floor_us, 4),
        "floor_ratio": round(per_call_us_rank / floor_us, 3),
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": traffic_for(args.workload),
                     "algorithmic_bytes": w0.algorithmic_bytes(), "peak_source": peak_note,
                     "frac_nominal_8tbs": round(gbs / NOMINAL_HBM_GBS, 4)},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks,
    }
    if headline_pdl is not None:
        line["behind_producer"] = headline_pdl
    line.update(context)
    if context_errors:
        line["context_errors"] = context_errors
    if rank == 0 and not args.no_cpu_baseline and world == 1:
        line["cpu_baseline"] = cpu_baseline(args.workload)
        line["cpu_baseline_all_cores"] = cpu_baseline_all_cores(args.workload)
    return line


def flag_names(f: int) -> str:
    names = [n for bit, n in ((W.FLAG_ROPE, "rope"), (W.FLAG_Q_FP8, "q_fp8"), (W.FLAG_KV_FP8, "kv_fp8"))
             if f & bit]
    return "+".join(names) if names else "none"


def sweep_names(headline: str):
    names = ["decode_t4_h16", "split_boundary_t64_h16_rope", "split_boundary_t65_h16_rope",
             "decode_sweep_t128_h16_rope_fp8", "decode_sweep_t256_h16_rope_fp8",
             "prefill_t1024_h128_strided", "batch_t8192_h16_pdl_fp8"]
    return [n for n in names if n != headline]


def absorb_measure(E, stream, device, peak_gbs):
    """The query side with the absorption product folded in (tcgen05 kernel)
    at T=8192, H=16, RoPE, e4m3, against the same work unfused: a cuBLAS
    batched matmul writing the 512-wide product, then the epilogue (which
    also writes the cache rows)."""
    try:
        peak_tf = float(json.load(open(os.path.join(ROOT, "MEASURED_PEAKS.json")))["bf16_tflops"])
    except (OSError, KeyError, ValueError):
        peak_tf = 1590.0
    sets = []
    for k in range(2):
        w = W.make_absorb("absorb_t8192_h16_rope_fp8", 8192, 16, W.FLAG_ROPE | W.FLAG_Q_FP8, seed=k,
                          rope_rows=131072).to(device)
        q_out = torch.empty((w.T, w.H, W.ROW), dtype=torch.uint8, device=device)
        sets.append((w, q_out))
    w0 = sets[0][0]

    def fused(i):
        w, q = sets[i % 2]
        rc = E.launch_absorb_workload(w, q, stream=stream)
        if rc != E.MLA_OK:
            raise E.MlaError(rc, "mla_absorb_launch")

    n = 20
    r = GraphRunner(fused, n, stream)
    r.replay()
    torch.cuda.synchronize()
    us = median_us(r, device, n, CONTEXT_REPLAYS)
    del r
    # unfused: torch.bmm (cuBLAS) for the product, then the epilogue on it
    e_sets = []
    for k, (w, q) in enumerate(sets):
        ew = W.make("absorb_unfused", w.T, w.H, W.FLAG_ROPE | W.FLAG_Q_FP8 | W.FLAG_KV_FP8, seed=k,
                    num_blocks=16384, rope_rows=131072).to(device)
        ql = torch.empty((w.H, w.T, W.NOPE), dtype=torch.bfloat16, device=device)
        ew.q_nope = ql.transpose(0, 1)
        ew.q_pe = w.q_pe
        e_sets.append((w, ew, ql, torch.empty((w.T, w.H, W.ROW), dtype=torch.uint8, device=device)))

    def bmm_only(i):
        w, _, ql, _ = e_sets[i % 2]
        with torch.cuda.stream(stream):
            torch.bmm(w.q_nope_c.transpose(0, 1), w.w_uk.transpose(1, 2), out=ql)

    def unfused(i):
        bmm_only(i)
        _, ew, _, q = e_sets[i % 2]
        rc = E.launch_workload(ew, q, stream=stream)
        if rc != E.MLA_OK:
            raise E.MlaError(rc, "mla_epilogue_launch")

    # cuBLAS creates its handle and workspace on first use, which cannot happen inside a graph capture
    bmm_only(0)
    torch.cuda.synchronize()
    out = {}
    for key, fn in (("bmm_us", bmm_only), ("bmm_plus_epilogue_us", unfused)):
        g = GraphRunner(fn, n, stream)
        g.replay()
        torch.cuda.synchronize()
        out[key] = round(median_us(g, device, n, CONTEXT_REPLAYS), 3)
        del g
    gbs = w0.algorithmic_bytes() / (us * 1e-6) / 1e9
    tfs = w0.flops() / (us * 1e-6) / 1e12
    return {"workload": "absorb_t8192_h16_rope_fp8",
            "recipe": "T=8192 H=16: q_nope_c [8192,16,128] and q_pe bf16 N(0,1), W_UK [16,512,128] N(0,1/128), "
                      "RoPE (131072-row table), e4m3 scale 0.05; two input sets, seeds 0 and 1",
            "us_per_call": round(us, 3), "bytes_per_call": w0.algorithmic_bytes(), "flops_per_call": w0.flops(),
            "gbs": round(gbs, 1), "frac_hbm": round(gbs / peak_gbs, 4), "tflops": round(tfs, 1),
            "frac_tensor": round(tfs / peak_tf, 4), "bound": "hbm" if gbs / peak_gbs > tfs / peak_tf else "tensor",
            **out}


def run_e2e(args, w0, stream, device, world):
    """Same metric through the user-facing call, with host buffers: every step
    copies its inputs from pinned host memory, runs the epilogue and copies
    q_out back, timed with CUDA events.  The per-step inputs (q_nope, q_pe,
    kv_c, k_pe, slot_mapping, positions) sit in one pinned staging buffer at
    16-byte aligned offsets, so each step is one host-to-device copy, the
    call, and one device-to-host copy.

    Two schedules.  Serial: all three on the launch stream, one step after
    the other.  Pipelined (the reported value; the user-facing call is made
    every step): uploads, calls and downloads on three streams over two
    buffer sets, the way a serving loop overlaps them: step i+1's upload runs
    while step i computes and step i-1's result comes back; events order
    every reuse of a buffer."""
    from mla_decode_attention_10_b200 import epilogue as E
    parts = [(k, getattr(w0, k).contiguous()) for k in ("q_nope", "q_pe", "kv_c", "k_pe", "slot_mapping", "positions")
             if getattr(w0, k) is not None]
    offsets, total = {}, 0
    for k, v in parts:
        offsets[k] = total
        total += -(-v.numel() * v.element_size() // 16) * 16
    cache = w0.cache.to(device)
    cos_sin = w0.cos_sin.to(device) if w0.cos_sin is not None else None
    qs = w0.q_scale.to(device) if w0.q_scale is not None else None
    ks = w0.kv_scale.to(device) if w0.kv_scale is not None else None

    def buffer_set():
        host = torch.empty(total, dtype=torch.uint8).pin_memory()
        for k, v in parts:
            n = v.numel() * v.element_size()
            host[offsets[k]:offsets[k] + n].copy_(v.view(-1).view(torch.uint8))
        dbuf = torch.empty(total, dtype=torch.uint8, device=device)
        dev = {k: dbuf[offsets[k]:offsets[k] + v.numel() * v.element_size()].view(v.dtype).view(v.shape)
               for k, v in parts}
        q_out = torch.empty((w0.T, w0.H, W.ROW), dtype=w0.q_out_dtype(), device=device)
        q_host = torch.empty(q_out.shape, dtype=q_out.dtype).pin_memory()
        return {"host": host, "dbuf": dbuf, "dev": dev, "q_out": q_out, "q_host": q_host}

    sets = [buffer_set(), buffer_set()]
    h2d = sum(v.numel() * v.element_size() for _, v in parts)
    d2h = sets[0]["q_host"].numel() * sets[0]["q_host"].element_size()

    def call(b, s):
        dev = b["dev"]
        E.fused_mla_decode_q_concat_kv_cache_insert(
            dev["q_nope"], dev["q_pe"], dev["kv_c"], dev["k_pe"], cache, dev["slot_mapping"],
            positions=dev.get("positions"), cos_sin=cos_sin, q_scale=qs, kv_scale=ks, q_out=b["q_out"], stream=s)

    def serial_step(i):
        b = sets[0]
        with torch.cuda.stream(stream):
            b["dbuf"].copy_(b["host"], non_blocking=True)
            call(b, stream)
            b["q_host"].copy_(b["q_out"], non_blocking=True)

    up, down = torch.cuda.Stream(device=device), torch.cuda.Stream(device=device)
    ev = [{n: torch.cuda.Event() for n in ("up", "comp", "down")} for _ in sets]
    for e in ev:  # every event starts out recorded, so the first waits pass
        for n in e:
            e[n].record(stream)

    def pipelined_step(i):
        b, e = sets[i % 2], ev[i % 2]
        up.wait_event(e["comp"])   # the call two steps back has read this input buffer
        with torch.cuda.stream(up):
            b["dbuf"].copy_(b["host"], non_blocking=True)
        e["up"].record(up)
        stream.wait_event(e["up"])
        stream.wait_event(e["down"])  # the download two steps back has read this q_out
        call(b, stream)
        e["comp"].record(stream)
        down.wait_event(e["comp"])
        with torch.cuda.stream(down):
            b["q_host"].copy_(b["q_out"], non_blocking=True)
        e["down"].record(down)

    def timed_run(step_fn, k):
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        torch.cuda.synchronize()
        barrier(device)
        e0.record(stream)
        up.wait_stream(stream)
        down.wait_stream(stream)
        for i in range(k):
            step_fn(i)
        stream.wait_stream(up)
        stream.wait_stream(down)
        e1.record(stream)
        torch.cuda.synchronize()
        barrier(device)
        return max_over_ranks(e0.elapsed_time(e1), device)

    k = max(10, min(args.steps, 100))
    for i in range(max(args.warmup, 3)):
        serial_step(i)
    serial_ms = timed_run(serial_step, k)
    for i in range(max(args.warmup, 3)):
        pipelined_step(i)
    pipe_ms = timed_run(pipelined_step, k)
    return {"value": round(job_us_per_call(pipe_ms, k, world), 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": k,
            "serial_value": round(job_us_per_call(serial_ms, k, world), 3),
            "path": "epilogue.fused_mla_decode_q_concat_kv_cache_insert; per step one host-to-device copy of the "
                    "inputs from a pinned staging buffer, the call, and q_out back to pinned host memory; value: "
                    "uploads, calls and downloads pipelined on three streams over two buffer sets, the call made "
                    "every step; serial_value: all on the launch stream, one step after the other"}


# ---------------------------------------------------------------------------------------
# CPU oracle: the baseline and the reference arm
# ---------------------------------------------------------------------------------------

def _oracle_call(w, threads=1):
    import oracle
    return oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, w.cache, w.flags,
                      positions=w.positions, cos_sin=w.cos_sin, q_scale=w.q_scale, kv_scale=w.kv_scale,
                      threads=threads)


def token_slice(w: W.Workload, n: int) -> W.Workload:
    """The first n tokens of a workload (same cache, table and scales): a
    bounded sample of the same work, n/T of a call."""
    if n >= w.T:
        return w
    import dataclasses
    return dataclasses.replace(w, T=n, q_nope=w.q_nope[:n], q_pe=w.q_pe[:n], kv_c=w.kv_c[:n], k_pe=w.k_pe[:n],
                               slot_mapping=w.slot_mapping[:n],
                               positions=None if w.positions is None else w.positions[:n])


def sampled_oracle(w: W.Workload, seconds: float, threads: int = 1):
    """Time the oracle, as it stands, on token slices of `w` for about
    `seconds` of host time; returns (µs per full call, calls, tokens per call)."""
    probe = token_slice(w, max(1, w.T // 16))
    t0 = time.perf_counter()
    _oracle_call(probe, threads)
    est_full = (time.perf_counter() - t0) * w.T / probe.T
    n_tok = w.T if est_full <= seconds / 4 else max(1, int(w.T * seconds / 4 / est_full))
    s = token_slice(w, n_tok)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds or n == 0:
        _oracle_call(s, threads)
        n += 1
    dt = time.perf_counter() - t0
    return dt / n * 1e6 * w.T / n_tok, n, n_tok


def cpu_baseline(name: str, seconds: float = 12.0):
    """The single-threaded CPU oracle, as it stands, on token slices of the
    workload for about `seconds` of host time, scaled to one full call."""
    w = named_variant(name, 0)
    us, n, n_tok = sampled_oracle(w, seconds)
    return {"value": round(us, 2), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} calls on {n_tok} of the {w.T} tokens of {name} (H={w.H}) in ~{seconds:.0f} s, one host "
                      f"thread, scaled by {w.T}/{n_tok} ({os.cpu_count()} cores on the host)"}


def cpu_baseline_all_cores(name: str, seconds: float = 6.0):
    """The same oracle function, as it stands, on contiguous token slices on
    every host core at once (one std::thread per slice inside the oracle
    library).  Reported as a baseline only."""
    w = named_variant(name, 0)
    cores = max(1, min(os.cpu_count() or 1, w.T))
    us, n, n_tok = sampled_oracle(w, seconds, threads=cores)
    return {"value": round(us, 2), "unit": UNIT, "cores": cores, "kind": "oracle, token slices on threads",
            "sample": f"{n} calls on {n_tok} of the {w.T} tokens of {name} in ~{seconds:.0f} s, {cores} threads, "
                      f"scaled by {w.T}/{n_tok}; baseline only"}


def run_reference(args, rank, world, budget_s: float = 150.0):
    """The oracle as the reference arm: every step a token slice of the
    workload sized so that warm-up and timed steps together take about
    `budget_s` seconds at most, its time scaled to a full call."""
    if rank != 0:
        return None
    w = named_variant(args.workload, 0)
    probe = token_slice(w, max(1, w.T // 16))
    t0 = time.perf_counter()
    _oracle_call(probe)
    est_full = (time.perf_counter() - t0) * w.T / probe.T
    per_step = budget_s / (args.steps + args.warmup)
    n_tok = w.T if est_full <= per_step else max(1, int(w.T * per_step / est_full))
    s = token_slice(w, n_tok)
    for _ in range(args.warmup):
        _oracle_call(s)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_call(s)
    dt = time.perf_counter() - t0
    us = dt / args.steps * 1e6 * w.T / n_tok
    sample = (f"{args.steps} steps, each the oracle on {n_tok} of the {w.T} tokens of {args.workload} (H={w.H}), "
              f"one host thread, scaled by {w.T}/{n_tok}")
    cb = {"value": round(us, 3), "unit": UNIT, "cores": 1, "kind": "oracle", "sample": sample}
    return {"impl": "reference", "metric": METRIC, "value": round(us, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(us / 1e3, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "f32",
            "data": "synthetic",
            "config": dict(common_config(args.workload), implementation="CPU oracle (oracle/mla_oracle.cpp), "
                                                                        "one host thread"),
            "cpu_baseline": cb,
            "e2e": {"value": round(us, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------------------

def parse(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=20)
    p.add_argument("--warmup", type=int, default=5)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=HEADLINE, choices=W.names())
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    p.add_argument("--split-policy", action="store_true",
                   help="measure the split / rows crossover instead (one JSON line per shape)")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be at least 3")
    if a.steps < 1:
        p.error("--steps must be positive")
    return a


def main(argv=None):
    args = parse(argv)
    rank, world, local_rank = rank_info()
    if args.split_policy:
        split_policy(args)
        return 0
    if args.impl == "reference":
        line = run_reference(args, rank, world)
        if line is not None:
            print(json.dumps(line), flush=True)
        return 0
    if world > 1:
        import torch.distributed as dist
        torch.cuda.set_device(local_rank)
        dist.init_process_group("nccl", timeout=_dt.timedelta(seconds=120),
                                device_id=torch.device("cuda", local_rank))
    try:
        line = run_ours(args, rank, world, local_rank)
        if rank == 0:
            print(json.dumps(line), flush=True)
    finally:
        if world > 1:
            import torch.distributed as dist
            dist.destroy_process_group()
    return 0


if __name__ == "__main__":
    sys.exit(main())
