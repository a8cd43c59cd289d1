"""Benchmark of the fused MLA decode epilogue on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]
                    [--workload NAME] [--no-sweep] [--no-cpu-baseline]

One step is one call of the epilogue (the whole hot path) on one batch of
the workload.  Default workload: the row-split boundary case, T=64 tokens,
H=16 heads, bf16, RoPE (the decode size at which the vLLM PR #54896 report
switches to three warps per row).  Inputs are device-resident when the timed
region starts; consecutive steps rotate over input sets whose total is more
than twice the L2, so every step reads HBM.  The K calls are replayed from
CUDA graphs on one stream and timed with CUDA events on that stream; the
bare-launch floor is an empty kernel with the same grid, block and launch
attributes, timed the same way.

Printed: one JSON line (rank 0) with the metric in microseconds per call,
achieved HBM GB/s against the measured copy bandwidth, the launch floor, a
sweep over the other workload sizes, the end-to-end time through the Python
API with pinned host buffers, the CPU oracle as a baseline and the SM clocks
seen under load.  ``--impl reference`` times the CPU oracle instead (the only
reference implementation this operation has here).
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
HEADLINE = "split_boundary_t64_h16_rope"
FALLBACK_HBM_GBS = 6650.0

# DRAM bytes (dram__bytes_read.sum + dram__bytes_write.sum) of one launch of
# the epilogue kernel, from ncu captures of `bench.py --steps 3 --warmup 3
# --no-sweep --no-cpu-baseline --workload <name>` (third launch; summaries in
# profiles/).  Keyed by a hash of the kernel sources they were taken on: a
# changed kernel reports null until it is captured again.
KERNEL_SOURCES = ("mla_decode_attention_10_b200/csrc/mla_epilogue.cu",
                  "mla_decode_attention_10_b200/csrc/latent_math.cuh", "include/mla_epilogue.h")
TRAFFIC_SOURCE_HASH = "097d8a46e6e610e8"
TRAFFIC_BYTES = {
    "split_boundary_t64_h16_rope": 1277952 + 0,
    "prefill_t1024_h128_strided": 152627456 + 102022400,
    "batch_t8192_h16_pdl_fp8": 164003328 + 55213568,
}
L2_BYTES = 126 * 2 ** 20
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

def run_ours(args, rank, world, local_rank):
    from mla_decode_attention_10_b200 import epilogue as E

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    E.lib()  # fail loudly if the CUDA library is missing
    stream = torch.cuda.Stream(device)
    peak, peak_note = measured_hbm_gbs()

    def epilogue_step(ds, extra=0, single_set=False):
        def f(i):
            d, q_out, _ = ds.sets[0 if single_set else i % len(ds.sets)]
            rc = E.launch_workload(d, q_out, extra_flags=extra, stream=stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_epilogue_launch")
        return f

    def floor_step(T, H, flags):
        plan = E.mla_epilogue_plan(T, H, flags)

        def f(i):
            rc = E.mla_harness_empty(plan.blocks, plan.threads_per_block, flags & E.MLA_FLAG_PDL, stream.cuda_stream)
            if rc != E.MLA_OK:
                raise E.MlaError(rc, "mla_harness_empty")
        return f, plan

    def measure(step, steps, warmup):
        warm = GraphRunner(step, max(warmup, 1), stream)
        warm.replay()
        torch.cuda.synchronize()
        runner = GraphRunner(step, steps, stream)
        runner.replay()  # first replay uploads the graphs
        torch.cuda.synchronize()
        return runner

    # ---- headline workload
    ds = DeviceSets(args.workload)
    w0 = ds.w0
    step = epilogue_step(ds)
    runner = measure(step, args.steps, args.warmup)
    fstep, plan = floor_step(w0.T, w0.H, 0)
    frunner = measure(fstep, args.steps, args.warmup)
    for _ in range(args.warmup):
        runner.replay()
    torch.cuda.synchronize()

    with ClockSampler(local_rank) as clk:
        # a short soak of the same graphs so that clocks are sampled under this load
        t_soak = time.time()
        while time.time() - t_soak < 1.5:
            runner.replay()
            torch.cuda.synchronize()
        t0 = time.time()
        ms = timed(runner, device)
        t1 = time.time()
        time.sleep(0.25)
    clocks = clk.summary(t0, t1)
    floor_ms = timed(frunner, device)

    us = job_us_per_call(ms, args.steps, world)
    per_call_us_rank = ms * 1e3 / args.steps
    gbs = w0.algorithmic_bytes() / (per_call_us_rank * 1e-6) / 1e9
    floor_us = floor_ms * 1e3 / args.steps

    # PDL-chained variant of the same call sequence (each call a programmatic
    # dependent of the previous one; sets are disjoint, so the contract holds)
    prunner = measure(epilogue_step(ds, E.MLA_FLAG_PDL), args.steps, args.warmup)
    pfstep, _ = floor_step(w0.T, w0.H, E.MLA_FLAG_PDL)
    pfrunner = measure(pfstep, args.steps, args.warmup)
    pdl_us = timed(prunner, device) * 1e3 / args.steps
    pdl_floor_us = timed(pfrunner, device) * 1e3 / args.steps
    del prunner, pfrunner

    # same inputs every call: they stay in L2, as when the upstream kernel has just written them
    wrunner = measure(epilogue_step(ds, 0, single_set=True), args.steps, args.warmup)
    warm_us = timed(wrunner, device, flush=False) * 1e3 / args.steps
    del wrunner

    # producer -> epilogue -> consumer, with and without programmatic dependent launch
    chain = producer_consumer_chain(ds, E, stream, device, min(args.steps, 500), args.warmup)

    # ---- end to end through the Python API: pinned host inputs -> call -> q_out to host
    e2e = run_e2e(args, w0, stream, device, world)

    # ---- sweep of the other sizes (their own bench lines are not printed; this is context)
    # the headline is measured; what follows is context, and an error in it is
    # reported in the line rather than losing the line
    sweep = []
    context_errors = []
    if not args.no_sweep:
        for name in sweep_names(args.workload):
            try:
                sweep.append(sweep_one(name, E, stream, device, peak, epilogue_step, floor_step, measure))
            except Exception as exc:  # noqa: BLE001
                context_errors.append(f"{name}: {type(exc).__name__}: {str(exc).splitlines()[0][:200]}")
            torch.cuda.empty_cache()

    absorb = None
    if not args.no_sweep:
        try:
            absorb = absorb_measure(E, stream, device, peak)
        except Exception as exc:  # noqa: BLE001
            context_errors.append(f"absorbed_query: {type(exc).__name__}: {str(exc).splitlines()[0][:200]}")

    line = {
        "metric": METRIC, "value": round(us, 4), "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": round(ms / args.steps, 6), "higher_is_better": False,
        "scaling": "weak", "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": {"workload": args.workload, "T": w0.T, "H": w0.H, "flags": flag_names(w0.flags),
                   "recipe": w0.recipe, "mode": "split" if plan.mode == E.MLA_MODE_SPLIT else "rows",
                   "grid": [plan.blocks, plan.threads_per_block],
                   "l2": f"inputs larger than L2: {len(ds.sets)} rotating input sets touching "
                         f"{ds.touched / 2 ** 20:.0f} MiB (> 2x L2); L2 written over before each timed region",
                   "timing": f"CUDA graphs of <= {GRAPH_CALLS} calls on one stream, CUDA events",
                   "parallelism": "replicas" if world > 1 else "single GPU"},
        "gbs": round(gbs, 1),
        "launch_floor_us": round(floor_us, 4),
        "floor_ratio": round(per_call_us_rank / floor_us, 3),
        "pdl_chain": {"us_per_call": round(pdl_us, 4), "floor_us": round(pdl_floor_us, 4),
                      "floor_ratio": round(pdl_us / pdl_floor_us, 3),
                      "note": "each call a programmatic dependent of the previous one (disjoint input sets)"},
        "l2_warm": {"us_per_call": round(warm_us, 4), "floor_ratio": round(warm_us / floor_us, 3),
                    "note": "the same inputs every call, so they are L2-resident (not the headline: the "
                            "headline reads HBM)"},
        "producer_epilogue_consumer": chain,
        "roofline": {"bound": "hbm", "achieved": round(gbs, 1), "peak": peak, "unit": "GB/s",
                     "frac": round(gbs / peak, 4), "traffic": traffic_for(args.workload),
                     "algorithmic_bytes": w0.algorithmic_bytes(),
                     "peak_source": peak_note,
                     "note": "decode-size call: launch and memory latency bound, not bandwidth bound; "
                             "see sweep for the bandwidth-bound sizes. traffic counts DRAM bytes inside the "
                             "launch: written rows stay in L2 (write-back) and reach DRAM later"},
        "e2e": e2e,
        "gpu_launches": args.steps,
        "clocks": clocks,
        "sweep": sweep,
    }
    if absorb is not None:
        line["absorbed_query"] = absorb
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
    names = ["decode_t4_h16", "split_boundary_t64_h16_rope", "split_boundary_t65_h16_rope"]
    names += [f"decode_sweep_t{t}_h16_rope_fp8" for t in W.DECODE_SWEEP_T]
    names += ["prefill_t1024_h128_strided", "batch_t8192_h16_pdl_fp8"]
    return [n for n in names if n != headline]


def sweep_one(name, E, stream, device, peak, epilogue_step, floor_step, measure, steps=None):
    ds = DeviceSets(name)
    w0 = ds.w0
    big = w0.algorithmic_bytes() > 32 * 2 ** 20
    n = steps or (20 if big else max(1000, len(ds.sets)))
    r = measure(epilogue_step(ds), n, 3)
    us = timed(r, device) * 1e3 / n
    fstep, plan = floor_step(w0.T, w0.H, 0)
    fr = measure(fstep, n, 3)
    floor_us = timed(fr, device) * 1e3 / n
    gbs = w0.algorithmic_bytes() / (us * 1e-6) / 1e9
    out = {"workload": name, "T": w0.T, "H": w0.H, "flags": flag_names(w0.flags),
           "mode": "split" if plan.mode == E.MLA_MODE_SPLIT else "rows",
           "bytes_per_call": w0.algorithmic_bytes(), "traffic": traffic_for(name), "us_per_call": round(us, 3),
           "gbs": round(gbs, 1), "frac": round(gbs / peak, 4), "launch_floor_us": round(floor_us, 3),
           "floor_ratio": round(us / floor_us, 3), "calls": n, "sets": len(ds.sets),
           "l2": f"{ds.touched / 2 ** 20:.0f} MiB touched per rotation"}
    if w0.producer:
        out.update(producer_pdl(ds, E, stream, device, n))
    del r, fr
    return out


def producer_pdl(ds, E, stream, device, n):
    """Producer alone vs producer + epilogue launched with PDL behind it."""
    def prod(i):
        d, _, (sn, sp) = ds.sets[i % len(ds.sets)]
        rc = E.mla_harness_produce(sn.data_ptr(), sp.data_ptr(), d.q_nope.data_ptr(), d.q_nope.stride(0),
                                   d.q_nope.stride(1), d.q_pe.data_ptr(), d.q_pe.stride(0), d.q_pe.stride(1),
                                   d.T, d.H, 0, stream.cuda_stream)
        assert rc == E.MLA_OK

    def pair(i):
        prod(i)
        d, q_out, _ = ds.sets[i % len(ds.sets)]
        rc = E.launch_workload(d, q_out, extra_flags=E.MLA_FLAG_PDL, stream=stream)
        assert rc == E.MLA_OK

    def pair_nopdl(i):
        prod(i)
        d, q_out, _ = ds.sets[i % len(ds.sets)]
        rc = E.launch_workload(d, q_out, stream=stream)
        assert rc == E.MLA_OK

    res = {}
    for key, fn in (("producer_us", prod), ("producer_plus_epilogue_pdl_us", pair),
                    ("producer_plus_epilogue_no_pdl_us", pair_nopdl)):
        g = GraphRunner(fn, n, stream)
        g.replay()
        torch.cuda.synchronize()
        res[key] = round(timed(g, device) * 1e3 / n, 3)
        del g
    res["epilogue_increment_pdl_us"] = round(res["producer_plus_epilogue_pdl_us"] - res["producer_us"], 3)
    return res


def producer_consumer_chain(ds, E, stream, device, n, warmup):
    """Per step: the synthetic producer writes a set's q_nope / q_pe, the
    epilogue runs on that set, and the synthetic consumer reads its q_out and
    cache rows.  Timed with the epilogue and the consumer launched as
    programmatic dependents (PDL) and without; `producer_us` alone for
    reference.  Values do not matter here (the producer copies the next
    set's query inputs); stream order keeps every step after the last."""
    S = len(ds.sets)
    w0 = ds.w0
    scores = torch.empty(w0.T * w0.H, dtype=torch.float32, device=device)
    cflags = (E.MLA_FLAG_Q_FP8 if w0.q_fp8 else 0) | (E.MLA_FLAG_KV_FP8 if w0.kv_fp8 else 0)

    sources = {}

    def source(k):
        # the producer reads contiguous [T,H,512] / [T,H,64] buffers
        if k not in sources:
            d, _, src = ds.sets[k]
            sources[k] = src if src is not None else (d.q_nope.contiguous(), d.q_pe.contiguous())
        return sources[k]

    def prod(i):
        d, _, _ = ds.sets[i % S]
        sn, sp = source((i + 1) % S) if ds.sets[i % S][2] is None else source(i % S)
        rc = E.mla_harness_produce(sn.data_ptr(), sp.data_ptr(), d.q_nope.data_ptr(), d.q_nope.stride(0),
                                   d.q_nope.stride(1), d.q_pe.data_ptr(), d.q_pe.stride(0), d.q_pe.stride(1),
                                   d.T, d.H, 0, stream.cuda_stream)
        assert rc == E.MLA_OK

    def chain(pdl):
        def f(i):
            prod(i)
            d, q_out, _ = ds.sets[i % S]
            assert E.launch_workload(d, q_out, extra_flags=pdl, stream=stream) == E.MLA_OK
            assert E.mla_harness_consume(q_out.data_ptr(), d.cache.data_ptr(), d.slot_mapping.data_ptr(), d.T, d.H,
                                         d.num_blocks * d.block_size, cflags | pdl, scores.data_ptr(),
                                         stream.cuda_stream) == E.MLA_OK
        return f

    out = {}
    for key, fn in (("producer_us", prod), ("chain_pdl_us", chain(E.MLA_FLAG_PDL)), ("chain_no_pdl_us", chain(0))):
        g = GraphRunner(fn, n, stream)
        g.replay()
        torch.cuda.synchronize()
        out[key] = round(timed(g, device) * 1e3 / n, 3)
        del g
    out["pdl_saves_us"] = round(out["chain_no_pdl_us"] - out["chain_pdl_us"], 3)
    out["steps"] = n
    return out


def absorb_measure(E, stream, device, peak_gbs):
    """The query side with the absorption product folded in (tcgen05 kernel)
    at T=8192, H=16, RoPE, e4m3, against the same work unfused: a cuBLAS
    batched matmul writing the 512-wide product, then the epilogue (which
    also writes the cache rows)."""
    peak_tf = None
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
        assert E.launch_absorb_workload(w, q, stream=stream) == E.MLA_OK

    n = 20
    r = GraphRunner(fused, n, stream)
    r.replay()
    torch.cuda.synchronize()
    us = min(timed(r, device) for _ in range(3)) * 1e3 / n
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
        assert E.launch_workload(ew, q, stream=stream) == E.MLA_OK

    # cuBLAS creates its handle and workspace on first use, which cannot happen inside a graph capture
    bmm_only(0)
    torch.cuda.synchronize()
    out = {}
    for key, fn in (("bmm_us", bmm_only), ("bmm_plus_epilogue_us", unfused)):
        g = GraphRunner(fn, n, stream)
        g.replay()
        torch.cuda.synchronize()
        out[key] = round(min(timed(g, device) for _ in range(3)) * 1e3 / n, 3)
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

    Three schedules are timed.  Serial: all three on the launch stream, one
    step after the other.  Pipelined (the reported value: the user-facing
    call is made every step): uploads, calls and downloads on three streams
    with two buffer sets, the way a serving loop overlaps them: step i+1's
    upload runs while step i computes and step i-1's result comes back;
    events order every reuse of a buffer.  Graphed (context): the pipelined
    schedule of 20 steps captured once as a CUDA graph, with its copy nodes,
    and replayed, as decode loops launch their steps; every replayed step
    still moves its inputs and its result over the host link."""
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

    def serial_step():
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

    def pipelined_step(i, first=False):
        b, e = sets[i % 2], ev[i % 2]
        if not first:
            up.wait_event(e["comp"])   # the call two steps back has read this input buffer
        with torch.cuda.stream(up):
            b["dbuf"].copy_(b["host"], non_blocking=True)
        e["up"].record(up)
        stream.wait_event(e["up"])
        if not first:
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

    k = max(10, min(args.steps, 200))
    for _ in range(max(args.warmup, 3)):
        serial_step()
    serial_ms = timed_run(lambda i: serial_step(), k)
    for i in range(max(args.warmup, 3)):
        pipelined_step(i)
    pipe_ms = timed_run(pipelined_step, k)
    # the same schedule as one CUDA graph of G steps (the first two steps of
    # a replay wait for nothing: the previous replay has completed)
    G = 20
    graph_ms, graph_note, g = None, None, None
    try:
        torch.cuda.synchronize()
        g = torch.cuda.CUDAGraph()
        with torch.cuda.graph(g, stream=stream):
            up.wait_stream(stream)
            down.wait_stream(stream)
            for i in range(G):
                pipelined_step(i, first=i < 2)
            stream.wait_stream(up)
            stream.wait_stream(down)
        with torch.cuda.stream(stream):
            for _ in range(2):
                g.replay()
        torch.cuda.synchronize()
    except RuntimeError as exc:  # capture refused: report the stream-pipelined figure
        graph_note = f"graph capture failed: {exc}"[:200]
        g = None
    # every rank takes the same branch, so the collectives inside timed_run match
    if max_over_ranks(0.0 if g is not None else 1.0, device) == 0.0:
        reps = max(1, k // G)

        def replay(i):
            with torch.cuda.stream(stream):
                g.replay()

        graph_ms = timed_run(replay, reps)
        graph_steps = G * reps
    elif graph_note is None:
        graph_note = "graph capture failed on another rank"
    out = {"value": round(job_us_per_call(pipe_ms, k, world), 3), "unit": UNIT, "h2d_bytes_per_step": h2d,
            "d2h_bytes_per_step": d2h, "steps": k,
            "graphed_value": (round(job_us_per_call(graph_ms, graph_steps, world), 3)
                              if graph_ms is not None else None),
            "serial_value": round(job_us_per_call(serial_ms, k, world), 3),
            "path": "epilogue.fused_mla_decode_q_concat_kv_cache_insert; per step one host-to-device copy of the "
                    "inputs from a pinned staging buffer, the call, and q_out back to pinned host memory; value: "
                    "uploads, calls and downloads pipelined on three streams over two buffer sets, the call made "
                    "every step; graphed_value: the same schedule captured as a CUDA graph of 20 steps and "
                    "replayed; serial_value: all on the launch stream, one step after the other"}
    if graph_note:
        out["note"] = graph_note
    return out


# ---------------------------------------------------------------------------------------
# CPU oracle: the baseline and the reference arm
# ---------------------------------------------------------------------------------------

def _oracle_call(w):
    import oracle
    return oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, w.cache, w.flags,
                      positions=w.positions, cos_sin=w.cos_sin, q_scale=w.q_scale, kv_scale=w.kv_scale)


def cpu_baseline(name: str, seconds: float = 10.0):
    """The single-threaded CPU oracle, as it stands, repeated on the workload
    for about `seconds` of host time."""
    w = named_variant(name, 0)
    _oracle_call(w)
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        _oracle_call(w)
        n += 1
    dt = time.perf_counter() - t0
    return {"value": round(dt / n * 1e6, 2), "unit": UNIT, "cores": 1, "kind": "oracle",
            "sample": f"{n} calls of {name} (T={w.T}, H={w.H}) in {dt:.1f} s, one host thread "
                      f"({os.cpu_count()} cores on the host)"}


def cpu_baseline_all_cores(name: str, seconds: float = 5.0):
    """The same oracle function, as it stands, on contiguous token slices on
    every host core at once (one std::thread per slice inside the oracle
    library).  Reported as a baseline only."""
    import oracle
    w = named_variant(name, 0)
    cores = max(1, min(os.cpu_count() or 1, w.T))

    def call():
        oracle.run(w.q_nope, w.q_pe, w.kv_c, w.k_pe, w.slot_mapping, w.cache, w.flags, positions=w.positions,
                   cos_sin=w.cos_sin, q_scale=w.q_scale, kv_scale=w.kv_scale, threads=cores)

    call()
    n, t0 = 0, time.perf_counter()
    while time.perf_counter() - t0 < seconds:
        call()
        n += 1
    dt = time.perf_counter() - t0
    return {"value": round(dt / n * 1e6, 2), "unit": UNIT, "cores": cores, "kind": "oracle, token slices on threads",
            "sample": f"{n} calls of {name} (T={w.T}, H={w.H}) in {dt:.1f} s, {cores} threads of "
                      f"{-(-w.T // cores)} tokens at most; baseline only"}


def run_reference(args, rank, world):
    if rank != 0:
        return None
    w = named_variant(args.workload, 0)
    for _ in range(args.warmup):
        _oracle_call(w)
    t0 = time.perf_counter()
    for _ in range(args.steps):
        _oracle_call(w)
    dt = time.perf_counter() - t0
    us = dt / args.steps * 1e6
    cb = {"value": round(us, 3), "unit": UNIT, "cores": 1, "kind": "oracle",
          "sample": f"{args.steps} calls of {args.workload} (T={w.T}, H={w.H}), one host thread"}
    return {"impl": "reference", "metric": METRIC, "value": round(us, 3), "unit": UNIT, "n_gpus": world,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": round(dt / args.steps * 1e3, 4),
            "higher_is_better": False, "scaling": "weak", "vs_baseline": None, "dtype": "bf16",
            "data": "synthetic",
            "config": {"workload": args.workload, "T": w.T, "H": w.H, "flags": flag_names(w.flags),
                       "recipe": w.recipe, "implementation": "CPU oracle (oracle/mla_oracle.cpp)"},
            "cpu_baseline": cb,
            "e2e": {"value": round(us, 3), "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}


# ---------------------------------------------------------------------------------------

def parse(argv=None):
    p = argparse.ArgumentParser(description=__doc__.splitlines()[0])
    p.add_argument("--gpus", type=int, default=1)
    p.add_argument("--steps", type=int, default=2000)
    p.add_argument("--warmup", type=int, default=20)
    p.add_argument("--impl", choices=("ours", "reference"), default="ours")
    p.add_argument("--workload", default=HEADLINE, choices=W.names())
    p.add_argument("--no-sweep", action="store_true")
    p.add_argument("--no-cpu-baseline", action="store_true")
    a = p.parse_args(argv)
    if a.warmup < 3:
        p.error("--warmup must be at least 3")
    if a.steps < 1:
        p.error("--steps must be positive")
    return a


def main(argv=None):
    args = parse(argv)
    rank, world, local_rank = rank_info()
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
