"""The benchmark's multi-rank logic on CPU: two gloo ranks (replicas only, no
collective on the data path) agree on the max of their timings, and the
reference arm runs on rank 0 alone."""

import json
import os
import subprocess
import sys

import torch.multiprocessing as mp

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _worker(rank, world, port, out):
    import torch
    import torch.distributed as dist
    sys.path.insert(0, ROOT)
    import bench
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port))
    dist.init_process_group("gloo", rank=rank, world_size=world)
    try:
        dev = torch.device("cpu")
        local_ms = [3.0, 7.5][rank]
        bench.barrier(dev)
        got = bench.max_over_ranks(local_ms, dev)
        us = bench.job_us_per_call(got, steps=100, world=world)
        out[rank] = (got, us)
    finally:
        dist.destroy_process_group()


def test_max_over_ranks_and_job_rate_with_two_gloo_ranks():
    import socket
    s = socket.socket()
    s.bind(("127.0.0.1", 0))
    port = s.getsockname()[1]
    s.close()
    mgr = mp.Manager()
    out = mgr.dict()
    mp.spawn(_worker, args=(2, port, out), nprocs=2, join=True)
    assert out[0] == out[1]
    got, us = out[0]
    assert got == 7.5
    # two ranks x 100 calls in 7.5 ms: 37.5 us per call for the job
    assert abs(us - 7.5e3 / 200) < 1e-9


def test_reference_arm_prints_on_rank_zero_only():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2", LOCAL_RANK="1")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "1", "--warmup", "3", "--workload", "decode_t4_h16"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0 and r.stdout.strip() == ""
    env = dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0")
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", "2", "--warmup", "3", "--workload", "decode_t4_h16"],
                       capture_output=True, text=True, env=env, timeout=300)
    assert r.returncode == 0
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference" and line["unit"] == "µs/call" and line["higher_is_better"] is False
    assert line["cpu_baseline"]["kind"] == "oracle" and line["e2e"]["h2d_bytes_per_step"] == 0
    assert line["config"]["workload"] == "decode_t4_h16"


def test_bench_rejects_short_warmup():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--warmup", "2"],
                       capture_output=True, text=True, timeout=120)
    assert r.returncode != 0 and "warmup" in r.stderr


def test_reference_arm_samples_token_slices_of_the_workload():
    """With a small time budget the reference arm runs the oracle on a token
    slice of the workload and scales its time to a full call; the slice is
    the workload's first tokens with the same cache, table and scales."""
    sys.path.insert(0, ROOT)
    import bench
    from mla_decode_attention_10_b200 import workloads as W
    w = W.named("decode_sweep_t64_h16_rope_fp8")
    s = bench.token_slice(w, 5)
    assert s.T == 5 and s.H == w.H and s.q_nope.shape[0] == 5 and s.slot_mapping.shape[0] == 5
    assert s.positions.shape[0] == 5 and s.cache is w.cache and s.cos_sin is w.cos_sin
    assert bench.token_slice(w, 64) is w
    args = bench.parse(["--impl", "reference", "--steps", "2", "--warmup", "3",
                        "--workload", "decode_sweep_t64_h16_rope_fp8"])
    line = bench.run_reference(args, 0, 1, budget_s=1e-6)   # forces the smallest slice
    assert line["impl"] == "reference" and line["value"] > 0
    assert "of the 64 tokens" in line["cpu_baseline"]["sample"] and "scaled by 64/" in line["cpu_baseline"]["sample"]
    assert line["config"] == dict(bench.common_config("decode_sweep_t64_h16_rope_fp8"),
                                  implementation=line["config"]["implementation"])
