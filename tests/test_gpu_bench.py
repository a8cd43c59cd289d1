"""bench.py end to end on the GPU: a short run prints one JSON line with the
keys of the benchmark contract and sane values."""

import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_bench_prints_one_contract_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--steps", "20", "--warmup", "3",
                        "--no-sweep", "--no-cpu-baseline"], capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip()]
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "roofline", "e2e", "gpu_launches", "clocks"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 20 and d["warmup"] == 3 and d["higher_is_better"] is False
    assert d["config"]["workload"] == "batch_t8192_h16_pdl_fp8"
    # the reference arm prints the same config apart from its implementation
    ref = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                          "--warmup", "3"], capture_output=True, text=True, timeout=900)
    assert ref.returncode == 0, ref.stderr[-2000:]
    rc = json.loads(ref.stdout.strip().splitlines()[-1])["config"]
    assert {k: v for k, v in rc.items() if k != "implementation"} == \
        {k: v for k, v in d["config"].items() if k != "implementation"}
    assert 10.0 < d["value"] < 500.0
    rf = d["roofline"]
    assert rf["bound"] == "hbm" and rf["unit"] == "GB/s" and 0 < rf["frac"] < 1.5
    assert abs(rf["achieved"] / rf["peak"] - rf["frac"]) < 1e-3
    assert len(d["timing"]["region_us_per_call_sorted"]) == d["timing"]["regions"] >= 10
    e = d["e2e"]
    assert e["value"] > d["value"] and e["h2d_bytes_per_step"] > 0 and e["d2h_bytes_per_step"] > 0
    assert d["gpu_launches"] == 20
    assert d["launch_floor_us"] > 0
    bp = d["behind_producer"]
    assert bp["producer_us"] > 0 and bp["epilogue_increment_pdl_us"] > 0


def test_decode_floor_readings_behind_both_producers(monkeypatch):
    """bench's decode readings at T=1, short: standalone, behind the plain
    producer and behind the producer that streams weights first."""
    import torch
    sys.path.insert(0, ROOT)
    import bench as B
    from mla_decode_attention_10_b200 import epilogue as E
    monkeypatch.setattr(B, "DECODE_T", (1,))
    dev = torch.device("cuda", 0)
    hx = B.Harness(E, torch.cuda.Stream(dev))
    (row,) = B.decode_floors(hx, dev, 6650.0, calls=20, reps=2)
    assert row["T"] == 1 and row["mode"] == "split"
    assert row["gemm_producer_us"] > row["producer_us"] > 0
    for p in ("", "gemm_"):
        assert row[p + "epilogue_increment_pdl_us"] > 0 and row[p + "empty_wait_increment_us"] > -1.0
        assert row[p + "increment_over_launch_floor"] > 0
