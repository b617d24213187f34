"""bench.py end to end on the GPU at a small size: the one JSON line it prints carries the
fields the benchmark contract asks for, with values that hang together (the time-based
figures agree with each other, the roofline objects come from the live gather probe and
the measured copy bandwidth, the launch count matches the plan, the clocks were sampled)."""
from __future__ import annotations

import json
import subprocess
import sys
from pathlib import Path

import pytest

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parent.parent


def _bench(*args):
    out = subprocess.run([sys.executable, str(ROOT / "bench.py"), *args], cwd=ROOT,
                         capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    lines = [l for l in out.stdout.splitlines() if l.startswith("{")]
    assert len(lines) == 1, out.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_small_case(cuda_device):
    d = _bench("--rows", "256", "--steps", "5", "--warmup", "3", "--cpu-seconds", "1")
    for key in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
                "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
                "roofline", "hbm", "l2_gather", "cpu_baseline", "e2e", "gpu_launches", "clocks"):
        assert key in d, key
    assert d["n_gpus"] == 1 and d["steps"] == 5 and d["warmup"] == 3
    assert d["unit"] == "TFLOP/s" and d["higher_is_better"] is True and d["scaling"] == "weak"
    assert d["config"]["workload"].startswith("long_prefill") and d["config"]["Tq"] == 256
    assert d["value"] > 0 and d["ms_per_step"] > 0
    # TFLOP/s and query-slot pairs/s are the same time seen two ways
    flops_per_pair = d["config"]["Hq"] * 4 * 256
    assert abs(d["pairs_per_s"] * flops_per_pair / 1e12 - d["value"]) < 1e-6 * d["value"]
    rf = d["roofline"]
    assert rf["bound"] in ("l2", "hbm") and rf["unit"] == "GB/s"
    assert abs(rf["frac"] - rf["achieved"] / rf["peak"]) < 1e-9
    assert d["l2_gather"]["peak"] == d["gather_probe"]["tb_per_s"] * 1e3
    assert d["gpu_launches"] == d["steps"] * (1 if d["config"]["nsplit"] == 1 else 2)
    assert d["e2e"]["h2d_bytes_per_step"] > 0 and d["e2e"]["d2h_bytes_per_step"] > 0
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["cores"] >= 1
    assert d["clocks"]["samples"] >= 0


def test_reference_arm_line(cuda_device):
    d = _bench("--impl", "reference", "--steps", "1", "--warmup", "1")
    assert d["impl"] == "reference" and d["unit"] == "TFLOP/s"
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["cpu_baseline"]["kind"] == "oracle"


def test_context_parallel_bench_line(cuda_device):
    """The context-parallel measurement (ranks emulated on one GPU) at a decode shape:
    one JSON line whose per-R entries carry the shard, combine and link-byte figures."""
    out = subprocess.run([sys.executable, "-m", "top_sparse_attention_index_b200.context_parallel_bench",
                          "--rows", "64", "--ranks", "2,3", "--reps", "3"], cwd=ROOT,
                         capture_output=True, text=True, timeout=900)
    assert out.returncode == 0, out.stderr[-2000:]
    d = json.loads([l for l in out.stdout.splitlines() if l.startswith("{")][-1])
    assert d["unit"] == "us" and d["unsharded_us"] > 0
    assert [(e["R"], e["record"]) for e in d["ranks"]] == [(2, "bfloat16"), (3, "bfloat16"),
                                                           (2, "float32"), (3, "float32")]
    for e in d["ranks"]:
        assert len(e["shard_us"]) == e["R"] and e["shard_max_us"] == max(e["shard_us"])
        assert e["all_gather_bytes_in_per_rank"] == (e["R"] - 1) * e["record_bytes_per_rank"]
        assert e["peer_bytes_in_per_rank"] < e["all_gather_bytes_in_per_rank"]
