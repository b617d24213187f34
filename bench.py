"""Benchmark of the sparse-prefill hot path on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference]

One step = one full pass of the hot path (slot compaction, K/V gather, QK^T, online
softmax, PV, epilogue; plus the LSE combine when the plan splits W) over the long
prefill batch: Hq=16, Hkv=2, D=256, S=65,536 cache slots, Tq=7,810 query rows,
W=2,051 distinct unordered slots per row (the long-prefill case of the article
"Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in CANN prefill PR",
section "Nine tests that passed, ...").  Inputs are synthetic (N(0,1) bf16, uniform
distinct slots) and resident in HBM before the timed region; L2 is flushed between
steps by writing a 512 MiB buffer.  Multi-GPU runs are independent replicas (the path
has no exchange step): every rank processes its own batch and the value is the total
over ranks divided by the slowest rank's time.

Rank 0 prints one JSON line.  ``--impl reference`` times the CPU oracle on a bounded
sample of the same workload instead (rank 0 only).
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import subprocess
import sys
import time
from pathlib import Path

import torch

ROOT = Path(__file__).resolve().parent
sys.path.insert(0, str(ROOT))

from top_sparse_attention_index_b200 import workloads as wl  # noqa: E402
from top_sparse_attention_index_b200.gather_probe import PROBE_CONFIGS, gather_peak  # noqa: E402,F401

METRIC = "sparse prefill TFLOP/s & query-slot pairs/s, 7810q×2051 sel; % of roofline"

# The five configurations (see workloads.py); the benchmark line is long_prefill.
WORKLOADS = {
    "long_prefill": lambda: wl.long_prefill(),
    "long_prefill_block4": lambda: wl.long_prefill_block4(),
    "long_prefill_e4m3kv": lambda: wl.long_prefill_e4m3kv(),
    "tiny": lambda: wl.tiny(),
    "width_sweep": lambda: wl.width_sweep(),
    "causal_two_request": lambda: wl.causal_two_request(),
    "causal_two_request_e4m3kv": lambda: wl.with_e4m3_cache(wl.causal_two_request()),
    "max_extent_g6_uniform": lambda: wl.max_extent(6, False),
    "max_extent_g6_clustered": lambda: wl.max_extent(6, True),
    "max_extent_g3_uniform": lambda: wl.max_extent(3, False),
    "max_extent_g3_clustered": lambda: wl.max_extent(3, True),
}
FALLBACK_HBM_GBS = 6650.0
L2_FLUSH_BYTES = 512 << 20


def parse_args():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=300)
    ap.add_argument("--warmup", type=int, default=5)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--no-e2e", action="store_true")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=12.0,
                    help="target CPU time of the oracle sample")
    ap.add_argument("--rows", type=int, default=0,
                    help="keep only the first ROWS query rows (small cases for ncu captures, "
                         "decode-like batches)")
    ap.add_argument("--workload", default="long_prefill", choices=sorted(WORKLOADS),
                    help="workload to time (the default is the benchmark's)")
    ap.add_argument("--graph", action="store_true",
                    help="time replays of a CUDA graph that holds one step")
    return ap.parse_args()


def pairs_per_row(w: wl.Workload) -> torch.Tensor:
    """Valid (t, slot) pairs of every query row (int64 [Tq]); with block selection every
    valid entry names w.block slots."""
    pos = torch.arange(w.W)[None, :]
    wt = torch.full((w.Tq, 1), w.W) if w.width is None else w.width.to(torch.int64)[:, None]
    ok = (pos < wt) & (w.slot_idx >= 0) & ((w.slot_idx.to(torch.int64) + 1) * w.block <= w.S)
    return ok.sum(dim=1) * w.block


def work_counts(w: wl.Workload):
    """Valid (t, slot) pairs and the algorithmic FLOPs / bytes of one pass."""
    W = w.W
    pairs = int(pairs_per_row(w).sum())
    D = w.q.shape[2]
    flops = pairs * w.Hq * 4 * D                         # 2D (QK^T) + 2D (PV) per head
    kv_bytes = 1 if w.kv_format == "e4m3" else 2
    gathered = pairs * w.Hkv * 2 * D * kv_bytes          # K and V rows (pairs count slots)
    other = w.Tq * w.Hq * D * 2 * 2 + w.Tq * W * 4       # Q in, out, indices
    return pairs, flops, gathered + other, gathered


def reduce_max(x: float, dist=None, device=None) -> float:
    """Max of a per-rank scalar over all ranks (identity without a process group)."""
    if dist is None:
        return float(x)
    t = torch.tensor([float(x)], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def measured_peaks():
    p = ROOT / "MEASURED_PEAKS.json"
    if p.exists():
        d = json.loads(p.read_text())
        return float(d["hbm_gbs"]), "measured"
    return FALLBACK_HBM_GBS, "fallback"


class ClockSampler:
    """nvidia-smi sampling of SM clocks and throttle reasons during the timed region.

    A reader thread collects the samples; entering waits (up to 5 s) until the first
    sample has arrived, so that even a timed region of a few tens of milliseconds falls
    inside the sampled span."""

    FIELDS = ("timestamp,clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.active,"
              "clocks_event_reasons.hw_slowdown,clocks_event_reasons.hw_thermal_slowdown,"
              "clocks_event_reasons.sw_thermal_slowdown,clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        ids = [x.strip() for x in vis.split(",")] if vis else []
        self.gpu_index = ids[gpu_index] if gpu_index < len(ids) else str(gpu_index)
        self.proc = None
        self.lines = []
        self._thread = None

    def _read(self):
        for line in self.proc.stdout:
            if line.strip():
                self.lines.append(line)

    def __enter__(self):
        import threading
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu_index), f"--query-gpu={self.FIELDS}",
                 "--format=csv,noheader,nounits", "-lms", "20"],
                stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
        except OSError:
            self.proc = None
            return self
        self._thread = threading.Thread(target=self._read, daemon=True)
        self._thread.start()
        t_end = time.time() + 5.0
        while not self.lines and time.time() < t_end and self.proc.poll() is None:
            time.sleep(0.01)
        time.sleep(0.05)
        return self

    def __exit__(self, *exc):
        if self.proc is not None:
            time.sleep(0.05)  # a sample after the end of the timed region
            self.proc.terminate()
            try:
                self.proc.wait(timeout=5)
            except subprocess.TimeoutExpired:
                self.proc.kill()
                self.proc.wait()
            if self._thread is not None:
                self._thread.join(timeout=5)

    def summary(self, t0=None, t1=None):
        """Median SM clock and the throttle reasons seen between wall times t0 and t1."""
        import datetime
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for line in getattr(self, "lines", []):
            f = [x.strip() for x in line.split(",")]
            if len(f) < 9:
                continue
            if t0 is not None:
                try:
                    ts = datetime.datetime.strptime(f[0], "%Y/%m/%d %H:%M:%S.%f").timestamp()
                except ValueError:
                    ts = None
                if ts is not None and not (t0 - 0.06 <= ts <= t1 + 0.06):
                    continue
            try:
                sm.append(float(f[1]))
                mx.append(float(f[2]))
            except ValueError:
                continue
            for name, val in zip(names, f[5:9]):
                if val.lower().startswith("active"):
                    reasons.add(name)
        if not sm:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["unsampled"], "samples": 0}
        return {"sm_mhz": statistics.median(sm), "sm_max_mhz": max(mx),
                "reasons": sorted(reasons), "samples": len(sm)}


def cpu_baseline(w: wl.Workload, target_s: float):
    """The oracle as it stands on the host cores, on a bounded sample of query rows."""
    import oracle
    o = oracle.default()
    scale = w.scales[0]
    probe = list(range(min(16, w.Tq)))

    def fwd(rows):
        if w.kv_format == "e4m3":
            o.forward_fp8kv(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, scale, w.k_scale,
                            w.v_scale, rows=rows, block=w.block)
        else:
            o.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, scale, rows=rows,
                      block=w.block)

    t0 = time.perf_counter()
    fwd(probe)
    dt = max(time.perf_counter() - t0, 1e-3)
    n = int(min(w.Tq, max(64, len(probe) * target_s / dt)))
    rows = list(range(n))
    t0 = time.perf_counter()
    fwd(rows)
    dt = time.perf_counter() - t0
    flops = int(pairs_per_row(w)[:n].sum()) * w.Hq * 4 * 256
    return {"value": flops / dt / 1e12, "unit": "TFLOP/s", "cores": o.num_threads(),
            "nproc": os.cpu_count(), "cpu_model": _cpu_model(),
            "kind": "oracle", "seconds": round(dt, 3),
            "sample": f"first {n} of {w.Tq} query rows of the same workload (all heads, all selected slots)"}


def _cpu_model() -> str:
    try:
        for line in open("/proc/cpuinfo"):
            if line.startswith("model name"):
                return line.split(":", 1)[1].strip()
    except OSError:
        pass
    return "unknown"


def run_reference(args, rank):
    """--impl reference: the CPU oracle, timed on the host, rank 0 only."""
    if rank != 0:
        return
    import oracle
    w = wl.long_prefill()
    pairs, flops, _, _ = work_counts(w)
    per_row = flops / w.Tq
    o = oracle.default()
    rows_per_step = 128
    for s in range(args.warmup):
        o.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0,
                  rows=list(range((s * rows_per_step) % w.Tq, (s * rows_per_step) % w.Tq + rows_per_step)))
    times = []
    for s in range(args.steps):
        r0 = ((args.warmup + s) * rows_per_step) % (w.Tq - rows_per_step)
        t0 = time.perf_counter()
        o.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0,
                  rows=list(range(r0, r0 + rows_per_step)))
        times.append(time.perf_counter() - t0)
    sec = sum(times)
    value = per_row * rows_per_step * args.steps / sec / 1e12
    sample = f"{rows_per_step} consecutive query rows per step (of {w.Tq}), all heads and slots"
    print(json.dumps({
        "impl": "reference", "metric": METRIC, "value": value, "unit": "TFLOP/s",
        "n_gpus": args.gpus, "steps": args.steps, "warmup": args.warmup,
        "ms_per_step": 1e3 * sec / args.steps, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "f32", "data": "synthetic",
        "config": {"workload": w.name, "Tq": w.Tq, "Hq": w.Hq, "Hkv": w.Hkv, "D": 256, "S": w.S,
                   "W": w.W, "valid_pairs": pairs, "parallelism": "replicas"},
        "cpu_baseline": {"value": value, "unit": "TFLOP/s", "cores": o.num_threads(),
                         "nproc": os.cpu_count(), "cpu_model": _cpu_model(),
                         "kind": "oracle", "sample": sample},
        "e2e": {"value": value, "unit": "TFLOP/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0},
    }))


def main():
    args = parse_args()
    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local_rank = int(os.environ.get("LOCAL_RANK", "0"))
    if args.impl == "reference":
        run_reference(args, rank)
        return
    assert args.warmup >= 3, "at least 3 warm-up steps"

    import top_sparse_attention_index_b200 as qsa

    device = torch.device("cuda", local_rank)
    torch.cuda.set_device(device)
    dist = None
    if world > 1:
        import datetime

        import torch.distributed as dist
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=device)

    w = WORKLOADS[args.workload]()
    if args.rows:
        w = wl.Workload(f"{w.name}_rows{args.rows}", w.q[:args.rows], w.k_cache, w.v_cache,
                        w.slot_idx[:args.rows], None if w.width is None else w.width[:args.rows],
                        scales=w.scales, block=w.block, kv_format=w.kv_format,
                        k_scale=w.k_scale, v_scale=w.v_scale)
    pairs, flops, alg_bytes, gathered = work_counts(w)
    q, k, v, idx = (x.to(device) for x in (w.q, w.k_cache, w.v_cache, w.slot_idx))
    width = None if w.width is None else w.width.to(device)
    scale = w.scales[0]
    out = torch.empty(w.Tq, w.Hq, 256, dtype=torch.bfloat16, device=device)
    num_sms = torch.cuda.get_device_properties(device).multi_processor_count
    nsplit, ws_bytes = qsa.qsa_sparse_prefill_block_plan(w.Tq, w.Hq, w.Hkv, 256, w.W, w.block,
                                                         num_sms)
    launches_per_step = 1 if nsplit == 1 else 2
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)
    stream = torch.cuda.current_stream(device)

    def step():
        qsa.sparse_prefill(q, k, v, idx, width, scale=scale, out=out, block=w.block,
                           k_scale=w.k_scale, v_scale=w.v_scale)

    for _ in range(args.warmup):
        flush.zero_()
        step()
    torch.cuda.synchronize()
    if args.graph:
        graph = torch.cuda.CUDAGraph()
        with torch.cuda.graph(graph):
            step()
        step = graph.replay
        for _ in range(args.warmup):
            flush.zero_()
            step()
        torch.cuda.synchronize()

    starts = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    ends = [torch.cuda.Event(enable_timing=True) for _ in range(args.steps)]
    if dist is not None:
        dist.barrier()
    torch.cuda.synchronize()
    with ClockSampler(local_rank) as clocks:
        t0_epoch = time.time()
        t_wall = time.perf_counter()
        for i in range(args.steps):
            flush.zero_()
            starts[i].record(stream)
            step()
            ends[i].record(stream)
        torch.cuda.synchronize()
        t_wall = time.perf_counter() - t_wall
        t1_epoch = time.time()
    if dist is not None:
        dist.barrier()
    kernel_ms = [s.elapsed_time(e) for s, e in zip(starts, ends)]
    total_ms = reduce_max(sum(kernel_ms), dist, device)   # the slowest rank's device time
    ms_per_step = total_ms / args.steps

    # warm-cache figure, outside the timed region: the same launch repeated with no L2
    # flush in between, median over the launches (the slowest rank's median)
    n_warm = min(args.steps, 50)
    w_starts = [torch.cuda.Event(enable_timing=True) for _ in range(n_warm)]
    w_ends = [torch.cuda.Event(enable_timing=True) for _ in range(n_warm)]
    for i in range(n_warm):
        w_starts[i].record(stream)
        step()
        w_ends[i].record(stream)
    torch.cuda.synchronize()
    warm_ms = reduce_max(statistics.median(s.elapsed_time(e) for s, e in zip(w_starts, w_ends)),
                         dist, device)

    # end to end through the public host-buffer API: pinned host inputs -> device ->
    # kernels -> pinned host output, transfers overlapped with the kernels by row chunks
    e2e = None
    if not args.no_e2e:
        hq, hk, hv, hidx = (x.pin_memory() for x in (w.q, w.k_cache, w.v_cache, w.slot_idx))
        hout = torch.empty(out.shape, dtype=out.dtype).pin_memory()
        h2d = sum(x.numel() * x.element_size() for x in (hq, hk, hv, hidx))
        d2h = hout.numel() * hout.element_size()

        def e2e_step():
            _, fin = qsa.sparse_prefill_from_host(hq, hk, hv, hidx, w.width, scale=scale,
                                                  out=hout, device=device, block=w.block,
                                                  k_scale=w.k_scale, v_scale=w.v_scale)
            return fin

        for _ in range(3):
            e2e_step().synchronize()
        e_steps = max(3, min(args.steps, 10))
        if dist is not None:
            dist.barrier()
        torch.cuda.synchronize()
        t0 = time.perf_counter()
        for _ in range(e_steps):
            e2e_step().synchronize()   # the result is on the host when the step ends
        e_ms = reduce_max((time.perf_counter() - t0) * 1e3 / e_steps, dist, device)
        e2e = {"value": world * flops / (e_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
               "ms_per_step": e_ms, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h}

    # the SM-side roofline, measured right after the timed region on the same device
    probe = gather_peak(device, 256 if w.kv_format == "e4m3" else 512)  # (gather_probe.py)

    if dist is not None:
        dist.destroy_process_group()
    if rank != 0:
        return

    hbm_peak, peak_kind = measured_peaks()
    t_s = ms_per_step * 1e-3
    achieved = alg_bytes / t_s / 1e9
    traffic, ncu_rec = None, None
    prof = ROOT / "profiles" / "traffic.json"
    if prof.exists():
        # one record per workload; a record counts only while the kernel sources it was
        # captured with are unchanged
        for rec in json.loads(prof.read_text()).get("records", []):
            if rec.get("kernel_source_hash") == _kernel_hash() and rec.get("workload_name") == w.name:
                traffic, ncu_rec = rec.get("bytes_per_launch"), rec
    result = {
        "metric": METRIC,
        "value": world * flops / t_s / 1e12,
        "unit": "TFLOP/s",
        "n_gpus": world,
        "steps": args.steps,
        "warmup": args.warmup,
        "ms_per_step": ms_per_step,
        "higher_is_better": True,
        "scaling": "weak",
        "vs_baseline": None,
        # the MMA input type (bf16 caches: bf16; E4M3 caches: f16 from the 8-bit codes)
        "dtype": "f16 (e4m3 kv)" if w.kv_format == "e4m3" else "bf16",
        "data": "synthetic",
        "config": {"workload": w.name, "Tq": w.Tq, "Hq": w.Hq, "Hkv": w.Hkv, "D": 256, "S": w.S,
                   "W": w.W, "valid_pairs": pairs, "nsplit": nsplit,
                   "l2": "flushed between steps (512 MiB write)", "parallelism": f"replicas x{world}",
                   "launch": "cuda graph replay" if args.graph else "eager"},
        "pairs_per_s": world * pairs / t_s,
        "pairs_x_hkv_per_s": world * pairs * w.Hkv / t_s,
        "gathered_gb_per_s": gathered / t_s / 1e9,
        # the two bounds of a gather whose rows are partly L2 hits: the L2 -> shared-memory
        # gather of all algorithmic bytes against the gather probe's best rate (measured
        # live on this device), and the DRAM bytes the launch moves (ncu, one full-size
        # launch of the current kernel code) against the measured copy bandwidth; the
        # roofline is the one whose time bound is larger (the other stays beside it)
        **_rooflines(achieved, alg_bytes, t_s, probe, traffic, ncu_rec, hbm_peak, peak_kind),
        "gather_probe": probe,
        "warm_l2": {"ms_per_step_median": warm_ms, "launches": n_warm,
                    "value": world * flops / (warm_ms * 1e-3) / 1e12, "unit": "TFLOP/s",
                    "note": "no L2 flush between launches; not the timed region"},
        "gpu_launches": args.steps * launches_per_step,
        "clocks": clocks.summary(t0_epoch, t1_epoch),
        "wall_s_timed_region": t_wall,
    }
    if e2e is not None:
        result["e2e"] = e2e
    if not args.no_cpu_baseline:
        result["cpu_baseline"] = cpu_baseline(w, args.cpu_seconds)
    print(json.dumps(result))


def _rooflines(achieved, alg_bytes, t_s, probe, traffic, ncu_rec, hbm_peak, peak_kind):
    """{"roofline": the binding bound, "hbm": the DRAM bound, "l2_gather": the gather
    bound}.  The gather bound's time is alg_bytes / probe peak; the DRAM bound's is the
    measured DRAM traffic / copy bandwidth (only when a traffic record of the current
    kernel exists; otherwise the gather bound is reported as the roofline)."""
    l2_peak = probe["tb_per_s"] * 1e3
    gather = {"bound": "l2", "achieved": achieved, "peak": l2_peak, "unit": "GB/s",
              "frac": achieved / l2_peak, "traffic": traffic,
              "algorithmic_bytes_per_launch": alg_bytes,
              "peak_source": "measured live: gather probe (qsa_probe_gather), best of "
                             f"{len(probe['runs'])} pipeline shapes: {probe['best']}",
              "ncu_l2_throughput_pct": (ncu_rec or {}).get(
                  "lts__throughput.avg.pct_of_peak_sustained_elapsed")}
    hbm = {"bound": "hbm", "achieved": traffic / t_s / 1e9 if traffic else None,
           "peak": hbm_peak, "unit": "GB/s",
           "frac": traffic / t_s / 1e9 / hbm_peak if traffic else None, "traffic": traffic,
           "peak_source": f"{peak_kind} hbm_gbs (achieved: ncu DRAM bytes of one launch)"}
    binding = gather
    if traffic and traffic / (hbm_peak * 1e9) > alg_bytes / (l2_peak * 1e9):
        binding = hbm
    return {"roofline": binding, "hbm": hbm, "l2_gather": gather}


def _code_only(text: str) -> str:
    """C++ source with comments removed and whitespace collapsed (string and character
    literals kept), so that editing a comment does not change the kernel's hash."""
    import re
    token = re.compile(r'//[^\n]*|/\*.*?\*/|"(?:\\.|[^"\\])*"|\'(?:\\.|[^\'\\])*\'', re.S)
    text = token.sub(lambda m: " " if m.group(0).startswith("/") else m.group(0), text)
    return " ".join(text.split())


def _kernel_hash():
    """Hash of the kernel code, comments and whitespace aside (the DRAM traffic record
    is valid while it matches)."""
    import hashlib
    h = hashlib.sha256()
    csrc = ROOT / "top_sparse_attention_index_b200" / "csrc"
    for name in ("qsa_attn.cu", "qsa_internal.h", "qsa_ptx.cuh"):
        h.update(_code_only((csrc / name).read_text()).encode())
    return h.hexdigest()[:16]


if __name__ == "__main__":
    main()
