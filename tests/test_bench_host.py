"""Host-side pieces of bench.py: the work bookkeeping and the multi-rank reduction
(world size 2 over gloo on the CPU; on GPUs the same code runs over NCCL)."""
from __future__ import annotations

import datetime
import os
import socket
import sys
from pathlib import Path

import pytest
import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent
sys.path.insert(0, str(ROOT))

import bench  # noqa: E402
from top_sparse_attention_index_b200 import workloads as wl  # noqa: E402


def test_work_counts_tiny():
    w = wl.tiny()
    pairs, flops, alg_bytes, gathered = bench.work_counts(w)
    assert pairs == 124 * 64                       # four of 128 rows are fully masked
    assert flops == pairs * 16 * 4 * 256           # 2D (QK^T) + 2D (PV) per query head
    assert gathered == pairs * 2 * 2 * 256 * 2     # K and V rows of both KV heads, bf16
    assert alg_bytes == gathered + 128 * 16 * 256 * 2 * 2 + 128 * 64 * 4


def test_work_counts_width_sweep():
    w = wl.width_sweep()
    pairs, *_ = bench.work_counts(w)
    ref = sum(int(((w.slot_idx[t, : int(w.width[t])] >= 0)).sum()) for t in range(w.Tq))
    assert pairs == ref


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _rank_main(rank, world, port, queue):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    local = 10.0 + 5.0 * rank                      # rank 1 is the slow one
    queue.put((rank, bench.reduce_max(local, dist, torch.device("cpu"))))
    dist.barrier()
    dist.destroy_process_group()


def test_max_over_ranks_gloo():
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, 2, port, queue)) for r in range(2)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=120) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    assert results == {0: 15.0, 1: 15.0}


def test_reduce_without_process_group():
    assert bench.reduce_max(3.5) == 3.5


def test_reference_arm_runs_on_rank0_only(capsys):
    class A:
        gpus, steps, warmup = 2, 1, 0
    assert bench.run_reference(A(), rank=1) is None
    assert capsys.readouterr().out == ""


def test_kernel_hash_ignores_comments_and_whitespace():
    """The traffic record's key: comments and layout do not change it, code does, and
    string or character literals that look like comments are kept."""
    a = 'int f() { return 1; } // one\n/* block\n comment */ const char* s = "// x";'
    b = 'int  f()  {\n  return 1;  }\nconst char* s = "// x"; // other comment'
    c = 'int f() { return 2; } const char* s = "// x";'
    d = 'int f() { return 1; } const char* s = "// y";'
    assert bench._code_only(a) == bench._code_only(b)
    assert bench._code_only(a) != bench._code_only(c)
    assert bench._code_only(a) != bench._code_only(d)
    assert bench._code_only("char q = '/'; // c") == "char q = '/';"
    assert len(bench._kernel_hash()) == 16


def test_gather_probe_shapes_fit_one_sm():
    """Every pipeline shape the benchmark's gather probe runs fits the shared memory of one
    SM at its CTAs per SM (228 KiB, 1 KiB reserved per CTA) and the probe's limits."""
    for row_bytes, shapes in bench.PROBE_CONFIGS.items():
        assert row_bytes in (256, 512)
        for warps, stages, per_sm in shapes:
            assert 1 <= warps <= 15 and 2 <= stages <= 4 and per_sm >= 1
            smem = warps * stages * 16 * row_bytes + 2 * warps * stages * 8
            assert smem <= 227 * 1024
            assert per_sm * (smem + 1024) <= 228 * 1024

def test_binding_roofline_is_the_slower_bound():
    """The long prefill's rows are L2 hits: the gather bound (algorithmic bytes against the
    gather probe) binds.  A cache twice the size of L2 moves most rows from DRAM: the
    DRAM bound (measured traffic against the copy bandwidth) binds.  Without a traffic
    record of the current kernel only the gather bound is known."""
    probe = {"tb_per_s": 18.0, "runs": [{}] * 8, "best": {}}
    lp = bench._rooflines(33e9 / 2.02e-3 / 1e9, 33e9, 2.02e-3, probe, 1.76e9, None, 6548.8, "m")
    assert lp["roofline"]["bound"] == "l2" and lp["roofline"] is lp["l2_gather"]
    assert abs(lp["roofline"]["frac"] - (33e9 / 2.02e-3) / 18e12) < 1e-9
    assert abs(lp["hbm"]["frac"] - 1.76e9 / 2.02e-3 / 6548.8e9) < 1e-9
    mx = bench._rooflines(8.65e9 / 0.922e-3 / 1e9, 8.65e9, 0.922e-3, probe, 5.9e9, None,
                          6548.8, "m")
    assert mx["roofline"]["bound"] == "hbm" and mx["roofline"] is mx["hbm"]
    assert abs(mx["roofline"]["frac"] - 5.9e9 / 0.922e-3 / 6548.8e9) < 1e-9
    none = bench._rooflines(1.0, 8.65e9, 0.922e-3, probe, None, None, 6548.8, "m")
    assert none["roofline"]["bound"] == "l2" and none["hbm"]["frac"] is None
