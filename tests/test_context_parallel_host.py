"""Host side of context parallelism (the cache split by slot range across ranks): the
shard ranges and the exchange of the ranks' partial records, run as world-size-2 and 3
gloo process groups on the CPU.  The kernels are replaced by exact float64 restatements
of what the entry points document (the record: output normalised over the rank's valid
slots and the base-2 log-sum-exp of their scaled scores; the combine: log-sum-exp
weights), so the test checks the sharding and the exchange order; the result must equal
the CPU oracle on the whole cache.  The CUDA records and combine are checked on the GPU
in test_parity_gpu.py."""
from __future__ import annotations

import datetime
import math
import os
import socket
import sys
from pathlib import Path

import numpy as np
import torch
import torch.multiprocessing as mp

ROOT = Path(__file__).resolve().parent.parent
sys.path.insert(0, str(ROOT))

from top_sparse_attention_index_b200 import context_parallel as cp  # noqa: E402
from top_sparse_attention_index_b200 import workloads as wl  # noqa: E402

D = 256


def _case():
    g = torch.Generator().manual_seed(91)
    Tq, Hq, Hkv, S, W = 6, 8, 2, 120, 40
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[1, :] = -1                         # a fully masked row
    idx[2, 5:] = idx[2, 5:].clamp(max=20)  # row 2 mostly in the first shard
    return q, k, v, idx


def _partial_double(q, k_local, v_local, slot_idx, slot_lo, S_total, width=None, scale=None,
                    block=1, k_scale=1.0, v_scale=1.0, record_dtype=torch.float32):
    """float64 restatement of qsa_sparse_prefill_partial's documented record (the
    normalised output rounded to record_dtype, the log-sum-exp in fp32)."""
    scale = 1.0 / 16.0 if scale is None else scale
    Tq, Hq, _ = q.shape
    S_loc, Hkv, _ = k_local.shape
    G = Hq // Hkv
    o = np.zeros((Tq, Hq, D), dtype=np.float32)
    lse = np.full((Tq, Hq), -np.inf, dtype=np.float32)
    qd, kd, vd = q.double().numpy(), k_local.double().numpy(), v_local.double().numpy()
    for t in range(Tq):
        sel = [int(s) - slot_lo for s in slot_idx[t] if slot_lo <= int(s) < slot_lo + S_loc]
        if not sel:
            continue
        for h in range(Hq):
            x = scale * math.log2(math.e) * (kd[sel, h // G] @ qd[t, h])
            m = x.max()
            p = np.exp2(x - m)
            o[t, h] = (p @ vd[sel, h // G]) / p.sum()
            lse[t, h] = m + math.log2(p.sum())
    return torch.from_numpy(o).to(record_dtype), torch.from_numpy(lse)


def _combine_double(g_o, g_l, out=None):
    o, l = g_o.double().numpy(), g_l.double().numpy()
    m = l.max(axis=0)
    w = np.where(np.isfinite(l), np.exp2(l - np.where(np.isfinite(m), m, 0)), 0.0)
    num = (w[..., None] * np.nan_to_num(o)).sum(axis=0)
    den = w.sum(axis=0)
    return torch.from_numpy(np.where(den[..., None] > 0, num / np.maximum(den, 1e-300)[..., None], 0.0))


def _rank_main(rank, world, port, queue, record_dtype):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    q, k, v, idx = _case()
    S = k.shape[0]
    lo, hi = cp.shard_ranges(S, world)[rank]
    out = cp.sparse_prefill_context_parallel(q, k[lo:hi], v[lo:hi], idx, lo, S,
                                             partial_fn=_partial_double,
                                             combine_fn=_combine_double,
                                             record_dtype=record_dtype)
    queue.put((rank, out.numpy()))
    dist.barrier()
    dist.destroy_process_group()


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _run(world, record_dtype=torch.float32):
    ctx = mp.get_context("spawn")
    queue = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_rank_main, args=(r, world, port, queue, record_dtype))
             for r in range(world)]
    for p in procs:
        p.start()
    results = dict(queue.get(timeout=180) for _ in procs)
    for p in procs:
        p.join(timeout=60)
        assert p.exitcode == 0
    return results


def test_context_parallel_exchange_matches_the_whole_cache(oracle_lib):
    q, k, v, idx = _case()
    ref = oracle_lib.forward(q, k, v, idx, None, 1.0 / 16.0)
    for world in (2, 3):
        results = _run(world)
        for r in range(world):
            np.testing.assert_allclose(results[r], ref, rtol=1e-5, atol=1e-6)
        assert np.all(results[0][1] == 0)   # the fully masked row


def test_context_parallel_bf16_records(oracle_lib):
    """bf16 records: every record's normalised output is rounded to bf16 (relative error at
    most 2^-9) and the combine is a convex combination of the records, so the result is
    within 2^-9 of the largest |V| element of the row's selected rows of the whole-cache
    oracle (here bounded by the largest |V| of the cache)."""
    q, k, v, idx = _case()
    ref = oracle_lib.forward(q, k, v, idx, None, 1.0 / 16.0)
    bound = 2.0 ** -9 * float(v.float().abs().max()) + 1e-6
    for world in (2, 3):
        results = _run(world, torch.bfloat16)
        for r in range(world):
            assert np.abs(results[r] - ref).max() <= bound
            np.testing.assert_array_equal(results[r], results[0])
        assert np.all(results[0][1] == 0)


def test_shard_ranges_cover_the_cache_once():
    for S, world, block in ((65536, 8, 1), (1000, 3, 4), (7, 2, 1), (10, 4, 4)):
        r = cp.shard_ranges(S, world, block)
        assert len(r) == world and r[0][0] == 0 and r[-1][1] == S
        assert all(a[1] == b[0] for a, b in zip(r, r[1:]))
        assert all(hi >= lo and (lo % block == 0 or hi == lo) for lo, hi in r)


# ---- the peer exchange (records read in place, outputs stored to every rank) -------------

class _FakeIPC:
    """Stands in for the CUDA IPC helpers on the CPU: a handle names (rank, buffer number)
    and an import returns a synthetic base address for it (never dereferenced)."""

    def __init__(self, rank):
        self.rank, self.n, self.opened, self.closed = rank, 0, [], []

    def ipc_export(self, t):
        self.n += 1
        return bytes([self.rank, self.n]) + bytes(62), 16 * self.n

    def ipc_import(self, handle, device):
        base = ((1 + handle[0]) << 40) | (handle[1] << 32)
        self.opened.append(base)
        return base

    def ipc_close(self, base, device):
        self.closed.append(base)


def _peer_combine_emulated(o_ptrs, lse_ptrs, record_dtype, Tq, Hq, outs, t0, t1, device=None):
    """The peer combine restated on the CPU: the pointer table is checked against the
    exchange's buffers; reading the other ranks' records in place is emulated by a gather,
    and storing the rows [t0, t1) to every rank's output by a gather of the row blocks."""
    import torch.distributed as dist
    ex = next(iter(cp._EXCHANGES.values()))
    for r in range(ex.world):
        own = r == ex.rank
        base = ((1 + r) << 40)
        assert o_ptrs[r] == (ex.part_o.data_ptr() if own else (base | 1 << 32) + 16)
        assert lse_ptrs[r] == (ex.part_lse.data_ptr() if own else (base | 2 << 32) + 32)
        assert outs[r][0] == (ex.out.data_ptr() if own else (base | 3 << 32) + 48)
    assert (t0, t1) == tuple(cp.shard_ranges(Tq, ex.world)[ex.rank])
    g_o = [torch.empty_like(ex.part_o) for _ in range(ex.world)]
    g_l = [torch.empty_like(ex.part_lse) for _ in range(ex.world)]
    dist.all_gather(g_o, ex.part_o)
    dist.all_gather(g_l, ex.part_lse)
    rows = _combine_double(torch.stack(g_o)[:, t0:t1], torch.stack(g_l)[:, t0:t1])
    blocks = [None] * ex.world
    dist.all_gather_object(blocks, (t0, t1, rows.to(torch.bfloat16)))
    for a, b, blk in blocks:
        ex.out[a:b] = blk


def _partial_into(q, k_local, v_local, slot_idx, slot_lo, S_total, part_o=None, part_lse=None,
                  **kw):
    o, lse = _partial_double(q, k_local, v_local, slot_idx, slot_lo, S_total, **kw)
    part_o.copy_(o)
    part_lse.copy_(lse)
    return part_o, part_lse


def _peer_rank_main(rank, world, port, queue):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=60))
    q, k, v, idx = _case()
    S = k.shape[0]
    lo, hi = cp.shard_ranges(S, world)[rank]
    ipc = _FakeIPC(rank)
    outs = []
    for _ in range(2):  # the second call reuses the exchange (no new export or import)
        outs.append(cp.sparse_prefill_context_parallel(
            q, k[lo:hi], v[lo:hi], idx, lo, S, exchange="peer", partial_fn=_partial_into,
            peer_combine_fn=_peer_combine_emulated, ipc=ipc, record_dtype=torch.bfloat16))
    opened = list(ipc.opened)
    cp.release_peer_exchanges()
    queue.put((rank, [o.float().numpy() for o in outs], opened, list(ipc.closed), ipc.n))
    dist.barrier()
    dist.destroy_process_group()


def test_peer_exchange_protocol(oracle_lib):
    """World sizes 2 and 3: every rank exports its three buffers once, maps the other ranks'
    (one mapping per exported allocation), combines its own share of the rows, and ends
    with the whole output; both calls give the whole-cache result (bf16 records and bf16
    output: within 2^-8 of the largest |V|), the same on every rank; release unmaps exactly
    what was mapped."""
    q, k, v, idx = _case()
    ref = oracle_lib.forward(q, k, v, idx, None, 1.0 / 16.0)
    bound = 2.0 ** -8 * float(v.float().abs().max()) + 1e-6
    for world in (2, 3):
        ctx = mp.get_context("spawn")
        queue = ctx.Queue()
        port = _free_port()
        procs = [ctx.Process(target=_peer_rank_main, args=(r, world, port, queue))
                 for r in range(world)]
        for p in procs:
            p.start()
        results = {}
        for _ in procs:
            rank, outs, opened, closed, exported = queue.get(timeout=180)
            results[rank] = outs
            assert exported == 3
            assert len(opened) == 3 * (world - 1) and sorted(closed) == sorted(opened)
        for p in procs:
            p.join(timeout=60)
            assert p.exitcode == 0
        for r in range(world):
            for out in results[r]:
                assert np.abs(out - ref).max() <= bound
                np.testing.assert_array_equal(out, results[0][0])
            assert np.all(results[r][0][1] == 0)   # the fully masked row


# ---- a rank that fails: the others end with an error instead of waiting for good -------

def _failing_rank_main(rank, world, port, queue, exchange):
    import torch.distributed as dist
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=5))
    if rank == world - 1:
        queue.put((rank, "left"))          # this rank leaves before the exchange
        return
    q, k, v, idx = _case()
    S = k.shape[0]
    lo, hi = cp.shard_ranges(S, world)[rank]
    try:
        kw = dict(partial_fn=_partial_into, peer_combine_fn=_peer_combine_emulated,
                  ipc=_FakeIPC(rank)) if exchange == "peer" else \
             dict(partial_fn=_partial_double, combine_fn=_combine_double)
        cp.sparse_prefill_context_parallel(q, k[lo:hi], v[lo:hi], idx, lo, S, exchange=exchange,
                                           record_dtype=torch.float32, **kw)
        queue.put((rank, "no error"))
    except Exception as e:  # noqa: BLE001 - the collective's error is what the test wants
        queue.put((rank, "error: " + type(e).__name__))


def test_a_rank_that_leaves_ends_the_exchange_with_an_error():
    """World size 3 with a 5-second process-group timeout; the last rank leaves before the
    exchange (host-side failure, no device involved).  The remaining ranks' exchange (the
    all-gather, or the peer exchange's handle exchange and barriers) ends with an error
    within the timeout instead of waiting for good."""
    import time
    for exchange in ("all_gather", "peer"):
        ctx = mp.get_context("spawn")
        queue = ctx.Queue()
        port = _free_port()
        procs = [ctx.Process(target=_failing_rank_main, args=(r, 3, port, queue, exchange))
                 for r in range(3)]
        t0 = time.time()
        for p in procs:
            p.start()
        results = dict(queue.get(timeout=120) for _ in procs)
        for p in procs:
            p.join(timeout=60)
            if p.is_alive():
                p.kill()
                p.join()
        assert results[2] == "left"
        for r in (0, 1):
            assert results[r].startswith("error"), (exchange, results)
        assert time.time() - t0 < 110
