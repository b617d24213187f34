"""Context parallelism measured with the ranks emulated on one GPU.

    python -m top_sparse_attention_index_b200.context_parallel_bench [--rows N] [--ranks 2,4,8]

For a cache split by slot range over R ranks (context_parallel.py), times on this device,
one after another: the unsharded call; every shard's partial record (the slowest is what
a rank of R would wait for); the combine of the R records stacked as an all-gather leaves
them (qsa_combine_partials); the combine reading each record through its own pointer, all
query rows (qsa_combine_peer_records, what a rank does with the other ranks' records
mapped into it); and one rank's share of the rows stored to R outputs (the peer exchange's
combine).  The records are local here, so the NVLink transfers the exchanges need on
several GPUs are not in these times: the line gives their bytes per rank and the time
they take at a link rate given on the command line (770 GB/s per direction measured for
one peer copy on this machine's B200 nodes), by construction, not measured.

Inputs: the long-prefill workload (or its first --rows query rows: a decode-shape batch),
resident in HBM; L2 flushed before every launch (512 MiB write); CUDA events around each
launch, median of --reps.  Prints one JSON line.
"""
from __future__ import annotations

import argparse
import json

import torch

from . import _binding
from . import workloads as wl
from .context_parallel import shard_ranges

L2_FLUSH_BYTES = 512 << 20


def _timer(device, reps):
    flush = torch.empty(L2_FLUSH_BYTES, dtype=torch.uint8, device=device)

    def timeit(fn):
        for _ in range(3):
            flush.zero_()
            fn()
        torch.cuda.synchronize(device)
        evs = []
        for _ in range(reps):
            flush.zero_()
            a, b = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
            a.record()
            fn()
            b.record()
            evs.append((a, b))
        torch.cuda.synchronize(device)
        return sorted(x.elapsed_time(y) for x, y in evs)[reps // 2] * 1e3  # us
    return timeit


def measure(rows=0, ranks=(2, 4, 8), reps=20, link_gbs=770.0, device=None):
    device = torch.device(device or "cuda")
    w = wl.long_prefill()
    if rows:
        w = wl.Workload(f"{w.name}_rows{rows}", w.q[:rows], w.k_cache, w.v_cache,
                        w.slot_idx[:rows], None)
    q, k, v, idx = (x.to(device) for x in (w.q, w.k_cache, w.v_cache, w.slot_idx))
    Tq, Hq = q.shape[0], q.shape[1]
    timeit = _timer(device, reps)
    result = {"metric": "context parallel, ranks emulated one after another on one GPU",
              "workload": w.name, "unit": "us", "reps": reps, "link_gbs_per_direction": link_gbs,
              "unsharded_us": timeit(lambda: _binding.sparse_prefill(q, k, v, idx)),
              "ranks": []}
    out_bytes = Tq * Hq * 256 * 2
    for rec in (torch.bfloat16, torch.float32):
        for R in ranks:
            shards = shard_ranges(w.S, R)
            recs = [_binding.sparse_prefill_partial(q, k[lo:hi], v[lo:hi], idx, lo, w.S,
                                                    record_dtype=rec) for lo, hi in shards]
            shard_us = [timeit(lambda lo=lo, hi=hi: _binding.sparse_prefill_partial(
                q, k[lo:hi], v[lo:hi], idx, lo, w.S, record_dtype=rec)) for lo, hi in shards]
            g_o = torch.stack([r[0] for r in recs])
            g_l = torch.stack([r[1] for r in recs])
            o_ptrs = [r[0].data_ptr() for r in recs]
            l_ptrs = [r[1].data_ptr() for r in recs]
            out = torch.empty(Tq, Hq, 256, dtype=torch.bfloat16, device=device)
            outs = [torch.empty_like(out) for _ in range(R)]
            t0, t1 = shard_ranges(Tq, R)[0]
            stacked_us = timeit(lambda: _binding.combine_partials(g_o, g_l, out=out))
            peer_all_us = timeit(lambda: _binding.combine_peer_records(
                o_ptrs, l_ptrs, rec, Tq, Hq, [out]))
            peer_share_us = timeit(lambda: _binding.combine_peer_records(
                o_ptrs, l_ptrs, rec, Tq, Hq, outs, t0=t0, t1=t1))
            record_bytes = g_o[0].numel() * g_o.element_size() + g_l[0].numel() * 4
            share = (t1 - t0) / max(Tq, 1)
            ag_in = (R - 1) * record_bytes                       # all-gather: into each rank
            peer_in = (R - 1) * share * record_bytes             # peer: its rows' records
            peer_out = (R - 1) * share * out_bytes               # peer: its rows to the others
            result["ranks"].append({
                "R": R, "record": str(rec).replace("torch.", ""),
                "shard_max_us": max(shard_us), "shard_us": shard_us,
                "combine_stacked_us": stacked_us, "combine_peer_all_rows_us": peer_all_us,
                "combine_peer_row_share_to_R_outputs_us": peer_share_us,
                "record_bytes_per_rank": record_bytes,
                "all_gather_bytes_in_per_rank": ag_in,
                "peer_bytes_in_per_rank": peer_in, "peer_bytes_out_per_rank": peer_out,
                "all_gather_link_us_by_construction": ag_in / (link_gbs * 1e3),
                "peer_link_us_by_construction": max(peer_in, peer_out) / (link_gbs * 1e3),
            })
    return result


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--rows", type=int, default=0, help="first ROWS query rows only (decode shape)")
    ap.add_argument("--ranks", default="2,4,8")
    ap.add_argument("--reps", type=int, default=20)
    ap.add_argument("--link-gbs", type=float, default=770.0,
                    help="NVLink rate per direction used for the by-construction times")
    a = ap.parse_args()
    if not torch.cuda.is_available():
        raise SystemExit("context_parallel_bench needs a CUDA device")
    r = measure(a.rows, tuple(int(x) for x in a.ranks.split(",")), a.reps, a.link_gbs)
    print(json.dumps(r))


if __name__ == "__main__":
    main()
