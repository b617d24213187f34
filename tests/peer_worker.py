"""One rank of the two-process context-parallel test on a single GPU (started with the
spawn method by test_peer_gpu.py; not a test module).

Both ranks run on cuda:0 in separate processes, joined by a gloo process group (host
barriers: no kernel of either rank waits on the other).  Each holds one slot-range shard
of the same seeded cache and calls sparse_prefill_context_parallel with exchange="peer":
the records and outputs are mapped between the two processes with CUDA IPC, and each
rank's combine reads the other rank's records and writes into the other rank's output.
The outputs of two calls in a row (different inputs, the same buffers) are saved for the
parent to check.
"""
from __future__ import annotations

import datetime
import os
import sys
from pathlib import Path

ROOT = Path(__file__).resolve().parent.parent


def case(seed, Tq=300, Hq=16, Hkv=2, S=16384, W=2051):
    import torch
    from top_sparse_attention_index_b200 import workloads as wl
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, 256, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, 256, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, 256, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[torch.rand(Tq, W, generator=g) < 0.05] = -1
    idx[3] = -1                                     # a fully masked row
    width = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32)
    width[4] = 0                                    # a zero-width row
    return q, k, v, idx, width


def main(rank, world, port, out_dir, seeds, record_dtype_name):
    sys.path.insert(0, str(ROOT))
    import torch
    import torch.distributed as dist
    import top_sparse_attention_index_b200 as qsa
    from top_sparse_attention_index_b200 import context_parallel as cp
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("gloo", rank=rank, world_size=world,
                            timeout=datetime.timedelta(seconds=120))
    dev = torch.device("cuda", 0)
    torch.cuda.set_device(dev)
    rec = getattr(torch, record_dtype_name)
    try:
        for seed in seeds:
            q, k, v, idx, width = case(seed)
            S = k.shape[0]
            lo, hi = qsa.shard_ranges(S, world)[rank]
            out = cp.sparse_prefill_context_parallel(
                q.to(dev), k[lo:hi].to(dev), v[lo:hi].to(dev), idx.to(dev), lo, S,
                width=width.to(dev), scale=1.0 / 16.0, exchange="peer", record_dtype=rec)
            torch.cuda.synchronize()
            torch.save(out.cpu(), Path(out_dir) / f"out_{seed}_{rank}.pt")
        cp.release_peer_exchanges()
    finally:
        dist.destroy_process_group()
