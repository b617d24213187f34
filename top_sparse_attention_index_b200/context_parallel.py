"""Context parallelism: the K/V cache split by slot range across the ranks of a process
group (decode context parallelism, named for this attention path in the article
"Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in CANN prefill PR", section
"Where this sits in the Qwen4Exp serving build-out").

Every rank holds a contiguous slot range of the cache and sees the same global selection.
Each rank computes its partial record in the CUDA kernels (qsa_sparse_prefill_partial:
the output normalised over its own slots, bf16 by default, and the fp32 base-2
log-sum-exp of their scores); the records are exchanged with one all-gather
(torch.distributed, NCCL on GPUs) and combined in the CUDA combine kernel
(qsa_combine_partials), which gives the attention over the whole cache.  bf16 records
halve the bytes every rank sends (512 instead of 1,024 per (query row, head)).
This module only shards, exchanges and marshals: the arithmetic is in the kernels.
"""
from __future__ import annotations

import torch

from . import _binding


def shard_ranges(S_total: int, world: int, block: int = 1):
    """Contiguous slot ranges [lo, hi) of a cache of S_total slots over `world` ranks, each
    non-empty range starting at a multiple of `block` (a block never straddles two ranks);
    earlier ranks take the remainder, so sizes differ by at most one block, and ranks past
    the last block get empty ranges at S_total."""
    if world < 1 or block < 1 or S_total < 0:
        raise ValueError("world and block must be positive, S_total non-negative")
    nblocks = -(-S_total // block)
    base, extra = divmod(nblocks, world)
    out, lo = [], 0
    for r in range(world):
        n = base + (1 if r < extra else 0)
        hi = min(S_total, lo + n * block)
        out.append((lo, hi))
        lo = hi
    return out


def exchange_records(part_o: torch.Tensor, part_lse: torch.Tensor, group=None):
    """All-gather of the ranks' records: ([R, Tq, Hq, D], [R, Tq, Hq]) in rank order, the
    layout combine_partials reads."""
    import torch.distributed as dist
    R = dist.get_world_size(group)
    # concatenated along the first dimension (the form every backend accepts), which is
    # the stacked [R, ...] layout in memory
    g_o = torch.empty((R * part_o.shape[0], *part_o.shape[1:]), dtype=part_o.dtype,
                      device=part_o.device)
    g_l = torch.empty((R * part_lse.shape[0], *part_lse.shape[1:]), dtype=part_lse.dtype,
                      device=part_lse.device)
    dist.all_gather_into_tensor(g_o, part_o.contiguous(), group=group)
    dist.all_gather_into_tensor(g_l, part_lse.contiguous(), group=group)
    return g_o.view(R, *part_o.shape), g_l.view(R, *part_lse.shape)


def sparse_prefill_context_parallel(q, k_local, v_local, slot_idx, slot_lo, S_total,
                                    group=None, width=None, scale=None, block=1, k_scale=1.0,
                                    v_scale=1.0, out=None, partial_fn=None, combine_fn=None,
                                    record_dtype=torch.bfloat16):
    """Selected-slot sparse attention over a cache split by slot range across the ranks of
    `group`: this rank's k_local / v_local hold global slots [slot_lo, slot_lo + S_local)
    (see shard_ranges); q, slot_idx (global slot numbers) and width are the same on every
    rank.  Returns the bf16 output [Tq, Hq, 256] on every rank.  record_dtype (bfloat16 or
    float32) is the type of the exchanged normalised outputs.

    partial_fn / combine_fn default to the CUDA entry points (sparse_prefill_partial,
    combine_partials); they are parameters so that the exchange can be exercised on hosts
    without a GPU.
    """
    partial_fn = partial_fn or _binding.sparse_prefill_partial
    combine_fn = combine_fn or _binding.combine_partials
    part_o, part_lse = partial_fn(q, k_local, v_local, slot_idx, slot_lo, S_total, width=width,
                                  scale=scale, block=block, k_scale=k_scale, v_scale=v_scale,
                                  record_dtype=record_dtype)
    g_o, g_l = exchange_records(part_o, part_lse, group)
    return combine_fn(g_o, g_l, out=out)
