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

exchange="peer" (the ranks of one node) fuses the exchange into the combine instead: each
rank's record and output buffers are mapped into every other rank with CUDA IPC, and
each rank's combine kernel (qsa_combine_peer_records) reads the records of its own share
of the query rows from all ranks where they lie (peer loads over NVLink / NVSwitch) and
stores the combined rows to every rank's output.  No gathered copy of the records exists,
and the all-gather of the outputs is the combine's own stores.  A collective on the
compute stream before and after the combine orders it with every rank's other kernels.
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


class PeerExchange:
    """Record (O, lse) and output buffers of this rank for one (Tq, Hq, record type), with
    the same buffers of every rank of `group` mapped here (CUDA IPC; the ranks share one
    node).  Creating one is collective: every rank of the group creates it in the same
    call.  o_ptrs / lse_ptrs / out_ptrs: one device pointer per rank, in rank order (this
    rank's own pointer at its own position).  `ipc` supplies ipc_export / ipc_import /
    ipc_close (the library's by default)."""

    def __init__(self, group, device, Tq, Hq, record_dtype, ipc=None):
        import torch.distributed as dist
        self.group, self.device = group, torch.device(device)
        self.rank, self.world = dist.get_rank(group), dist.get_world_size(group)
        if self.world > _binding.QSA_MAX_PEERS:
            raise ValueError("the peer exchange serves at most %d ranks (got %d): use "
                             'exchange="all_gather"' % (_binding.QSA_MAX_PEERS, self.world))
        self.Tq, self.Hq, self.record_dtype = Tq, Hq, record_dtype
        self._ipc = ipc or _binding
        dev = self.device
        self.part_o = torch.empty(Tq, Hq, 256, dtype=record_dtype, device=dev)
        self.part_lse = torch.empty(Tq, Hq, dtype=torch.float32, device=dev)
        self.out = torch.empty(Tq, Hq, 256, dtype=torch.bfloat16, device=dev)
        self.flag = torch.zeros(1, dtype=torch.float32, device=dev)
        local = (self.part_o, self.part_lse, self.out)
        mine = [self._ipc.ipc_export(t) for t in local]
        table = [None] * self.world
        dist.all_gather_object(table, mine, group=group)
        # one mapping per exported allocation: a rank's buffers may share one
        self._bases = {}
        ptrs = []
        for r, entries in enumerate(table):
            row = []
            for (handle, off), t in zip(entries, local):
                if r == self.rank:
                    row.append(t.data_ptr())
                    continue
                key = (r, handle)
                if key not in self._bases:
                    self._bases[key] = self._ipc.ipc_import(handle, dev)
                row.append(self._bases[key] + off)
            ptrs.append(row)
        self.o_ptrs = [p[0] for p in ptrs]
        self.lse_ptrs = [p[1] for p in ptrs]
        self.out_ptrs = [p[2] for p in ptrs]

    def close(self):
        """Unmaps the other ranks' buffers (collective: a barrier first, so no rank still
        uses a mapping or a buffer, and one after, so no buffer is freed while mapped)."""
        barrier(self.group, self)
        for base in self._bases.values():
            self._ipc.ipc_close(base, self.device)
        self._bases = {}
        barrier(self.group, self)


def barrier(group, ex):
    """Orders the ranks' device work: on return (NCCL: on the compute stream) every rank's
    work issued before it is complete.  NCCL: a one-element all-reduce on the current
    stream (each rank's stream reaches it only after its own earlier kernels; nothing waits
    on the host).  Other backends: the current stream synchronised, then a process-group
    barrier."""
    import torch.distributed as dist
    if dist.get_backend(group) == "nccl":
        dist.all_reduce(ex.flag, group=group)
    else:
        if ex.device.type == "cuda":
            torch.cuda.current_stream(ex.device).synchronize()
        dist.barrier(group=group)


_EXCHANGES = {}


def peer_exchange(group, device, Tq, Hq, record_dtype, ipc=None):
    """The PeerExchange of this shape, created on first use (collectively) and kept until
    release_peer_exchanges(), which every rank must call before the group is destroyed."""
    import torch.distributed as dist
    key = (id(group) if group is not None else None, dist.get_rank(group),
           torch.device(device), Tq, Hq, record_dtype)
    if key not in _EXCHANGES:
        _EXCHANGES[key] = PeerExchange(group, device, Tq, Hq, record_dtype, ipc=ipc)
    return _EXCHANGES[key]


def release_peer_exchanges():
    """Closes every kept PeerExchange (collective over each one's group, in creation
    order, so every rank must call it)."""
    for key in list(_EXCHANGES):
        _EXCHANGES.pop(key).close()


def sparse_prefill_context_parallel(q, k_local, v_local, slot_idx, slot_lo, S_total,
                                    group=None, width=None, scale=None, block=1, k_scale=1.0,
                                    v_scale=1.0, out=None, partial_fn=None, combine_fn=None,
                                    record_dtype=torch.bfloat16, exchange="all_gather",
                                    peer_combine_fn=None, ipc=None):
    """Selected-slot sparse attention over a cache split by slot range across the ranks of
    `group`: this rank's k_local / v_local hold global slots [slot_lo, slot_lo + S_local)
    (see shard_ranges); q, slot_idx (global slot numbers) and width are the same on every
    rank.  Returns the bf16 output [Tq, Hq, 256] on every rank.  record_dtype (bfloat16 or
    float32) is the type of the exchanged normalised outputs.

    exchange: "all_gather" (records gathered by the process group, then combined; any
    backend, any number of nodes) or "peer" (one node: the records read in place by the
    combine over CUDA IPC mappings, each rank combining its own share of the query rows
    (shard_ranges over Tq) and storing it to every rank's output; see PeerExchange).

    partial_fn / combine_fn / peer_combine_fn default to the CUDA entry points
    (sparse_prefill_partial, combine_partials, combine_peer_records) and ipc to the
    library's IPC helpers; they are parameters so that the exchange can be exercised on
    hosts without a GPU.
    """
    partial_fn = partial_fn or _binding.sparse_prefill_partial
    if exchange == "all_gather":
        combine_fn = combine_fn or _binding.combine_partials
        part_o, part_lse = partial_fn(q, k_local, v_local, slot_idx, slot_lo, S_total,
                                      width=width, scale=scale, block=block, k_scale=k_scale,
                                      v_scale=v_scale, record_dtype=record_dtype)
        g_o, g_l = exchange_records(part_o, part_lse, group)
        return combine_fn(g_o, g_l, out=out)
    if exchange != "peer":
        raise ValueError('exchange must be "all_gather" or "peer"')
    peer_combine_fn = peer_combine_fn or _binding.combine_peer_records
    Tq, Hq = q.shape[0], q.shape[1]
    ex = peer_exchange(group, q.device, Tq, Hq, record_dtype, ipc=ipc)
    partial_fn(q, k_local, v_local, slot_idx, slot_lo, S_total, width=width, scale=scale,
               block=block, k_scale=k_scale, v_scale=v_scale, record_dtype=record_dtype,
               part_o=ex.part_o, part_lse=ex.part_lse)
    barrier(group, ex)  # every rank's record is complete
    t0, t1 = shard_ranges(Tq, ex.world)[ex.rank]
    peer_combine_fn(ex.o_ptrs, ex.lse_ptrs, record_dtype, Tq, Hq,
                    [(p, ex.out.stride(0), ex.out.stride(1)) for p in ex.out_ptrs],
                    t0=t0, t1=t1, device=q.device)
    barrier(group, ex)  # every rank's rows are in every output; the records are free again
    if out is None:
        return ex.out.clone()
    out.copy_(ex.out)
    return out
