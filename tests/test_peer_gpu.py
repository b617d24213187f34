"""The context-parallel combine over records addressed one pointer each
(qsa_combine_peer_records, include/qsa_peer.h) and the peer exchange built on it.

Ranks are emulated on one GPU in two ways: (1) one process holding every shard's record
in its own buffer, the combine given one pointer per record (what a rank does with the
other ranks' records mapped into it); (2) two processes on the same GPU, joined by a gloo
group, exchanging their record and output buffers with CUDA IPC (host barriers between
the steps; no kernel waits on the other process).  Both are compared with the CPU oracle
at the parity gates and bitwise with the all-gather path (the same arithmetic in the same
order)."""
from __future__ import annotations

import socket
import sys
import tempfile
from pathlib import Path

import pytest
import torch
import torch.multiprocessing as mp

import top_sparse_attention_index_b200 as qsa
from helpers import check_gates, valid_counts
from top_sparse_attention_index_b200 import _binding, workloads as wl

pytestmark = pytest.mark.gpu

ROOT = Path(__file__).resolve().parent.parent
D = 256


def _case(seed, Tq, Hq, Hkv, S, W, minus1=0.05):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[torch.rand(Tq, W, generator=g) < minus1] = -1
    idx[3] = -1
    width = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32)
    width[4] = 0
    return q, k, v, idx, width


def _records(d, S, R, rec):
    """Every shard's record in buffers of its own (one device standing in for R ranks)."""
    q, k, v, idx, width = d
    outs = []
    for lo, hi in qsa.shard_ranges(S, R):
        outs.append(qsa.sparse_prefill_partial(q, k[lo:hi], v[lo:hi], idx, lo, S, width=width,
                                               scale=1.0 / 16.0, record_dtype=rec))
    return [o for o, _ in outs], [l for _, l in outs]


def _empty(idx, width, S):
    return (valid_counts(idx, width, S) == 0).nonzero().flatten().tolist()


@pytest.mark.parametrize("rec", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("R", [1, 2, 5, 16])
def test_peer_combine_equals_stacked_combine_and_oracle(cuda_device, oracle_lib, R, rec):
    q, k, v, idx, width = _case(300 + R, 300, 16, 2, 16384, 2051)
    d = [t.to(cuda_device) for t in (q, k, v, idx, width)]
    rec_o, rec_l = _records(d, 16384, R, rec)
    stacked = qsa.combine_partials(torch.stack(rec_o), torch.stack(rec_l))
    out = torch.full((300, 16, D), float("nan"), dtype=torch.bfloat16, device=cuda_device)
    _binding.combine_peer_records([o.data_ptr() for o in rec_o], [l.data_ptr() for l in rec_l],
                                  rec, 300, 16, [out])
    torch.cuda.synchronize()
    assert torch.equal(out.view(torch.int16), stacked.view(torch.int16))
    ref = oracle_lib.forward(q, k, v, idx, width, 1.0 / 16.0)
    check_gates(out.cpu().float(), torch.from_numpy(ref), _empty(idx, width, 16384),
                f"peer combine R={R} {rec}")


def test_peer_combine_row_range_and_several_outputs(cuda_device):
    """Rows [t0, t1) go to every output (one of them a strided view); rows outside the
    range are left untouched; an empty range writes nothing."""
    q, k, v, idx, width = _case(320, 257, 12, 1, 4096, 700)
    d = [t.to(cuda_device) for t in (q, k, v, idx, width)]
    rec_o, rec_l = _records(d, 4096, 3, torch.bfloat16)
    stacked = qsa.combine_partials(torch.stack(rec_o), torch.stack(rec_l))
    def filled(*shape):  # a NaN bit pattern no combine produces
        t = torch.empty(*shape, dtype=torch.bfloat16, device=cuda_device)
        t.view(torch.int16).fill_(0x7fc1)
        return t
    a, wide, c = filled(257, 12, D), filled(257, 2, 12, D), filled(257, 12, D)
    b = wide[:, 1]
    ptrs_o, ptrs_l = [o.data_ptr() for o in rec_o], [l.data_ptr() for l in rec_l]
    _binding.combine_peer_records(ptrs_o, ptrs_l, torch.bfloat16, 257, 12, [a, c], t0=37, t1=211)
    _binding.combine_peer_records(ptrs_o, ptrs_l, torch.bfloat16, 257, 12, [b], t0=5, t1=250)
    _binding.combine_peer_records(ptrs_o, ptrs_l, torch.bfloat16, 257, 12, [b], t0=100, t1=100)
    torch.cuda.synchronize()
    s16 = stacked.view(torch.int16)
    for o, (t0, t1) in ((a, (37, 211)), (c, (37, 211)), (b, (5, 250))):
        o16 = o.view(torch.int16)
        assert torch.equal(o16[t0:t1], s16[t0:t1])
        assert (o16[:t0] == 0x7fc1).all() and (o16[t1:] == 0x7fc1).all()
    assert (wide[:, 0].view(torch.int16) == 0x7fc1).all()


def test_peer_combine_rejects_bad_arguments(cuda_device):
    o = torch.zeros(4, 2, D, dtype=torch.float32, device=cuda_device)
    l = torch.zeros(4, 2, dtype=torch.float32, device=cuda_device)
    out = torch.zeros(4, 2, D, dtype=torch.bfloat16, device=cuda_device)
    st = torch.cuda.current_stream().cuda_stream
    call = _binding.qsa_combine_peer_records
    good = dict(rec_o=[o.data_ptr()], rec_lse=[l.data_ptr()], R=1, record_bf16=0, Tq=4, Hq=2,
                D=D, t0=0, t1=4, out=[out.data_ptr()], n_out=1, out_stride_t=2 * D,
                out_stride_h=D, stream=st)
    assert call(**good) == qsa.QSA_OK
    for change, status in ((dict(R=0), qsa.QSA_ERR_INVALID_ARG),
                           (dict(R=17, rec_o=[o.data_ptr()] * 17, rec_lse=[l.data_ptr()] * 17),
                            qsa.QSA_ERR_INVALID_ARG),
                           (dict(record_bf16=2), qsa.QSA_ERR_INVALID_ARG),
                           (dict(t0=3, t1=2), qsa.QSA_ERR_INVALID_ARG),
                           (dict(t1=5), qsa.QSA_ERR_INVALID_ARG),
                           (dict(D=128), qsa.QSA_ERR_UNSUPPORTED),
                           (dict(out_stride_h=4), qsa.QSA_ERR_INVALID_ARG),
                           (dict(rec_o=[o.data_ptr() + 4]), qsa.QSA_ERR_INVALID_ARG),
                           (dict(rec_lse=[0]), qsa.QSA_ERR_INVALID_ARG),
                           (dict(out=[out.data_ptr() + 2]), qsa.QSA_ERR_INVALID_ARG),
                           (dict(n_out=0, out=[]), qsa.QSA_ERR_INVALID_ARG)):
        assert call(**{**good, **change}) == status, change
    torch.cuda.synchronize()


def test_ipc_export_names_the_allocation_and_offset(cuda_device):
    """Two views of one tensor share the exported handle and differ by their byte offset;
    importing a handle of this same process is refused (a status, not a fault)."""
    base = torch.empty(1 << 20, dtype=torch.uint8, device=cuda_device)
    h0, off0 = _binding.ipc_export(base)
    h1, off1 = _binding.ipc_export(base[4096:])
    assert h0 == h1 and off1 - off0 == 4096
    with pytest.raises(qsa.QSAError):
        _binding.ipc_import(h0, cuda_device)


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


@pytest.mark.parametrize("rec", ["bfloat16", "float32"])
def test_two_processes_exchange_records_over_ipc(cuda_device, oracle_lib, rec):
    sys.path.insert(0, str(Path(__file__).resolve().parent))
    import peer_worker
    seeds = (401, 402)
    ctx = mp.get_context("spawn")
    with tempfile.TemporaryDirectory() as tmp:
        port = _free_port()
        procs = [ctx.Process(target=peer_worker.main, args=(r, 2, port, tmp, seeds, rec))
                 for r in range(2)]
        for p in procs:
            p.start()
        for p in procs:
            p.join(timeout=300)
        for p in procs:
            if p.is_alive():
                p.kill()
                p.join()
        assert [p.exitcode for p in procs] == [0, 0]
        for seed in seeds:
            outs = [torch.load(Path(tmp) / f"out_{seed}_{r}.pt") for r in range(2)]
            q, k, v, idx, width = peer_worker.case(seed)
            d = [t.to(cuda_device) for t in (q, k, v, idx, width)]
            rec_o, rec_l = _records(d, k.shape[0], 2, getattr(torch, rec))
            stacked = qsa.combine_partials(torch.stack(rec_o), torch.stack(rec_l)).cpu()
            for out in outs:
                assert torch.equal(out.view(torch.int16), stacked.view(torch.int16))
            ref = oracle_lib.forward(q, k, v, idx, width, 1.0 / 16.0)
            check_gates(outs[0].float(), torch.from_numpy(ref), _empty(idx, width, k.shape[0]),
                        f"two processes over IPC, {rec}, seed {seed}")
