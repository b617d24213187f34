"""The entry point for callers that cannot allocate device memory.

Some users of this library run where cudaMalloc is off limits: a serving runtime that
gave all free HBM to its KV-cache pool at start-up, a plugin whose host framework owns
the allocator, code that must not allocate during stream capture.  They cannot hand
qsa_sparse_prefill the workspace that a split selection width needs, so
qsa_sparse_prefill_noalloc takes that scratch from a fixed-size device array inside
libqsa.so.  These tests call it through the C ABI, on several calls in a row whose
shapes and split counts differ (the array is shared and keeps the previous call's
contents, so a later call's log-sum-exp region lands on an earlier call's partial
outputs), and check every call against the CPU oracle with the parity gates and
bitwise against the workspace entry point with the same split plan.  Each test builds
its own inputs, so the file passes alone in a fresh process as well as after the
other tests; it is named so that pytest collects it last.
"""
from __future__ import annotations

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from helpers import check_gates, valid_counts
from top_sparse_attention_index_b200 import workloads as wl

pytestmark = pytest.mark.gpu

D = 256
HQ, HKV, S, W = 16, 2, 65536, 2051


def _case(seed, Tq, nsplit):
    """Random inputs with a fully masked row, a zero-width row and a row whose first
    split (of `nsplit` equal splits of W) holds only -1 entries."""
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, HQ, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, HKV, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, HKV, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[torch.rand(Tq, W, generator=g) < 0.1] = -1
    width = torch.randint(W // 2, W + 1, (Tq,), generator=g, dtype=torch.int32)
    idx[3] = -1                                   # fully masked row
    width[5] = 0                                  # zero-width row
    split_len = -(-W // nsplit)
    idx[7, :split_len] = -1                       # row 7: the first split is empty
    width[7] = W
    return q, k, v, idx, width


def _noalloc(d, out, nsplit):
    q, k, v, idx, width = d
    stream = torch.cuda.current_stream(q.device).cuda_stream
    return qsa.qsa_sparse_prefill_noalloc(
        q.data_ptr(), q.stride(0), q.stride(1), k.data_ptr(), k.stride(0), k.stride(1),
        v.data_ptr(), v.stride(0), v.stride(1), idx.data_ptr(), idx.stride(0), width.data_ptr(),
        q.shape[0], q.shape[1], k.shape[1], D, k.shape[0], idx.shape[1], 1.0 / 16.0,
        out.data_ptr(), out.stride(0), out.stride(1), nsplit, None, stream)


def test_noalloc_calls_in_a_row_match_oracle_and_workspace_entry_point(cuda_device, oracle_lib):
    num_sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    # (seed, Tq, nsplit): the split counts and row counts differ from call to call; the
    # last call repeats the first on the scratch the others have left behind
    calls = [(501, 16, 5), (502, 9, 3), (503, 16, 0), (501, 16, 5)]
    first = None
    for seed, Tq, nsplit in calls:
        q, k, v, idx, width = _case(seed, Tq, nsplit if nsplit else 9)
        n, need = qsa.qsa_sparse_prefill_plan(Tq, HQ, HKV, D, W, num_sms, nsplit)
        assert n > 1 and 0 < need <= qsa.QSA_STATIC_SCRATCH_BYTES  # the scratch is used
        d = [x.to(cuda_device) for x in (q, k, v, idx, width)]
        out = torch.full((Tq, HQ, D), 9.0, dtype=torch.bfloat16, device=cuda_device)
        st = _noalloc(d, out, nsplit)
        assert st == qsa.QSA_OK, qsa.qsa_last_error_detail()
        ref_ws = qsa.sparse_prefill(*d, scale=1.0 / 16.0, nsplit=n)
        torch.cuda.synchronize()
        got = out.cpu()
        label = f"noalloc seed {seed} Tq {Tq} nsplit {n}"
        # bitwise the workspace entry point with the same split plan
        assert torch.equal(got, ref_ws.cpu()), label
        # and within the parity gates of the oracle, empty rows exactly zero
        empty = (valid_counts(idx, width, S) == 0).nonzero().flatten().tolist()
        assert 3 in empty and 5 in empty and 7 not in empty
        ref = oracle_lib.forward(q, k, v, idx, width, 1.0 / 16.0)
        check_gates(got.float(), torch.from_numpy(ref), empty, label)
        assert (got[3] == 0).all() and (got[5] == 0).all()
        if first is None:
            first = got
        elif (seed, Tq, nsplit) == calls[0]:
            assert torch.equal(got, first), "a repeated call depends on what the scratch held"


def test_noalloc_rejects_shapes_beyond_the_static_scratch(cuda_device):
    Tq = 2000
    n, need = qsa.qsa_sparse_prefill_plan(Tq, HQ, HKV, D, W, 148, 16)
    assert need > qsa.QSA_STATIC_SCRATCH_BYTES
    q = torch.zeros(Tq, HQ, D, dtype=torch.bfloat16, device=cuda_device)
    kv = torch.zeros(64, HKV, D, dtype=torch.bfloat16, device=cuda_device)
    idx = torch.zeros(Tq, W, dtype=torch.int32, device=cuda_device)
    width = torch.full((Tq,), W, dtype=torch.int32, device=cuda_device)
    out = torch.full((Tq, HQ, D), 2.0, dtype=torch.bfloat16, device=cuda_device)
    assert _noalloc((q, kv, kv, idx, width), out, 16) == qsa.QSA_ERR_WORKSPACE
    assert "static scratch" in qsa.qsa_last_error_detail()
    torch.cuda.synchronize()
    assert (out == 2.0).all()                     # nothing was launched
