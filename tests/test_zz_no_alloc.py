"""The entry point for callers that cannot allocate device memory.

Some users of this library run where cudaMalloc is off limits: a serving runtime that
gave all free HBM to its KV-cache pool at start-up, a plugin whose host framework owns
the allocator, code that must not allocate during stream capture.  They cannot hand
qsa_sparse_prefill the workspace that a split selection width needs, so
qsa_sparse_prefill_noalloc takes that scratch from a fixed-size device array inside
libqsa.so.  These tests call it through the C ABI and check it against the workspace
entry point with the parity gates, on two calls in a row (the array is shared and
keeps the previous call's contents).  This file is named to be collected last.
"""
from __future__ import annotations

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from helpers import check_gates, valid_counts
from top_sparse_attention_index_b200 import workloads as wl

pytestmark = pytest.mark.gpu

D = 256


def _case(seed, Tq=16, Hq=16, Hkv=2, S=65536, W=2051):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[torch.rand(Tq, W, generator=g) < 0.1] = -1
    idx[3] = -1                                   # one fully masked row
    width = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32)
    width[5] = 0                                  # one zero-width row
    return q, k, v, idx, width


def _noalloc(q, k, v, idx, width, out, nsplit=0):
    stream = torch.cuda.current_stream(q.device).cuda_stream
    return qsa.qsa_sparse_prefill_noalloc(
        q.data_ptr(), q.stride(0), q.stride(1), k.data_ptr(), k.stride(0), k.stride(1),
        v.data_ptr(), v.stride(0), v.stride(1), idx.data_ptr(), idx.stride(0), width.data_ptr(),
        q.shape[0], q.shape[1], k.shape[1], D, k.shape[0], idx.shape[1], 1.0 / 16.0,
        out.data_ptr(), out.stride(0), out.stride(1), nsplit, None, stream)


@pytest.mark.parametrize("nsplit", [0, 5])
def test_noalloc_matches_workspace_entry_point(cuda_device, nsplit):
    num_sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    for seed in (501, 502):                       # two calls in a row, different inputs
        q, k, v, idx, width = _case(seed)
        n, need = qsa.qsa_sparse_prefill_plan(q.shape[0], q.shape[1], k.shape[1], D,
                                              idx.shape[1], num_sms, nsplit)
        assert n > 1 and 0 < need <= qsa.QSA_STATIC_SCRATCH_BYTES  # the scratch is used
        d = [x.to(cuda_device) for x in (q, k, v, idx, width)]
        ref = qsa.sparse_prefill(*d, scale=1.0 / 16.0, nsplit=nsplit)
        out = torch.full_like(ref, 9.0)
        st = _noalloc(*d, out, nsplit)
        assert st == qsa.QSA_OK, qsa.qsa_last_error_detail()
        torch.cuda.synchronize()
        empty = (valid_counts(idx, width, k.shape[0]) == 0).nonzero().flatten().tolist()
        assert 3 in empty and 5 in empty
        check_gates(out.cpu().float(), ref.cpu().float(), empty, f"noalloc seed {seed}")


def test_noalloc_rejects_shapes_beyond_the_static_scratch(cuda_device):
    Tq, Hq, Hkv, W = 2000, 16, 2, 2051
    n, need = qsa.qsa_sparse_prefill_plan(Tq, Hq, Hkv, D, W, 148, 16)
    assert need > qsa.QSA_STATIC_SCRATCH_BYTES
    q = torch.zeros(Tq, Hq, D, dtype=torch.bfloat16, device=cuda_device)
    kv = torch.zeros(64, Hkv, D, dtype=torch.bfloat16, device=cuda_device)
    idx = torch.zeros(Tq, W, dtype=torch.int32, device=cuda_device)
    width = torch.full((Tq,), W, dtype=torch.int32, device=cuda_device)
    out = torch.full((Tq, Hq, D), 2.0, dtype=torch.bfloat16, device=cuda_device)
    assert _noalloc(q, kv, kv, idx, width, out, nsplit=16) == qsa.QSA_ERR_WORKSPACE
    assert "static scratch" in qsa.qsa_last_error_detail()
    torch.cuda.synchronize()
    assert (out == 2.0).all()                     # nothing was launched
