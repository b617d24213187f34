"""Host-side tests of the C ABI (no GPU needed): the library loads, exports every
symbol include/qsa.h declares, the planner's choices, and argument validation that
returns before any CUDA call."""
from __future__ import annotations

import ctypes
import re
import subprocess
from pathlib import Path

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from top_sparse_attention_index_b200 import _binding, build_lib

INCLUDE = Path(__file__).resolve().parent.parent / "include"


def declared_functions():
    names = set()
    for header in sorted(INCLUDE.glob("*.h")):
        text = re.sub(r"/\*.*?\*/", "", header.read_text(), flags=re.S)
        names |= set(re.findall(r"^\s*(?:const\s+)?[\w\s\*]+?\b(qsa_\w+)\s*\(", text, flags=re.M))
    return sorted(names)


@pytest.fixture(scope="module")
def lib():
    build_lib.build()
    return _binding.load_library()


def test_header_declares_the_boundary():
    assert declared_functions() == sorted(_binding.SIGNATURES)


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.run(["nm", "-D", "--defined-only", str(_binding.LIBRARY)],
                         capture_output=True, text=True, check=True).stdout
    exported = set(re.findall(r"\bT (qsa_\w+)", out))
    for name in declared_functions():
        assert name in exported, name
        assert getattr(lib, name) is not None


def test_library_is_built_for_sm100a():
    text = build_lib.NVCC_FLAGS
    assert "arch=compute_100a,code=sm_100a" in text


def test_status_strings(lib):
    assert qsa.qsa_abi_version() == 2
    for code, name in [(0, "QSA_OK"), (1, "QSA_ERR_INVALID_ARG"), (2, "QSA_ERR_UNSUPPORTED"),
                       (3, "QSA_ERR_WORKSPACE"), (4, "QSA_ERR_CUDA")]:
        assert qsa.qsa_status_string(code) == name


@pytest.mark.parametrize("Tq,Hq,Hkv,W,expect", [
    (7810, 16, 2, 2051, 1),       # long prefill: enough units, one split
    (128, 16, 2, 64, 1),          # tiny: a 64-wide row is never split
    (16384, 24, 2, 2051, 1),      # causal two-request
    (4096, 6, 1, 2048, 1),        # max extent
])
def test_plan_without_split(lib, Tq, Hq, Hkv, W, expect):
    n, ws = qsa.qsa_sparse_prefill_plan(Tq, Hq, Hkv, 256, W, 148)
    assert n == expect and ws == 0


def test_plan_splits_small_batches(lib):
    # 16 rows x 2 KV heads = 32 units; one wave = 148 SMs x 2 resident CTAs = 296:
    # floor(296 / 32) = 9 splits fill it
    n, ws = qsa.qsa_sparse_prefill_plan(16, 16, 2, 256, 2051, 148)
    assert n == 9
    assert ws >= n * 16 * 16 * 256 * 4 + n * 16 * 16 * 4
    # one wave or more of units: no split
    assert qsa.qsa_sparse_prefill_plan(160, 16, 2, 256, 2051, 148)[0] == 1
    assert qsa.qsa_sparse_prefill_plan(300, 12, 1, 256, 2051, 148)[0] == 1
    n1, _ = qsa.qsa_sparse_prefill_plan(1, 16, 2, 256, 2051, 148)
    assert n1 == 16  # floor(2051 / 128): splits are never narrower than 128 positions
    assert -(-2051 // n1) >= 128


def test_block_plan(lib):
    # 2,048 blocks of 4 = 8,192 slots per row: ceil(8192 / 2240) = 4 splits
    n, ws = qsa.qsa_sparse_prefill_block_plan(7810, 16, 2, 256, 2048, 4, 148)
    assert n == 4 and ws > 0
    assert qsa.qsa_sparse_prefill_block_plan(7810, 16, 2, 256, 2051, 1, 148) == \
        qsa.qsa_sparse_prefill_plan(7810, 16, 2, 256, 2051, 148)
    for bad in (0, 17, -4):
        with pytest.raises(qsa.QSAError) as ei:
            qsa.qsa_sparse_prefill_block_plan(10, 16, 2, 256, 8, bad, 148)
        assert ei.value.status == qsa.QSA_ERR_INVALID_ARG


def test_plan_wide_rows_force_splits(lib):
    n, _ = qsa.qsa_sparse_prefill_plan(100000, 16, 2, 256, 6000, 148)
    assert n == 3  # ceil(6000 / 2240)
    n, _ = qsa.qsa_sparse_prefill_plan(100000, 16, 2, 256, 6000, 148, 1)
    assert n == 3  # a request below the minimum is raised
    n, _ = qsa.qsa_sparse_prefill_plan(10, 16, 2, 256, 5, 148, 64)
    assert n == 5  # ... and one above W lowered
    n, ws = qsa.qsa_sparse_prefill_plan(10, 16, 2, 256, 0, 148)
    assert n == 1 and ws == 0


@pytest.mark.parametrize("Tq,Hq,Hkv,W", [
    (7810, 16, 2, 2051), (16, 16, 2, 2051), (1, 16, 2, 2051), (257, 12, 1, 2051),
    (100000, 16, 2, 6000), (10, 16, 2, 0), (64, 6, 1, 2048),
])
def test_workspace_bytes_is_the_automatic_plan(lib, Tq, Hq, Hkv, W):
    # the raw C call, argument order (Tq, Hq, Hkv, W, D, num_sms)
    raw = lib.qsa_sparse_prefill_workspace_bytes(Tq, Hq, Hkv, W, 256, 148)
    _, ws = qsa.qsa_sparse_prefill_plan(Tq, Hq, Hkv, 256, W, 148)
    assert raw == ws
    assert qsa.qsa_sparse_prefill_workspace_bytes(Tq, Hq, Hkv, W, 256, 148) == ws


@pytest.mark.parametrize("shape,status", [
    ((4, 16, 3, 8, 256), qsa.QSA_ERR_INVALID_ARG),   # Hq % Hkv
    ((4, 16, 2, 8, 128), qsa.QSA_ERR_UNSUPPORTED),   # D != 256
    ((4, 17, 1, 8, 256), qsa.QSA_ERR_UNSUPPORTED),   # G = 17
    ((-1, 16, 2, 8, 256), qsa.QSA_ERR_INVALID_ARG),  # negative Tq
])
def test_workspace_bytes_rejects(lib, shape, status):
    assert lib.qsa_sparse_prefill_workspace_bytes(*shape, 148) == ctypes.c_size_t(-1).value
    assert qsa.qsa_last_error_detail() != ""
    with pytest.raises(qsa.QSAError) as ei:
        qsa.qsa_sparse_prefill_workspace_bytes(*shape, 148)
    assert ei.value.status == status


@pytest.mark.parametrize("shape,status", [
    ((4, 16, 3, 256, 8), qsa.QSA_ERR_INVALID_ARG),   # Hq % Hkv
    ((4, 16, 2, 128, 8), qsa.QSA_ERR_UNSUPPORTED),   # D != 256
    ((4, 17, 1, 256, 8), qsa.QSA_ERR_UNSUPPORTED),   # G = 17
    ((-1, 16, 2, 256, 8), qsa.QSA_ERR_INVALID_ARG),  # negative Tq
    ((4, 16, 2, 256, -3), qsa.QSA_ERR_INVALID_ARG),  # negative W
    ((4, 0, 2, 256, 8), qsa.QSA_ERR_INVALID_ARG),
])
def test_plan_rejects(lib, shape, status):
    with pytest.raises(qsa.QSAError) as ei:
        qsa.qsa_sparse_prefill_plan(*shape, 148)
    assert ei.value.status == status


def _call(**over):
    """A raw ABI call with fake (never dereferenced) aligned pointers; every test below
    makes exactly one argument invalid so the call returns before touching CUDA."""
    a = dict(q=0x10000, q_stride_t=16 * 256, q_stride_h=256, k_cache=0x20000, k_stride_s=512,
             k_stride_h=256, v_cache=0x30000, v_stride_s=512, v_stride_h=256, slot_idx=0x40000,
             idx_stride_t=8, width=None, Tq=4, Hq=16, Hkv=2, D=256, S=100, W=8, scale=0.0625,
             out=0x50000, out_stride_t=16 * 256, out_stride_h=256, nsplit=1, workspace=None,
             workspace_bytes=0, err_word=None, stream=None)
    a.update(over)
    return qsa.qsa_sparse_prefill(**a)


INVALID = [
    (dict(q=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(k_cache=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(v_cache=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(out=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(slot_idx=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(q=0x10008), qsa.QSA_ERR_INVALID_ARG),          # misaligned base
    (dict(out=0x50002), qsa.QSA_ERR_INVALID_ARG),
    (dict(slot_idx=0x40002), qsa.QSA_ERR_INVALID_ARG),
    (dict(width=0x60001), qsa.QSA_ERR_INVALID_ARG),
    (dict(q_stride_h=260), qsa.QSA_ERR_INVALID_ARG),      # stride not a multiple of 8
    (dict(k_stride_s=-512), qsa.QSA_ERR_INVALID_ARG),
    (dict(out_stride_t=12), qsa.QSA_ERR_INVALID_ARG),
    (dict(idx_stride_t=-1), qsa.QSA_ERR_INVALID_ARG),
    (dict(Hkv=3), qsa.QSA_ERR_INVALID_ARG),
    (dict(D=128), qsa.QSA_ERR_UNSUPPORTED),
    (dict(Hq=34), qsa.QSA_ERR_UNSUPPORTED),               # G = 17
    (dict(S=-1), qsa.QSA_ERR_INVALID_ARG),
    (dict(scale=float("nan")), qsa.QSA_ERR_INVALID_ARG),
    (dict(scale=float("inf")), qsa.QSA_ERR_INVALID_ARG),
    (dict(nsplit=-2), qsa.QSA_ERR_INVALID_ARG),
    (dict(k_stride_s=2 ** 31), qsa.QSA_ERR_UNSUPPORTED),  # slot stride of 4 GiB
    (dict(nsplit=2, W=8, workspace=None), qsa.QSA_ERR_WORKSPACE),
    (dict(nsplit=2, W=8, workspace=0x70000, workspace_bytes=16), qsa.QSA_ERR_WORKSPACE),
]


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake-pointer validation runs only where no GPU can be reached")
@pytest.mark.parametrize("over,status", INVALID, ids=[str(o) for o, _ in INVALID])
def test_invalid_arguments_rejected_before_launch(lib, over, status):
    assert _call(**over) == status
    assert qsa.qsa_last_error_detail() != ""


def test_empty_batch_is_a_noop(lib):
    assert _call(Tq=0, q=None, k_cache=None, v_cache=None, out=None, slot_idx=None) == qsa.QSA_OK


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_no_device_reports_cuda_error(lib):
    # valid arguments, automatic split: the device query fails without a GPU
    assert _call(nsplit=0) == qsa.QSA_ERR_CUDA


def test_wrapper_refuses_cpu_tensors():
    q = torch.zeros(2, 16, 256, dtype=torch.bfloat16)
    k = torch.zeros(4, 2, 256, dtype=torch.bfloat16)
    idx = torch.zeros(2, 3, dtype=torch.int32)
    with pytest.raises(ValueError):
        qsa.sparse_prefill(q, k, k, idx)


def _call8(**over):
    """A raw call of the fp8_e4m3-KV entry point with fake aligned pointers (strides of
    the E4M3 caches in bytes); each case makes one argument invalid."""
    a = dict(q=0x10000, q_stride_t=16 * 256, q_stride_h=256, k_cache=0x20000, k_stride_s=512,
             k_stride_h=256, v_cache=0x30000, v_stride_s=512, v_stride_h=256, slot_idx=0x40000,
             idx_stride_t=8, width=None, Tq=4, Hq=16, Hkv=2, D=256, S=100, W=8, block=1,
             scale=0.0625, k_scale=0.0135, v_scale=0.0125, out=0x50000, out_stride_t=16 * 256,
             out_stride_h=256, nsplit=1, workspace=None, workspace_bytes=0, err_word=None,
             stream=None)
    a.update(over)
    return qsa.qsa_sparse_prefill_fp8kv(**a)


INVALID8 = [
    (dict(k_stride_h=264), qsa.QSA_ERR_INVALID_ARG),    # 264 bytes: not a multiple of 16
    (dict(v_stride_s=520), qsa.QSA_ERR_INVALID_ARG),
    (dict(k_cache=0x20008), qsa.QSA_ERR_INVALID_ARG),   # misaligned base
    (dict(k_scale=float("nan")), qsa.QSA_ERR_INVALID_ARG),
    (dict(v_scale=float("inf")), qsa.QSA_ERR_INVALID_ARG),
    (dict(block=0), qsa.QSA_ERR_INVALID_ARG),
    (dict(q_stride_h=260), qsa.QSA_ERR_INVALID_ARG),     # q stays bf16: multiples of 8
    (dict(D=128), qsa.QSA_ERR_UNSUPPORTED),
    (dict(k_stride_s=2 ** 32), qsa.QSA_ERR_UNSUPPORTED),  # slot stride of 4 GiB
    (dict(nsplit=2, workspace=None), qsa.QSA_ERR_WORKSPACE),
]


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake-pointer validation runs only where no GPU can be reached")
@pytest.mark.parametrize("over,status", INVALID8, ids=[str(o) for o, _ in INVALID8])
def test_fp8kv_invalid_arguments_rejected_before_launch(lib, over, status):
    assert _call8(**over) == status
    assert qsa.qsa_last_error_detail() != ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_fp8kv_strides_accepted_up_to_the_device_query(lib):
    # E4M3 strides are bytes: any multiple of 16 is accepted; with valid arguments the
    # automatic split reaches the device query, which fails without a GPU
    assert _call8(k_stride_h=272, nsplit=0) == qsa.QSA_ERR_CUDA
    assert _call8(Tq=0, q=None, k_cache=None, v_cache=None, out=None, slot_idx=None) == qsa.QSA_OK


def test_wrapper_refuses_cpu_fp8_tensors():
    q = torch.zeros(2, 16, 256, dtype=torch.bfloat16)
    k = torch.zeros(4, 2, 256, dtype=torch.float8_e4m3fn)
    idx = torch.zeros(2, 3, dtype=torch.int32)
    with pytest.raises(ValueError):
        qsa.sparse_prefill(q, k, k, idx, k_scale=0.5, v_scale=0.5)


def _call_partial(**over):
    """A raw call of the slot-range partial entry point with fake aligned pointers."""
    a = dict(q=0x10000, q_stride_t=16 * 256, q_stride_h=256, k_cache=0x20000, k_stride_s=512,
             k_stride_h=256, v_cache=0x30000, v_stride_s=512, v_stride_h=256, slot_idx=0x40000,
             idx_stride_t=8, width=None, Tq=4, Hq=16, Hkv=2, D=256, S=100, W=8, block=1,
             slot_lo=0, S_total=100, kv_fp8=0, scale=0.0625, k_scale=1.0, v_scale=1.0,
             part_o=0x50000, part_lse=0x60000, record_bf16=0, nsplit=1, workspace=None,
             workspace_bytes=0, err_word=None, stream=None)
    a.update(over)
    return qsa.qsa_sparse_prefill_partial(**a)


INVALID_PARTIAL = [
    (dict(part_o=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(part_lse=None), qsa.QSA_ERR_INVALID_ARG),
    (dict(part_o=0x50004), qsa.QSA_ERR_INVALID_ARG),          # misaligned record
    (dict(slot_lo=-8), qsa.QSA_ERR_INVALID_ARG),
    (dict(slot_lo=6, block=4, S=96, S_total=200), qsa.QSA_ERR_INVALID_ARG),   # not a block multiple
    (dict(slot_lo=50, S_total=120), qsa.QSA_ERR_INVALID_ARG),  # S_total < slot_lo + S
    (dict(S_total=-1), qsa.QSA_ERR_INVALID_ARG),
    (dict(kv_fp8=2), qsa.QSA_ERR_INVALID_ARG),
    (dict(record_bf16=2), qsa.QSA_ERR_INVALID_ARG),
    (dict(record_bf16=-1), qsa.QSA_ERR_INVALID_ARG),
    (dict(D=128), qsa.QSA_ERR_UNSUPPORTED),
    (dict(k_cache=None), qsa.QSA_ERR_INVALID_ARG),            # S > 0 needs the caches
]


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake-pointer validation runs only where no GPU can be reached")
@pytest.mark.parametrize("over,status", INVALID_PARTIAL, ids=[str(o) for o, _ in INVALID_PARTIAL])
def test_partial_invalid_arguments_rejected_before_launch(lib, over, status):
    assert _call_partial(**over) == status
    assert qsa.qsa_last_error_detail() != ""


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_partial_valid_shard_reaches_the_device_query(lib):
    # a shard in the middle of the cache, E4M3 caches, and an empty shard with NULL caches
    assert _call_partial(slot_lo=100, S=50, S_total=400, nsplit=0) == qsa.QSA_ERR_CUDA
    assert _call_partial(kv_fp8=1, k_scale=0.5, v_scale=0.25, nsplit=0) == qsa.QSA_ERR_CUDA
    assert _call_partial(S=0, slot_lo=100, k_cache=None, v_cache=None, nsplit=0) == qsa.QSA_ERR_CUDA
    assert _call_partial(Tq=0, q=None, part_o=None, part_lse=None) == qsa.QSA_OK


@pytest.mark.skipif(torch.cuda.is_available(),
                    reason="fake-pointer validation runs only where no GPU can be reached")
def test_combine_partials_validation(lib):
    ok = dict(part_o=0x50000, part_lse=0x60000, record_bf16=0, R=2, Tq=4, Hq=16, D=256,
              out=0x70000, out_stride_t=16 * 256, out_stride_h=256, stream=None)
    bad = [dict(R=0), dict(Hq=0), dict(Tq=-1), dict(part_o=None), dict(out=None),
           dict(part_o=0x50008), dict(out_stride_h=12), dict(record_bf16=2)]
    for over in bad:
        assert qsa.qsa_combine_partials(**{**ok, **over}) == qsa.QSA_ERR_INVALID_ARG, over
    assert qsa.qsa_combine_partials(**{**ok, "D": 128}) == qsa.QSA_ERR_UNSUPPORTED
    assert qsa.qsa_combine_partials(**{**ok, "Tq": 0, "part_o": None}) == qsa.QSA_OK
    assert qsa.qsa_combine_partials(**ok) == qsa.QSA_ERR_CUDA   # valid: the launch fails
    assert qsa.qsa_combine_partials(**{**ok, "record_bf16": 1}) == qsa.QSA_ERR_CUDA


def test_shard_ranges():
    assert qsa.shard_ranges(65536, 2) == [(0, 32768), (32768, 65536)]
    r = qsa.shard_ranges(1000, 3, block=4)
    assert r[0][0] == 0 and r[-1][1] == 1000
    assert all(lo % 4 == 0 for lo, _ in r) and all(a[1] == b[0] for a, b in zip(r, r[1:]))
    assert qsa.shard_ranges(10, 4, block=4)[-1] == (10, 10)   # more ranks than blocks


@pytest.mark.parametrize("over", [
    dict(method=4), dict(method=-1), dict(read_back=3), dict(row_bytes=128),
    dict(stages=1), dict(stages=5), dict(warps=0), dict(warps=16), dict(ctas=0), dict(iters=0),
    dict(pitch=500), dict(pitch=256), dict(src=None), dict(sink=None), dict(src=0x1008),
    dict(warps=15, stages=4),                      # 480 KiB of shared memory
])
def test_probe_rejects_bad_arguments_before_cuda(lib, over):
    a = dict(method=0, read_back=1, src=0x1000, rows=1024, pitch=512, row_bytes=512, warps=4,
             stages=2, ctas=8, iters=4, sink=0x2000)
    a.update(over)
    st = qsa.qsa_probe_gather(a["method"], a["read_back"], a["src"], a["rows"], a["pitch"],
                              a["row_bytes"], a["warps"], a["stages"], a["ctas"], a["iters"], 1,
                              a["sink"], None)
    assert st == qsa.QSA_ERR_INVALID_ARG, qsa.qsa_last_error_detail()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_probe_valid_arguments_reach_the_device(lib):
    # without a GPU the first CUDA call fails: the arguments themselves were accepted
    st = qsa.qsa_probe_gather(1, 1, 0x1000, 1024, 512, 512, 4, 2, 8, 4, 1, 0x2000, None)
    assert st == qsa.QSA_ERR_CUDA


@pytest.mark.parametrize("over", [dict(method=2), dict(method=-1), dict(method=0, n=16),
                                  dict(method=1, n=0), dict(method=1, n=48), dict(rounds=0),
                                  dict(rounds=65537), dict(ctas=0), dict(out=0), dict(out=0x1004)])
def test_mma_probe_rejects_bad_arguments_before_cuda(lib, over):
    a = dict(method=1, n=16, rounds=10, ctas=4, out=0x1000)
    a.update(over)
    st = qsa.qsa_probe_mma_operands(a["method"], a["n"], a["rounds"], a["ctas"], a["out"], None)
    assert st == qsa.QSA_ERR_INVALID_ARG, qsa.qsa_last_error_detail()


@pytest.mark.skipif(torch.cuda.is_available(), reason="checks the no-GPU error path")
def test_mma_probe_valid_arguments_reach_the_device(lib):
    assert qsa.qsa_probe_mma_operands(0, 0, 10, 4, 0x1000, None) == qsa.QSA_ERR_CUDA
    assert qsa.qsa_probe_mma_operands(1, 256, 10, 4, 0x1000, None) == qsa.QSA_ERR_CUDA


def test_partial_plan_workspace(lib):
    """A shard smaller than the cache with an unsplit plan asks for the compaction buffer
    ([Tq, W] and [Tq] int32, each 256-byte aligned); the whole cache, a narrow selection
    or a split plan ask for what qsa_sparse_prefill_block_plan asks for."""
    def r256(x):
        return (x + 255) // 256 * 256
    n, ws = qsa.qsa_sparse_prefill_partial_plan(7810, 16, 2, 256, 2051, 1, 8192, 65536, 148)
    assert n == 1 and ws == r256(7810 * 2051 * 4) + r256(7810 * 4)
    assert qsa.qsa_sparse_prefill_partial_plan(7810, 16, 2, 256, 2051, 1, 65536, 65536, 148) == (1, 0)
    assert qsa.qsa_sparse_prefill_partial_plan(100, 16, 2, 256, 31, 1, 10, 100, 148) == (1, 0)
    split = qsa.qsa_sparse_prefill_partial_plan(4, 16, 2, 256, 2051, 1, 8192, 65536, 148)
    assert split == qsa.qsa_sparse_prefill_block_plan(4, 16, 2, 256, 2051, 1, 148) and split[0] > 1
    for S, S_total in ((10, 5), (-1, 5)):
        with pytest.raises(qsa.QSAError) as ei:
            qsa.qsa_sparse_prefill_partial_plan(4, 16, 2, 256, 64, 1, S, S_total, 148)
        assert ei.value.status == qsa.QSA_ERR_INVALID_ARG


def test_plan_properties_on_random_shapes(lib):
    """Seeded random shapes through the planner (host only): every split holds at most
    2,240 slots (the per-split slot list in shared memory), no split lies wholly past W,
    a split is never narrower than 128 slots unless W itself forces it, batches of at
    least one wave of units are not split beyond what W forces, a forced request is
    honoured within those limits, and the workspace is the fp32 partials plus the LSEs,
    each region 256-byte aligned (none without a split)."""
    import random
    rng = random.Random(2024)
    max_slots, min_slots, wave = 2240, 128, 148 * 2
    for _ in range(3000):
        Hkv = rng.choice([1, 2, 3, 4, 8])
        Hq = Hkv * rng.randint(1, 16)
        Tq = rng.choice([rng.randint(1, 16), rng.randint(1, 400), rng.randint(1, 20000)])
        block = rng.choice([1, 1, 1, 2, 4, 16])
        W = rng.randint(1, 30000 // block)
        request = rng.choice([0, 0, rng.randint(1, 64)])
        n, ws = qsa.qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, 256, W, block, 148, request)
        per_split = -(-W // n)                        # entries per split
        min_split = -(-W * block // max_slots)
        assert 1 <= n <= W and per_split * block <= max_slots, (Tq, Hq, Hkv, W, block, n)
        assert (n - 1) * per_split < W, "a split lies wholly past W"
        # the count the plan settles on for a wanted count (no split wholly past W)
        settle = lambda k: -(-W // -(-W // k))  # noqa: E731
        if request == 0:
            if Tq * Hkv >= wave:
                assert n == settle(min_split), (Tq, Hkv, W, n)
            elif n > settle(min_split):
                assert per_split * block >= min_slots, (Tq, Hkv, W, block, n)
        else:
            assert n == settle(min(max(request, min_split), W)), (W, block, request, n)
        r256 = lambda x: (x + 255) // 256 * 256  # noqa: E731
        want = 0 if n == 1 else r256(n * Tq * Hq * 256 * 4) + r256(n * Tq * Hq * 4)
        assert ws == want, (Tq, Hq, Hkv, W, block, n, ws, want)
