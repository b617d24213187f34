"""GPU parity: the CUDA path through the C ABI against the CPU oracle.

Gates (article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in CANN
prefill PR", section "Nine tests that passed, ..."): atol 0.025, rtol 0.025, rel-L2
below 0.008, empty rows exactly zero, all outputs finite.  Small configurations are
compared in full; the large ones are launched at full size in the configuration the
benchmark times and compared on sampled rows (the article's long-prefill check used 8
sampled rows; these tests use more).
"""
from __future__ import annotations

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from helpers import check_gates, load_golden, valid_counts
from top_sparse_attention_index_b200 import workloads as wl

pytestmark = pytest.mark.gpu

D = 256


def dev(w: wl.Workload, device):
    """Device copies that keep the layout (the width sweep's Q stays a strided view)."""
    if w.q.is_contiguous():
        q = w.q.to(device)
    else:
        base = w.q.as_strided((w.Tq, w.q.stride(0) // (w.Hq * D), w.Hq, D),
                              (w.q.stride(0), w.Hq * D, D, 1))
        q = base.to(device)[:, 0]
        assert q.stride() == w.q.stride()
    return dict(q=q, k_cache=w.k_cache.to(device), v_cache=w.v_cache.to(device),
                slot_idx=w.slot_idx.to(device),
                width=None if w.width is None else w.width.to(device))


def run(d, scale, nsplit=0, **kw):
    out = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], d["width"],
                             scale=scale, nsplit=nsplit, **kw)
    torch.cuda.synchronize()
    return out.cpu()


def empty_rows(w, rows=None):
    cnt = valid_counts(w.slot_idx, w.width, w.S)
    rows = range(w.Tq) if rows is None else rows
    return [i for i, t in enumerate(rows) if int(cnt[t]) == 0]


def compare_rows(w, got, oracle_lib, scale, rows, label):
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, scale, rows=rows)
    return check_gates(got[rows].float(), torch.from_numpy(ref), empty_rows(w, rows), label)


# ---- golden closed forms ------------------------------------------------------------

def test_golden_closed_forms(cuda_device):
    for c in load_golden():
        d = dict(q=c["q"].to(cuda_device), k_cache=c["k"].to(cuda_device),
                 v_cache=c["v"].to(cuda_device), slot_idx=c["slot_idx"].to(cuda_device),
                 width=None if c["width"] is None else c["width"].to(cuda_device))
        got = run(d, c["scale"])
        empty = (c["expected"].abs().sum(dim=(1, 2)) == 0).nonzero().flatten().tolist()
        check_gates(got.float(), c["expected"], empty, c["name"])


# ---- the five configurations --------------------------------------------------------

@pytest.mark.parametrize("nsplit", [0, 1, 2, 4])
def test_tiny(cuda_device, oracle_lib, nsplit):
    w = wl.tiny()
    got = run(dev(w, cuda_device), 1.0 / 16.0, nsplit)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), w.notes["masked_rows"], "tiny")


@pytest.fixture(scope="module")
def width_sweep():
    return wl.width_sweep()


@pytest.mark.parametrize("scale", [1.0 / 16.0, 0.05])
@pytest.mark.parametrize("nsplit", [0, 1, 3])
def test_width_sweep(cuda_device, oracle_lib, width_sweep, scale, nsplit):
    w = width_sweep
    d = dev(w, cuda_device)
    assert not d["q"].is_contiguous()
    got = run(d, scale, nsplit)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, scale)
    check_gates(got.float(), torch.from_numpy(ref), empty_rows(w), f"width_sweep s={scale}")
    # per-width gates as well (the article lists widths 1/63/64/65/2051 separately)
    for k, wd in enumerate(wl.WIDTH_CYCLE):
        rows = list(range(k, w.Tq, len(wl.WIDTH_CYCLE)))
        check_gates(got[rows].float(), torch.from_numpy(ref[rows]), empty_rows(w, rows),
                    f"width {wd}")


def _causal_rows(Tq):
    L = 8192
    rows = set(range(0, 8)) | {L - 1, L, L + 1, L + 4095, L + 4096, Tq - 1}
    rows |= {127, 128, 129, 2050, 2051, 2052}
    rows |= {L + p for p in (127, 128, 2050, 2051, 5000)}
    g = torch.Generator().manual_seed(5)
    rows |= set(torch.randint(0, Tq, (96,), generator=g).tolist())
    return sorted(r for r in rows if r < Tq)


def test_causal_two_request(cuda_device, oracle_lib):
    w = wl.causal_two_request()
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    assert torch.isfinite(got.float()).all()
    rows = _causal_rows(w.Tq)
    # the sampled rows cover every compression-ratio-4 tail remainder of the width
    assert {int(w.width[r]) % 4 for r in rows} == {0, 1, 2, 3}
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, "causal")


def test_long_prefill_headline(cuda_device, oracle_lib):
    """7,810 queries x 2,051 slots over 65,536 slots, launched as the benchmark does
    (automatic plan); 8 evenly spaced rows as in the article plus 248 random rows."""
    w = wl.long_prefill()
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    assert torch.isfinite(got.float()).all()
    eight = [int(i * (w.Tq - 1) / 7) for i in range(8)]
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, eight, "long prefill, 8 rows")
    g = torch.Generator().manual_seed(8)
    rows = sorted(set(torch.randint(0, w.Tq, (248,), generator=g).tolist()) | set(eight))
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, "long prefill, sampled")


@pytest.mark.parametrize("Hq", [6, 3])
@pytest.mark.parametrize("clustered", [False, True])
def test_max_extent(cuda_device, oracle_lib, Hq, clustered):
    w = wl.max_extent(Hq=Hq, clustered=clustered)
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    assert torch.isfinite(got.float()).all()
    g = torch.Generator().manual_seed(9)
    rows = sorted(set(torch.randint(0, w.Tq, (64,), generator=g).tolist()) | {0, w.Tq - 1})
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, w.name)


# ---- head shapes, row counts, split plans ---------------------------------------------

def _random_case(seed, Tq, Hq, Hkv, S, W, minus1=0.0, widths=False):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    if minus1:
        idx[torch.rand(Tq, W, generator=g) < minus1] = -1
    width = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32) if widths else None
    return wl.Workload(f"rand_{Hq}_{Hkv}_{Tq}", q, k, v, idx, width)


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (24, 2), (12, 1), (6, 1), (3, 1), (16, 1), (5, 1), (2, 2),
                                    (10, 1), (32, 2)])
@pytest.mark.parametrize("Tq", [1, 257])
def test_head_shapes(cuda_device, oracle_lib, Hq, Hkv, Tq):
    w = _random_case(1000 + Hq * 10 + Hkv + Tq, Tq, Hq, Hkv, 8192, 2051, minus1=0.05, widths=True)
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), empty_rows(w), f"heads ({Hq},{Hkv}) Tq={Tq}")


@pytest.mark.parametrize("nsplit", [1, 2, 7, 16, 2051])
def test_forced_splits_decode_shape(cuda_device, oracle_lib, nsplit):
    """Few query rows with a wide selection: all the parallelism comes from splitting W,
    down to one position per split."""
    w = _random_case(77, 3, 16, 2, 65536, 2051, minus1=0.3)
    got = run(dev(w, cuda_device), 1.0 / 16.0, nsplit)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), empty_rows(w), f"nsplit={nsplit}")


@pytest.mark.parametrize("Hq,Hkv,S,nsplit", [(8, 2, 8192, 1), (4, 2, 65536, 2), (16, 2, 4096, 0),
                                             (6, 1, 20000, 3), (24, 2, 12288, 2), (20, 2, 4096, 1),
                                             (12, 1, 30000, 0), (32, 2, 8192, 1)])
def test_many_wave_launches_with_masks_and_splits(cuda_device, oracle_lib, Hq, Hkv, S, nsplit):
    """Launches of many waves (at least five waves of three CTAs per SM) on caches of at
    most 65,536 rows, for one head tile (G <= 8), two tiles with the 12-row Q tile
    (G = 10, 12) and two tiles with the full one (G = 16): ragged widths, interior -1
    entries and empty rows, with one split, forced splits (partials and the combine) and
    the automatic plan; the oracle checks every 7th row plus the first and last."""
    Tq = 2400 if Hkv == 2 else 4000
    w = _random_case(430 + Hq + S % 97, Tq, Hq, Hkv, S, 300, minus1=0.1, widths=True)
    w.slot_idx[5] = -1  # an empty row
    got = run(dev(w, cuda_device), 1.0 / 16.0, nsplit=nsplit)
    rows = sorted(set(range(0, Tq, 7)) | {1, 5, Tq - 1})
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, f"many waves Hq={Hq} S={S} nsplit={nsplit}")
    assert torch.all(got[5] == 0)


def test_many_wave_launch_block_selection(cuda_device, oracle_lib):
    """Block selection (blocks of four slots) in a launch of many waves on a 32,768-slot
    cache: sampled rows against the oracle."""
    g = torch.Generator().manual_seed(437)
    Tq, Hq, Hkv, S, W, block = 2400, 16, 2, 32768, 128, 4
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S // block, W)
    idx[torch.rand(Tq, W, generator=g) < 0.05] = -1
    out = qsa.sparse_prefill(q.to(cuda_device), k.to(cuda_device), v.to(cuda_device),
                             idx.to(cuda_device), block=block)
    torch.cuda.synchronize()
    rows = list(range(0, Tq, 11)) + [Tq - 1]
    ref = oracle_lib.forward(q, k, v, idx, None, 1.0 / 16.0, rows=rows, block=block)
    check_gates(out.cpu()[rows].float(), torch.from_numpy(ref), None, "many waves, block 4")


def test_head_major_order_four_kv_heads(cuda_device, oracle_lib):
    """A 128 MB cache of four 32 MB head slices: the launch orders its work units KV head
    slowest (the long prefill does too, with two heads); every head's rows must land."""
    w = _random_case(79, 300, 16, 4, 32768, 700, minus1=0.05, widths=True)
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    rows = list(range(0, w.Tq, 3)) + [w.Tq - 1]
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, "4 KV heads, head-major")


def test_rows_wider_than_one_split(cuda_device, oracle_lib):
    """W = 6,000 > 2,240 slots per split forces at least three splits."""
    w = _random_case(78, 300, 16, 2, 20000, 6000, minus1=0.1, widths=True)
    n, _ = qsa.qsa_sparse_prefill_plan(w.Tq, 16, 2, D, w.W, 148)
    assert n >= 3
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    rows = list(range(0, w.Tq, 5))
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, "W=6000")


# ---- edge cases -----------------------------------------------------------------------

def test_empty_rows_are_exact_zero(cuda_device):
    w = _random_case(80, 40, 16, 2, 1000, 100)
    w.slot_idx[::3] = -1                       # fully masked rows
    w.width = torch.full((40,), 100, dtype=torch.int32)
    w.width[1::3] = 0                          # zero selection width
    for nsplit in (1, 4):
        got = run(dev(w, cuda_device), 1.0 / 16.0, nsplit)
        for t in list(range(0, 40, 3)) + list(range(1, 40, 3)):
            assert (got[t].view(torch.int16) == 0).all(), t   # +0.0 bit patterns
        assert (got[2::3].float().abs().sum(dim=(1, 2)) > 0).all()


def test_zero_width_axis_and_empty_batch(cuda_device):
    q = torch.randn(5, 16, D, device=cuda_device).to(torch.bfloat16)
    kv = torch.randn(10, 2, D, device=cuda_device).to(torch.bfloat16)
    idx = torch.empty(5, 0, dtype=torch.int32, device=cuda_device)
    out = torch.full((5, 16, D), 7.0, dtype=torch.bfloat16, device=cuda_device)
    qsa.sparse_prefill(q, kv, kv, idx, out=out)
    torch.cuda.synchronize()
    assert (out.view(torch.int16) == 0).all()
    out0 = qsa.sparse_prefill(q[:0], kv, kv, idx[:0])
    assert out0.shape == (0, 16, D)


def test_width_one_returns_v_exactly(cuda_device):
    w = _random_case(81, 64, 24, 2, 4096, 50)
    w.width = torch.ones(64, dtype=torch.int32)
    got = run(dev(w, cuda_device), 0.37)
    for t in range(64):
        s = int(w.slot_idx[t, 0])
        for h in range(24):
            assert torch.equal(got[t, h], w.v_cache[s, h // 12]), (t, h)


def test_zero_query_rows_give_mean_of_v(cuda_device, oracle_lib):
    """The 'zero rows' reading of an all-zero Q row: uniform weights, mean of V."""
    w = _random_case(82, 32, 16, 2, 3000, 300, minus1=0.2)
    w.q[::2] = 0
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), empty_rows(w), "zero q rows")
    for t in range(0, 32, 2):
        sel = [int(s) for s in w.slot_idx[t] if s >= 0]
        mean = w.v_cache[sel].double().mean(dim=0)          # [Hkv, D]
        assert torch.allclose(got[t].double(), mean.repeat_interleave(8, dim=0), atol=0.01)


def test_invalid_slots_and_widths_set_error_bits(cuda_device, oracle_lib):
    w = _random_case(83, 16, 16, 2, 500, 40, widths=True)
    bad = w.slot_idx.clone()
    bad[3, 0] = 500      # == S
    bad[5, 2] = -9
    wd = w.width.clone()
    wd[7] = 41           # > W
    wd[8] = -4
    d = dev(w, cuda_device)
    d["slot_idx"] = bad.to(cuda_device)
    d["width"] = wd.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = run(d, 1.0 / 16.0, err_word=err)
    bits = int(err.item())
    assert bits & qsa.QSA_ERRBIT_SLOT_RANGE and bits & qsa.QSA_ERRBIT_WIDTH_RANGE
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, bad, wd, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), None, "invalid slots")
    clean = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    run(dev(w, cuda_device), 1.0 / 16.0, err_word=clean)
    assert int(clean.item()) == 0


def test_strided_kv_and_out_views(cuda_device, oracle_lib):
    """K and V as views into one [S, 2, Hkv, D] buffer; out as a view of a wider
    buffer: only the strides change."""
    w = _random_case(84, 100, 16, 2, 2048, 300, minus1=0.1)
    kv = torch.stack([w.k_cache, w.v_cache], dim=1).to(cuda_device)   # [S, 2, Hkv, D]
    big = torch.zeros(100, 16, 2 * D, dtype=torch.bfloat16, device=cuda_device)
    out = big[:, :, D:]
    assert not out.is_contiguous()
    qsa.sparse_prefill(w.q.to(cuda_device), kv[:, 0], kv[:, 1], w.slot_idx.to(cuda_device),
                       scale=1.0 / 16.0, out=out)
    torch.cuda.synchronize()
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    check_gates(out.cpu().float(), torch.from_numpy(ref), empty_rows(w), "strided views")
    assert (big[:, :, :D] == 0).all()


def test_deterministic_and_inputs_untouched(cuda_device):
    """Cache-content reuse: the same call twice is bitwise identical; inputs unchanged."""
    w = _random_case(85, 500, 16, 2, 16384, 2051, minus1=0.05)
    d = dev(w, cuda_device)
    before = [t.clone() for t in (d["q"], d["k_cache"], d["v_cache"], d["slot_idx"])]
    a = run(d, 1.0 / 16.0)
    b = run(d, 1.0 / 16.0)
    assert torch.equal(a.view(torch.int16), b.view(torch.int16))
    for x, y in zip(before, (d["q"], d["k_cache"], d["v_cache"], d["slot_idx"])):
        assert torch.equal(x, y)


def test_duplicate_slots_count_per_occurrence(cuda_device, oracle_lib):
    w = _random_case(86, 20, 12, 1, 64, 48)
    w.slot_idx[:, 24:] = w.slot_idx[:, :24]
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), None, "duplicates")


def test_side_stream(cuda_device, oracle_lib):
    w = _random_case(87, 64, 16, 2, 4096, 700)
    d = dev(w, cuda_device)
    s = torch.cuda.Stream(cuda_device)
    with torch.cuda.stream(s):
        out = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"])
    s.synchronize()
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    check_gates(out.cpu().float(), torch.from_numpy(ref), None, "side stream")


def test_invalid_arguments_with_device_tensors(cuda_device):
    q = torch.randn(4, 16, D, device=cuda_device).to(torch.bfloat16)
    kv = torch.randn(10, 2, D, device=cuda_device).to(torch.bfloat16)
    idx = torch.zeros(4, 3, dtype=torch.int32, device=cuda_device)
    out = torch.full((4, 16, D), 3.0, dtype=torch.bfloat16, device=cuda_device)
    # a q view whose base is not 16-byte aligned
    qq = torch.randn(4 * 16 * D + 1, device=cuda_device).to(torch.bfloat16)[1:].view(4, 16, D)
    with pytest.raises(qsa.QSAError) as ei:
        qsa.sparse_prefill(qq, kv, kv, idx, out=out)
    assert ei.value.status == qsa.QSA_ERR_INVALID_ARG
    with pytest.raises(qsa.QSAError) as ei:
        qsa.sparse_prefill(q[:, :15], kv, kv, idx[:, :], out=out[:, :15], scale=float("nan"))
    assert ei.value.status == qsa.QSA_ERR_INVALID_ARG
    with pytest.raises(qsa.QSAError) as ei:
        qsa.sparse_prefill(q[:, :15], kv, kv, idx, out=out[:, :15])   # 15 % 2 != 0
    assert ei.value.status == qsa.QSA_ERR_INVALID_ARG
    torch.cuda.synchronize()
    assert (out == 3.0).all()   # nothing was launched


# ---- decode-like batches under CUDA graph capture -------------------------------------

def _raw_call(d, out, ws, nsplit, stream):
    q, k, v, idx = d["q"], d["k_cache"], d["v_cache"], d["slot_idx"]
    return qsa.qsa_sparse_prefill(
        q.data_ptr(), q.stride(0), q.stride(1), k.data_ptr(), k.stride(0), k.stride(1),
        v.data_ptr(), v.stride(0), v.stride(1), idx.data_ptr(), idx.stride(0),
        None if d["width"] is None else d["width"].data_ptr(), q.shape[0], q.shape[1], k.shape[1],
        D, k.shape[0], idx.shape[1], 1.0 / 16.0, out.data_ptr(), out.stride(0), out.stride(1),
        nsplit, None if ws is None else ws.data_ptr(), 0 if ws is None else ws.numel(), None,
        stream)


@pytest.mark.parametrize("Tq", [1, 8, 16, 64])
def test_cuda_graph_capture_decode_shape(cuda_device, oracle_lib, Tq):
    """Few query rows with a wide selection (all parallelism from split-W plus the
    combine kernel).  The call only enqueues kernels on the given stream, so it can be
    captured into a CUDA graph; replays on new inputs written into the same buffers
    match the oracle."""
    cases = [_random_case(900 + Tq + i, Tq, 16, 2, 65536, 2051, minus1=0.1, widths=True)
             for i in range(2)]
    d = dev(cases[0], cuda_device)
    num_sms = torch.cuda.get_device_properties(cuda_device).multi_processor_count
    nsplit, ws_bytes = qsa.qsa_sparse_prefill_plan(Tq, 16, 2, D, 2051, num_sms)
    if Tq * 2 < num_sms:
        assert nsplit > 1
    ws = torch.empty(max(ws_bytes, 16), dtype=torch.uint8, device=cuda_device)
    out = torch.empty(Tq, 16, D, dtype=torch.bfloat16, device=cuda_device)
    # one eager call first: it sets the kernels' per-device attributes
    assert _raw_call(d, out, ws, nsplit, torch.cuda.current_stream().cuda_stream) == qsa.QSA_OK
    torch.cuda.synchronize()
    g = torch.cuda.CUDAGraph()
    with torch.cuda.graph(g):
        st = _raw_call(d, out, ws, nsplit, torch.cuda.current_stream().cuda_stream)
    assert st == qsa.QSA_OK
    for w in cases:
        for key, src in (("q", w.q), ("k_cache", w.k_cache), ("v_cache", w.v_cache),
                         ("slot_idx", w.slot_idx), ("width", w.width)):
            d[key].copy_(src)
        out.fill_(7.0)
        g.replay()
        torch.cuda.synchronize()
        ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 1.0 / 16.0)
        check_gates(out.cpu().float(), torch.from_numpy(ref), empty_rows(w), f"graph Tq={Tq}")


# ---- block selection -------------------------------------------------------------------

def _block_case(seed, Tq, Hq, Hkv, S, Wb, block, minus1=0.1, widths=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S // block, Wb)
    if minus1:
        idx[torch.rand(Tq, Wb, generator=g) < minus1] = -1
    width = torch.randint(0, Wb + 1, (Tq,), generator=g, dtype=torch.int32) if widths else None
    return wl.Workload(f"block{block}_{Tq}", q, k, v, idx, width)


@pytest.mark.parametrize("block,Hq,Hkv", [(4, 16, 2), (2, 24, 2), (4, 6, 1), (16, 16, 2)])
@pytest.mark.parametrize("nsplit", [0, 3])
def test_block_selection(cuda_device, oracle_lib, block, Hq, Hkv, nsplit):
    """Each entry names `block` consecutive slots (block 4: micro-blocks of four tokens)."""
    w = _block_case(300 + block + Hq, 129, Hq, Hkv, 16384, 2048 // block, block)
    d = dev(w, cuda_device)
    out = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], d["width"],
                             scale=1.0 / 16.0, nsplit=nsplit, block=block)
    torch.cuda.synchronize()
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 1.0 / 16.0, block=block)
    cnt = valid_counts(w.slot_idx, w.width, w.S // block)
    check_gates(out.cpu().float(), torch.from_numpy(ref), (cnt == 0).nonzero().flatten().tolist(),
                f"block {block}")


def test_block4_budget_rows(cuda_device, oracle_lib):
    """The indexer's budget of 2,048 micro-blocks of 4 slots: 8,192 slots per query row,
    more than one split can hold, over the 65,536-slot long-prefill cache."""
    w = _block_case(310, 512, 16, 2, 65536, 2048, 4, minus1=0.0, widths=False)
    n, _ = qsa.qsa_sparse_prefill_block_plan(512, 16, 2, D, 2048, 4, 148)
    assert n >= 4
    d = dev(w, cuda_device)
    out = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], block=4)
    torch.cuda.synchronize()
    rows = list(range(0, 512, 9))
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0, rows=rows, block=4)
    check_gates(out.cpu()[rows].float(), torch.from_numpy(ref), None, "block4 budget")


def test_block_past_cache_end_is_flagged(cuda_device, oracle_lib):
    w = _block_case(320, 16, 16, 2, 1000, 40, 4, minus1=0.0, widths=False)
    w.slot_idx[2, 5] = 250          # slots 1000..1003: past S = 1000
    w.slot_idx[4, 0] = -3
    d = dev(w, cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], block=4,
                             err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) & qsa.QSA_ERRBIT_SLOT_RANGE
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0, block=4)
    check_gates(out.cpu().float(), torch.from_numpy(ref), None, "block past end")
    with pytest.raises(qsa.QSAError):
        qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], block=17)


# ---- host-buffer API -------------------------------------------------------------------

@pytest.mark.parametrize("chunk_rows", [None, 300, 7810])
def test_sparse_prefill_from_host_matches_device_call(cuda_device, chunk_rows):
    """The pipelined host-buffer form against the device call on the whole batch: every
    chunk uses the whole batch's split plan, so one chunk gives the same bits; smaller
    chunks launch fewer waves and may take the other kernel shape, which changes only the
    order of the sums (checked with the parity gates against the device call)."""
    w = wl.long_prefill()
    d = dev(w, cuda_device)
    ref = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"]).cpu()
    pinned = [x.pin_memory() for x in (w.q, w.k_cache, w.v_cache, w.slot_idx)]
    out, fin = qsa.sparse_prefill_from_host(*pinned, device=cuda_device, chunk_rows=chunk_rows)
    fin.synchronize()
    if chunk_rows == w.Tq:
        assert torch.equal(out.view(torch.int16), ref.view(torch.int16))
    else:
        check_gates(out.float(), ref.float(), None, f"from_host chunks of {chunk_rows}")


def test_sparse_prefill_from_host_width_and_masks(cuda_device, oracle_lib):
    w = wl.width_sweep()
    out, fin = qsa.sparse_prefill_from_host(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width,
                                            scale=0.05, device=cuda_device, chunk_rows=50)
    fin.synchronize()
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 0.05)
    check_gates(out.float(), torch.from_numpy(ref), empty_rows(w), "from_host width sweep")


# ---- maximum sizes ----------------------------------------------------------------------

def test_large_cache_two_million_slots(cuda_device, oracle_lib):
    """S = 2,097,152 slots at Hkv = 2 (2 GiB each for K and V on the device).  Only the
    selected rows hold data; the oracle runs on a compact copy of those rows with the
    indices renumbered (the definition does not depend on where a row lives)."""
    S, Hq, Hkv, Tq, W = 1 << 21, 16, 2, 64, 2051
    g = torch.Generator().manual_seed(401)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[:, ::7] = -1
    used = torch.unique(idx[idx >= 0])
    rows_k = torch.randn(used.numel(), Hkv, D, generator=g).to(torch.bfloat16)
    rows_v = torch.randn(used.numel(), Hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k_dev = torch.zeros(S, Hkv, D, dtype=torch.bfloat16, device=cuda_device)
    v_dev = torch.zeros(S, Hkv, D, dtype=torch.bfloat16, device=cuda_device)
    k_dev[used.to(cuda_device)] = rows_k.to(cuda_device)
    v_dev[used.to(cuda_device)] = rows_v.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = qsa.sparse_prefill(q.to(cuda_device), k_dev, v_dev, idx.to(cuda_device), err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    remap = torch.full((S,), -1, dtype=torch.int32)
    remap[used] = torch.arange(used.numel(), dtype=torch.int32)
    idx_c = torch.where(idx >= 0, remap[idx.clamp(min=0).long()], idx)
    ref = oracle_lib.forward(q, rows_k, rows_v, idx_c, None, 1.0 / 16.0)
    check_gates(out.cpu().float(), torch.from_numpy(ref), None, "2M-slot cache")
    del k_dev, v_dev


def _far_and_near(g, Tq, S, W, far):
    """Distinct slots per row: W // 2 from the last `far` slots of the cache, the rest
    from below them (shuffled together)."""
    a = (S - far) + wl.uniform_distinct(g, Tq, far, W // 2)
    b = wl.uniform_distinct(g, Tq, S - far, W - W // 2)
    idx = torch.cat([a, b], dim=1)
    perm = torch.argsort(torch.rand(Tq, W, generator=g), dim=1)
    return torch.gather(idx, 1, perm).to(torch.int32)


def test_cache_offsets_beyond_4gib(cuda_device, oracle_lib):
    """S = 9,000,000 slots at Hkv = 1: K and V are 4.6 GB each, and half of every row's
    selection lies past byte offset 4 GiB (slot 8,388,608), where a 32-bit row offset
    would wrap to another row.  Only the selected rows hold data; the oracle runs on a
    compact copy with the indices renumbered."""
    S, Hq, Hkv, Tq, W = 9_000_000, 8, 1, 48, 1500
    g = torch.Generator().manual_seed(404)
    idx = _far_and_near(g, Tq, S, W, far=S - (1 << 23))
    assert int((idx >= (1 << 23)).sum()) >= Tq * (W // 2)
    idx[:, ::11] = -1
    used = torch.unique(idx[idx >= 0])
    rows_k = torch.randn(used.numel(), Hkv, D, generator=g).to(torch.bfloat16)
    rows_v = torch.randn(used.numel(), Hkv, D, generator=g).to(torch.bfloat16)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k_dev = torch.zeros(S, Hkv, D, dtype=torch.bfloat16, device=cuda_device)
    v_dev = torch.zeros(S, Hkv, D, dtype=torch.bfloat16, device=cuda_device)
    k_dev[used.to(cuda_device)] = rows_k.to(cuda_device)
    v_dev[used.to(cuda_device)] = rows_v.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = qsa.sparse_prefill(q.to(cuda_device), k_dev, v_dev, idx.to(cuda_device), err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    remap = torch.full((S,), -1, dtype=torch.int32)
    remap[used] = torch.arange(used.numel(), dtype=torch.int32)
    idx_c = torch.where(idx >= 0, remap[idx.clamp(min=0).long()], idx)
    ref = oracle_lib.forward(q, rows_k, rows_v, idx_c, None, 1.0 / 16.0)
    check_gates(out.cpu().float(), torch.from_numpy(ref), None, "cache past 4 GiB")
    del k_dev, v_dev


def test_query_and_output_offsets_beyond_2gib(cuda_device, oracle_lib):
    """Tq = 270,000 rows at Hq = 16: Q and the output are 2.2 GB each, so rows from
    262,144 on start past byte offset 2 GiB (a signed 32-bit offset would be negative).
    Q repeats one 1,000-row block (built on the device by torch); the oracle checks the
    first rows, rows around the 2 GiB boundary and the last rows."""
    Tq, Hq, Hkv, S, W = 270_000, 16, 2, 4096, 8
    g = torch.Generator().manual_seed(405)
    q_small = torch.randn(1000, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = wl.uniform_distinct(g, Tq, S, W)
    idx[::5, 3] = -1
    idx[Tq - 1] = -1  # the very last row is empty: exact zeros past 2 GiB
    q_dev = q_small.to(cuda_device).repeat(Tq // 1000, 1, 1)
    out = qsa.sparse_prefill(q_dev, k.to(cuda_device), v.to(cuda_device), idx.to(cuda_device))
    torch.cuda.synchronize()
    rows = (list(range(0, 8)) + list(range(262_140, 262_150)) + list(range(Tq - 9, Tq)))
    got = out[torch.tensor(rows, device=cuda_device)].cpu()
    r = torch.tensor(rows)
    ref = oracle_lib.forward(q_small[r % 1000], k, v, idx[r], None, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), [len(rows) - 1], "output past 2 GiB")
    del q_dev, out


def test_very_wide_selection(cuda_device, oracle_lib):
    """W = 20,000 selected slots per row: at least eight splits, combined by the LSE
    kernel."""
    w = _random_case(402, 40, 16, 2, 65536, 20000, minus1=0.05, widths=True)
    n, _ = qsa.qsa_sparse_prefill_plan(40, 16, 2, D, 20000, 148)
    assert n >= 8
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    rows = list(range(0, 40, 3))
    compare_rows(w, got, oracle_lib, 1.0 / 16.0, rows, "W=20000")


def _convex_hull_all_rows(w, got, v_scale=1.0, chunk=128):
    """Every output element is a convex combination of the selected V rows' elements:
    it lies between their minimum and maximum for that (KV head, d), up to the bf16
    rounding of the output.  Checked for every row and head at full size on the GPU
    (torch gathers; the product path is not involved)."""
    dev = torch.device("cuda", 0)
    v = w.v_cache.to(dev)
    vf = (v.float() * v_scale) if v.dtype == torch.float8_e4m3fn else v.float()
    G = w.Hq // w.Hkv
    out = got.to(dev).float().view(w.Tq, w.Hkv, G, D)
    for r0 in range(0, w.Tq, chunk):
        idx = w.slot_idx[r0:r0 + chunk].to(dev).long()
        valid = idx >= 0
        rows = vf[idx.clamp_min(0)]                            # [c, W, Hkv, D]
        big = torch.finfo(torch.float32).max
        lo = torch.where(valid[..., None, None], rows, big).amin(dim=1)    # [c, Hkv, D]
        hi = torch.where(valid[..., None, None], rows, -big).amax(dim=1)
        o = out[r0:r0 + chunk]                                   # [c, Hkv, G, D]
        tol = 2.0 ** -7 * torch.maximum(lo.abs(), hi.abs())[:, :, None, :] + 1e-6
        assert (o >= lo[:, :, None, :] - tol).all() and (o <= hi[:, :, None, :] + tol).all(), r0


def test_long_prefill_all_rows_in_convex_hull(cuda_device):
    w = wl.long_prefill()
    got = run(dev(w, cuda_device), 1.0 / 16.0)
    _convex_hull_all_rows(w, got)


# ---- context parallelism: slot-range shards emulated on one device ----------------------

def _shards_combined(w, d, R, scale=1.0 / 16.0, nsplit=0, **kw):
    """Every shard's partial record (one device standing in for R ranks, one after
    another), stacked as an all-gather would and combined."""
    rec_o, rec_l = [], []
    for lo, hi in qsa.shard_ranges(w.S, R, w.block):
        po, pl = qsa.sparse_prefill_partial(d["q"], d["k_cache"][lo:hi], d["v_cache"][lo:hi],
                                            d["slot_idx"], lo, w.S, width=d["width"],
                                            scale=scale, nsplit=nsplit, block=w.block, **kw)
        rec_o.append(po)
        rec_l.append(pl)
    out = qsa.combine_partials(torch.stack(rec_o), torch.stack(rec_l))
    torch.cuda.synchronize()
    _shards_combined.last_records = rec_o
    return out.cpu(), rec_l


@pytest.mark.parametrize("rec", [torch.float32, torch.bfloat16], ids=["fp32", "bf16"])
@pytest.mark.parametrize("R", [1, 2, 3, 5])
def test_context_parallel_shards(cuda_device, oracle_lib, R, rec):
    w = _random_case(90 + R, 300, 16, 2, 16384, 2051, minus1=0.05, widths=True)
    d = dev(w, cuda_device)
    got, rec_l = _shards_combined(w, d, R, record_dtype=rec)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 1.0 / 16.0)
    check_gates(got.float(), torch.from_numpy(ref), empty_rows(w), f"context parallel R={R} {rec}")
    if R == 1:  # one shard holding the whole cache: bitwise the unsharded call
        assert torch.equal(got.view(torch.int16), run(d, 1.0 / 16.0).view(torch.int16))
    for t in empty_rows(w):
        assert all(torch.isinf(l[t]).all() for l in rec_l)
        # a record with no valid slot holds zeros (the documented record content)
        assert all((o[t] == 0).all() for o in _shards_combined.last_records)


def test_context_parallel_compaction_is_bitwise_the_full_scan(cuda_device):
    """A shard given the workspace for the compaction pass (every row's local entries
    copied first) returns bitwise the record of the same shard scanning the global
    selection itself, and flags the same invalid values: ragged widths (some outside
    [0, W]), interior -1, out-of-range slots, rows with no local entry; block selection
    too."""
    for block, R in ((1, 3), (4, 5)):
        w = _random_case(480 + block, 700, 16, 2, 16384, 2051 // block, minus1=0.1, widths=True)
        w.block = block
        w.slot_idx = wl.uniform_distinct(torch.Generator().manual_seed(481), 700, 16384 // block,
                                         2051 // block)
        w.slot_idx[torch.rand(700, 2051 // block, generator=torch.Generator().manual_seed(482)) < 0.1] = -1
        w.slot_idx[7, 3] = 16384 // block + 5          # invalid: past the cache
        w.slot_idx[8, 0] = -7                          # invalid: negative
        w.width[7] = w.width[8] = 2051 // block        # (both read)
        w.width[9] = 2051 // block + 3                 # invalid: width past W
        w.width[10] = -2                               # invalid: negative width
        d = dev(w, cuda_device)
        for lo, hi in qsa.shard_ranges(w.S, R, block):
            recs, errs = [], []
            for compact in (True, False):
                err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
                po, pl = qsa.sparse_prefill_partial(d["q"], d["k_cache"][lo:hi], d["v_cache"][lo:hi],
                                                    d["slot_idx"], lo, w.S, width=d["width"],
                                                    block=block, err_word=err, compact=compact,
                                                    record_dtype=torch.bfloat16)
                torch.cuda.synchronize()
                recs.append((po.cpu(), pl.cpu()))
                errs.append(int(err.item()))
            assert torch.equal(recs[0][0].view(torch.int16), recs[1][0].view(torch.int16))
            assert torch.equal(recs[0][1], recs[1][1])
            assert errs[0] == errs[1] == 3, errs


def test_context_parallel_wide_rows_and_decode(cuda_device, oracle_lib):
    """W = 6,000 (each shard combines its own splits into one record) and a decode-shape
    batch with forced split counts."""
    w = _random_case(95, 120, 16, 2, 20000, 6000, minus1=0.1, widths=True)
    rows = list(range(0, w.Tq, 4))
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 1.0 / 16.0, rows=rows)
    for rec in (torch.float32, torch.bfloat16):  # the shards' own splits combine into bf16 too
        got, _ = _shards_combined(w, dev(w, cuda_device), 3, record_dtype=rec)
        check_gates(got[rows].float(), torch.from_numpy(ref), empty_rows(w, rows),
                    f"context parallel W=6000 {rec}")
    w = _random_case(96, 3, 16, 2, 65536, 2051, minus1=0.2)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    for nsplit in (1, 4, 16):
        for rec in (torch.float32, torch.bfloat16):
            got, _ = _shards_combined(w, dev(w, cuda_device), 2, nsplit=nsplit, record_dtype=rec)
            check_gates(got.float(), torch.from_numpy(ref), empty_rows(w),
                        f"context parallel decode n={nsplit} {rec}")


def test_context_parallel_block4_and_empty_shard(cuda_device, oracle_lib):
    """Block selection with shard boundaries on block multiples, and more ranks than
    blocks (the last shard is empty: NULL-free zero-row caches, a record of -inf)."""
    w = _random_case(97, 64, 16, 2, 4096, 300, minus1=0.1)
    w.slot_idx = wl.uniform_distinct(torch.Generator().manual_seed(98), 64, 1024, 300)
    w.block = 4
    got, _ = _shards_combined(w, dev(w, cuda_device), 3, record_dtype=torch.bfloat16)
    ref = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0, block=4)
    check_gates(got.float(), torch.from_numpy(ref), None, "context parallel block4")
    t = _random_case(99, 8, 16, 2, 12, 10, minus1=0.0)
    t.block = 4  # 3 blocks over 4 ranks
    t.slot_idx = torch.tensor([[0, 1, 2, -1, -1, -1, -1, -1, -1, -1]] * 8, dtype=torch.int32)
    got, rec_l = _shards_combined(t, dev(t, cuda_device), 4, record_dtype=torch.bfloat16)
    assert torch.isinf(rec_l[3]).all()
    ref = oracle_lib.forward(t.q, t.k_cache, t.v_cache, t.slot_idx, None, 1.0 / 16.0, block=4)
    check_gates(got.float(), torch.from_numpy(ref), None, "context parallel empty shard")


def test_context_parallel_nccl_world_of_one(cuda_device):
    """The public context-parallel call end to end on one GPU: a one-rank NCCL group,
    its all-gather and the combine, then the peer exchange with its NCCL barriers; one
    shard holding the whole cache gives bitwise the unsharded call either way."""
    import datetime
    import os
    import socket

    import torch.distributed as dist
    if dist.is_initialized():
        pytest.skip("a process group already exists")
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        port = s.getsockname()[1]
    os.environ["MASTER_ADDR"] = "127.0.0.1"
    os.environ["MASTER_PORT"] = str(port)
    dist.init_process_group("nccl", rank=0, world_size=1, device_id=cuda_device,
                            timeout=datetime.timedelta(seconds=60))
    try:
        w = _random_case(89, 200, 16, 2, 16384, 2051, minus1=0.05, widths=True)
        d = dev(w, cuda_device)
        lo, hi = qsa.shard_ranges(w.S, dist.get_world_size())[dist.get_rank()]
        out = qsa.sparse_prefill_context_parallel(d["q"], d["k_cache"][lo:hi], d["v_cache"][lo:hi],
                                                  d["slot_idx"], lo, w.S, width=d["width"])
        torch.cuda.synchronize()
        unsharded = run(d, 1.0 / 16.0).view(torch.int16)
        assert torch.equal(out.cpu().view(torch.int16), unsharded)
        # the peer exchange over the same group: its buffers, the NCCL barriers on the
        # compute stream and the combine of this rank's rows (all of them), twice
        for _ in range(2):
            out = qsa.sparse_prefill_context_parallel(d["q"], d["k_cache"][lo:hi], d["v_cache"][lo:hi],
                                                      d["slot_idx"], lo, w.S, width=d["width"],
                                                      exchange="peer")
            torch.cuda.synchronize()
            assert torch.equal(out.cpu().view(torch.int16), unsharded)
        qsa.release_peer_exchanges()
    finally:
        dist.destroy_process_group()
