"""GPU parity of the fp8_e4m3 KV-cache path: the CUDA kernels through the C ABI
(qsa_sparse_prefill_fp8kv) against the oracle's fp8 path.

The format is the one the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside
SGLang's opt-in CANN prefill PR" names in section "Where this sits in the Qwen4Exp
serving build-out" (fp8_e4m3 KV cache); the cache holds E4M3 codes with one scale per
tensor.  The gates are the bf16 path's (section "Nine tests that passed, ..."): atol
0.025, rtol 0.025, rel-L2 below 0.008, empty rows exactly zero, all outputs finite.
Both sides read the same codes, so the only differences are rounding (f16 tensor-core
inputs, f16 softmax weights, fp32 accumulation, bf16 output).
"""
from __future__ import annotations

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from helpers import check_gates, valid_counts
from top_sparse_attention_index_b200 import workloads as wl

pytestmark = pytest.mark.gpu

D = 256
KS, VS = wl.E4M3_K_SCALE, wl.E4M3_V_SCALE


def dev(w, device):
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


def run(w, d, scale, nsplit=0, **kw):
    out = qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], d["width"],
                             scale=scale, nsplit=nsplit, block=w.block, k_scale=w.k_scale,
                             v_scale=w.v_scale, **kw)
    torch.cuda.synchronize()
    return out.cpu()


def empty_rows(w, rows=None):
    cnt = valid_counts(w.slot_idx, w.width, w.S // w.block if w.block > 1 else w.S)
    rows = range(w.Tq) if rows is None else rows
    return [i for i, t in enumerate(rows) if int(cnt[t]) == 0]


def oracle_rows(oracle_lib, w, scale, rows=None):
    return torch.from_numpy(oracle_lib.forward_fp8kv(
        w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, scale, w.k_scale, w.v_scale, rows=rows,
        block=w.block))


def compare(w, got, oracle_lib, scale, rows, label):
    ref = oracle_rows(oracle_lib, w, scale, rows)
    sel = got if rows is None else got[rows]
    return check_gates(sel.float(), ref, empty_rows(w, rows), label)


def _random_case(seed, Tq, Hq, Hkv, S, W, minus1=0.0, widths=False, ks=KS, vs=VS):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g)
    v = torch.randn(S, Hkv, D, generator=g)
    idx = wl.uniform_distinct(g, Tq, S, W)
    if minus1:
        idx[torch.rand(Tq, W, generator=g) < minus1] = -1
    width = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32) if widths else None
    return wl.Workload(f"e4m3_{Hq}_{Hkv}_{Tq}", q, wl.to_e4m3_cache(k, ks), wl.to_e4m3_cache(v, vs),
                       idx, width, kv_format="e4m3", k_scale=ks, v_scale=vs)


@pytest.mark.parametrize("nsplit", [0, 1, 2, 4])
def test_tiny(cuda_device, oracle_lib, nsplit):
    w = wl.with_e4m3_cache(wl.tiny())
    got = run(w, dev(w, cuda_device), 1.0 / 16.0, nsplit)
    compare(w, got, oracle_lib, 1.0 / 16.0, None, "e4m3 tiny")
    for t in w.notes["masked_rows"]:
        assert (got[t].view(torch.int16) == 0).all()


@pytest.mark.parametrize("scale", [1.0 / 16.0, 0.05])
@pytest.mark.parametrize("nsplit", [0, 3])
def test_width_sweep(cuda_device, oracle_lib, scale, nsplit):
    w = wl.with_e4m3_cache(wl.width_sweep())
    d = dev(w, cuda_device)
    assert not d["q"].is_contiguous()
    got = run(w, d, scale, nsplit)
    compare(w, got, oracle_lib, scale, None, f"e4m3 width_sweep s={scale}")


@pytest.mark.parametrize("Hq,Hkv", [(16, 2), (24, 2), (12, 1), (6, 1), (3, 1), (16, 1), (5, 1), (2, 2),
                                    (10, 1), (32, 2)])
@pytest.mark.parametrize("Tq", [1, 257])
def test_head_shapes(cuda_device, oracle_lib, Hq, Hkv, Tq):
    """Both kernel shapes (G <= 8 and G > 8), ragged widths and interior -1s."""
    w = _random_case(2000 + Hq * 10 + Hkv + Tq, Tq, Hq, Hkv, 8192, 2051, minus1=0.05, widths=True)
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    compare(w, got, oracle_lib, 1.0 / 16.0, None, f"e4m3 heads ({Hq},{Hkv}) Tq={Tq}")


@pytest.mark.parametrize("ks,vs", [(1.0, 1.0), (0.5, 0.03125), (0.0021, 0.0937)])
def test_scales(cuda_device, oracle_lib, ks, vs):
    """Power-of-two and general scales; k_scale sharpens or flattens the softmax."""
    w = _random_case(2100, 64, 16, 2, 4096, 700, minus1=0.1, ks=max(ks, 0.01), vs=vs)
    w.k_scale, w.v_scale = ks, vs
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    compare(w, got, oracle_lib, 1.0 / 16.0, None, f"e4m3 scales k={ks} v={vs}")


@pytest.mark.parametrize("nsplit", [1, 2, 16])
def test_forced_splits_decode_shape(cuda_device, oracle_lib, nsplit):
    w = _random_case(2200, 3, 16, 2, 65536, 2051, minus1=0.3)
    got = run(w, dev(w, cuda_device), 1.0 / 16.0, nsplit)
    compare(w, got, oracle_lib, 1.0 / 16.0, None, f"e4m3 nsplit={nsplit}")


def test_causal_two_request(cuda_device, oracle_lib):
    w = wl.with_e4m3_cache(wl.causal_two_request())
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    assert torch.isfinite(got.float()).all()
    g = torch.Generator().manual_seed(15)
    rows = sorted(set(torch.randint(0, w.Tq, (96,), generator=g).tolist()) | {0, 1, 127, 128, w.Tq - 1})
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, "e4m3 causal")


def test_long_prefill(cuda_device, oracle_lib):
    """The long prefill with an E4M3 cache, launched as the benchmark does."""
    w = wl.long_prefill_e4m3kv()
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    assert torch.isfinite(got.float()).all()
    eight = [int(i * (w.Tq - 1) / 7) for i in range(8)]
    compare(w, got, oracle_lib, 1.0 / 16.0, eight, "e4m3 long prefill, 8 rows")
    g = torch.Generator().manual_seed(18)
    rows = sorted(set(torch.randint(0, w.Tq, (248,), generator=g).tolist()) | set(eight))
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, "e4m3 long prefill, sampled")


def test_max_extent(cuda_device, oracle_lib):
    w = wl.with_e4m3_cache(wl.max_extent(Hq=6, clustered=True))
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    g = torch.Generator().manual_seed(19)
    rows = sorted(set(torch.randint(0, w.Tq, (64,), generator=g).tolist()) | {0, w.Tq - 1})
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, "e4m3 " + w.name)


@pytest.mark.parametrize("block", [2, 4])
def test_block_selection(cuda_device, oracle_lib, block):
    w = _random_case(2300 + block, 96, 16, 2, 8192, 700 // block, minus1=0.1, widths=True)
    w.slot_idx = wl.uniform_distinct(torch.Generator().manual_seed(5 + block), 96,
                                     8192 // block, 700 // block)
    w.slot_idx[torch.rand(96, 700 // block, generator=torch.Generator().manual_seed(6)) < 0.1] = -1
    w.block = block
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    compare(w, got, oracle_lib, 1.0 / 16.0, None, f"e4m3 block{block}")


def test_edge_cases(cuda_device, oracle_lib):
    """Fully masked rows and zero widths give +0; width 1 returns the dequantised V row
    rounded to bf16; out-of-range slots are masked and flagged; a repeat call is
    bitwise identical."""
    w = _random_case(2400, 40, 16, 2, 1000, 100, widths=True)
    w.slot_idx[::3] = -1
    w.width[1::3] = 0
    w.width[2::9] = 1
    bad = w.slot_idx.clone()
    bad[5, 0] = 1000
    bad[8, 3] = -6
    d = dev(w, cuda_device)
    d["slot_idx"] = bad.to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = run(w, d, 1.0 / 16.0, err_word=err)
    assert int(err.item()) & qsa.QSA_ERRBIT_SLOT_RANGE
    assert not int(err.item()) & qsa.QSA_ERRBIT_Q_RANGE
    for t in list(range(0, 40, 3)) + list(range(1, 40, 3)):
        assert (got[t].view(torch.int16) == 0).all(), t
    for t in range(2, 40, 9):
        if int(bad[t, 0]) >= 0:
            s = int(bad[t, 0])
            ref = (w.v_cache[s].float() * w.v_scale).to(torch.bfloat16)
            assert torch.equal(got[t], ref.repeat_interleave(8, dim=0)), t
    w.slot_idx = bad
    compare(w, got, oracle_lib, 1.0 / 16.0, None, "e4m3 edge cases")
    again = run(w, d, 1.0 / 16.0)
    assert torch.equal(again.view(torch.int16), got.view(torch.int16))


def test_query_outside_f16_range_is_flagged(cuda_device, oracle_lib):
    """|q| >= 65536 cannot be an f16 tensor-core input: the call flags it (its row is
    not valid); the other rows are unaffected."""
    w = _random_case(2500, 8, 16, 2, 500, 64)
    w.q[3, 5, 17] = 70000.0
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    got = run(w, dev(w, cuda_device), 1.0 / 16.0, err_word=err)
    assert int(err.item()) & qsa.QSA_ERRBIT_Q_RANGE
    rows = [0, 1, 2, 4, 5, 6, 7]
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, "e4m3 other rows")


def test_zero_width_axis(cuda_device):
    q = torch.randn(5, 16, D, device=cuda_device).to(torch.bfloat16)
    kv = torch.zeros(10, 2, D, device=cuda_device).to(torch.float8_e4m3fn)
    idx = torch.empty(5, 0, dtype=torch.int32, device=cuda_device)
    out = torch.full((5, 16, D), 7.0, dtype=torch.bfloat16, device=cuda_device)
    qsa.sparse_prefill(q, kv, kv, idx, out=out, k_scale=0.5, v_scale=0.5)
    torch.cuda.synchronize()
    assert (out.view(torch.int16) == 0).all()


def test_from_host_and_graph_capture(cuda_device, oracle_lib):
    """The host-buffer path and CUDA-graph replay with an E4M3 cache."""
    w = _random_case(2600, 64, 16, 2, 16384, 2051, minus1=0.05)
    pinned = {k: v.pin_memory() for k, v in dict(q=w.q, k=w.k_cache, v=w.v_cache, i=w.slot_idx).items()}
    out, ev = qsa.sparse_prefill_from_host(pinned["q"], pinned["k"], pinned["v"], pinned["i"],
                                           k_scale=w.k_scale, v_scale=w.v_scale, chunk_rows=24)
    ev.synchronize()
    d = dev(w, cuda_device)
    direct = run(w, d, 1.0 / 16.0)
    assert torch.equal(out.view(torch.int16), direct.view(torch.int16))
    # capture one call with a preallocated output and replay it on new indices
    o = torch.empty(w.Tq, w.Hq, D, dtype=torch.bfloat16, device=cuda_device)
    qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], out=o, nsplit=1,
                       k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph):
        qsa.sparse_prefill(d["q"], d["k_cache"], d["v_cache"], d["slot_idx"], out=o, nsplit=1,
                           k_scale=w.k_scale, v_scale=w.v_scale)
    w.slot_idx = wl.uniform_distinct(torch.Generator().manual_seed(99), w.Tq, w.S, w.W)
    d["slot_idx"].copy_(w.slot_idx.to(cuda_device))
    graph.replay()
    torch.cuda.synchronize()
    compare(w, o.cpu(), oracle_lib, 1.0 / 16.0, None, "e4m3 graph replay")
    del graph


def test_long_prefill_all_rows_in_convex_hull(cuda_device):
    """Every output element of the full-size E4M3 long prefill lies between the minimum and
    the maximum of its selected dequantised V elements (up to the output's bf16 rounding)."""
    from test_parity_gpu import _convex_hull_all_rows
    w = wl.long_prefill_e4m3kv()
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    _convex_hull_all_rows(w, got, v_scale=w.v_scale)


def test_forward_golden(cuda_device):
    """The hand-worked fp8 forward cases (tests/golden/e4m3_forward_cases.json) through the
    CUDA path, against their exact expected values."""
    from test_oracle_fp8kv_pins import load_forward_golden
    for c in load_forward_golden():
        out = qsa.sparse_prefill(c["q"].to(cuda_device),
                                 c["k"].view(torch.float8_e4m3fn).to(cuda_device),
                                 c["v"].view(torch.float8_e4m3fn).to(cuda_device),
                                 c["slot_idx"].to(cuda_device), scale=c["scale"],
                                 k_scale=c["k_scale"], v_scale=c["v_scale"])
        torch.cuda.synchronize()
        empty = (c["expected"].abs().sum(dim=(1, 2)) == 0).nonzero().flatten().tolist()
        check_gates(out.float().cpu(), c["expected"], empty, "e4m3 golden: " + c["name"])


def test_strided_kv_and_out_views(cuda_device, oracle_lib):
    """E4M3 K and V as views into one [S, 2, Hkv, D] code buffer (byte strides); out as a
    view of a wider buffer."""
    w = _random_case(2700, 100, 16, 2, 2048, 300, minus1=0.1)
    kv = torch.stack([w.k_cache.view(torch.uint8), w.v_cache.view(torch.uint8)], dim=1)
    kv = kv.view(torch.float8_e4m3fn).to(cuda_device)                  # [S, 2, Hkv, D]
    big = torch.zeros(100, 16, 2 * D, dtype=torch.bfloat16, device=cuda_device)
    out = big[:, :, D:]
    assert not out.is_contiguous() and not kv[:, 0].is_contiguous()
    qsa.sparse_prefill(w.q.to(cuda_device), kv[:, 0], kv[:, 1], w.slot_idx.to(cuda_device),
                       scale=1.0 / 16.0, out=out, k_scale=w.k_scale, v_scale=w.v_scale)
    torch.cuda.synchronize()
    compare(w, out.cpu(), oracle_lib, 1.0 / 16.0, None, "e4m3 strided views")
    assert (big[:, :, :D] == 0).all()


def test_context_parallel_shards(cuda_device, oracle_lib):
    """E4M3 cache split by slot range over 3 emulated ranks: records stacked and combined."""
    from test_parity_gpu import _shards_combined
    w = _random_case(2800, 200, 16, 2, 16384, 2051, minus1=0.05, widths=True)
    for rec in (torch.float32, torch.bfloat16):
        got, _ = _shards_combined(w, dev(w, cuda_device), 3, k_scale=w.k_scale,
                                  v_scale=w.v_scale, record_dtype=rec)
        compare(w, got, oracle_lib, 1.0 / 16.0, None, f"e4m3 context parallel R=3 {rec}")


def test_cache_offsets_beyond_4gib(cuda_device, oracle_lib):
    """S = 18,000,000 slots at Hkv = 1: the E4M3 K and V caches are 4.6 GB each (256-byte
    rows), and half of every row's selection lies past byte offset 4 GiB (slot
    16,777,216), where a 32-bit row offset would wrap.  Only the selected rows hold
    codes; the oracle runs on a compact copy with the indices renumbered."""
    S, Hq, Hkv, Tq, W = 18_000_000, 8, 1, 48, 1500
    far = S - (1 << 24)
    g = torch.Generator().manual_seed(406)
    a = (S - far) + wl.uniform_distinct(g, Tq, far, W // 2)
    b = wl.uniform_distinct(g, Tq, S - far, W - W // 2)
    idx = torch.cat([a, b], dim=1)
    idx = torch.gather(idx, 1, torch.argsort(torch.rand(Tq, W, generator=g), dim=1)).to(torch.int32)
    idx[:, ::11] = -1
    used = torch.unique(idx[idx >= 0])
    rows_k = wl.to_e4m3_cache(torch.randn(used.numel(), Hkv, D, generator=g), KS)
    rows_v = wl.to_e4m3_cache(torch.randn(used.numel(), Hkv, D, generator=g), VS)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k_dev = torch.zeros(S, Hkv, D, dtype=torch.uint8, device=cuda_device)
    v_dev = torch.zeros(S, Hkv, D, dtype=torch.uint8, device=cuda_device)
    k_dev[used.to(cuda_device)] = rows_k.view(torch.uint8).to(cuda_device)
    v_dev[used.to(cuda_device)] = rows_v.view(torch.uint8).to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = qsa.sparse_prefill(q.to(cuda_device), k_dev.view(torch.float8_e4m3fn),
                             v_dev.view(torch.float8_e4m3fn), idx.to(cuda_device), scale=1.0 / 16.0,
                             k_scale=KS, v_scale=VS, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0
    remap = torch.full((S,), -1, dtype=torch.int32)
    remap[used] = torch.arange(used.numel(), dtype=torch.int32)
    idx_c = torch.where(idx >= 0, remap[idx.clamp(min=0).long()], idx)
    ref = oracle_lib.forward_fp8kv(q, rows_k, rows_v, idx_c, None, 1.0 / 16.0, KS, VS)
    check_gates(out.cpu().float(), torch.from_numpy(ref), None, "E4M3 cache past 4 GiB")
    del k_dev, v_dev


@pytest.mark.parametrize("Hq,Hkv,S,nsplit", [(8, 2, 8192, 1), (6, 1, 30000, 3), (12, 1, 12000, 1),
                                              (24, 2, 12288, 2), (16, 1, 65536, 1)])
def test_many_wave_launches_with_masks_and_splits(cuda_device, oracle_lib, Hq, Hkv, S, nsplit):
    """E4M3 launches of many waves (at least four waves of three CTAs per SM) on caches of
    at most 65,536 rows, for G <= 8 and for 8 < G <= 16 (each has its own shape there):
    ragged widths, interior -1 entries, an empty row, one split and forced splits; the
    oracle's fp8 path checks every 7th row plus the first and last."""
    Tq = 2400 if Hkv == 2 else 4000
    w = _random_case(470 + Hq, Tq, Hq, Hkv, S, 300, minus1=0.1, widths=True)
    w.slot_idx[5] = -1
    d = dev(w, cuda_device)
    got = run(w, d, 1.0 / 16.0, nsplit=nsplit)
    rows = sorted(set(range(0, Tq, 7)) | {1, 5, Tq - 1})
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, f"E4M3 many waves Hq={Hq} S={S} nsplit={nsplit}")
    assert torch.all(got[5] == 0)


def test_many_wave_two_tile_shape_block_and_shards(cuda_device, oracle_lib):
    """The E4M3 shape for 8 < G <= 16 in many-wave launches (one slot lane, six CTAs per
    SM) with block selection (block 4), and as context-parallel shards (R = 3, bf16
    records) stacked and combined: every 9th row plus the first and last against the
    oracle's fp8 path."""
    from test_parity_gpu import _shards_combined
    Tq, Hq, Hkv, S, W = 4000, 12, 1, 16384, 150
    w = _random_case(2900, Tq, Hq, Hkv, S, W, minus1=0.1, widths=True)
    w.slot_idx = wl.uniform_distinct(torch.Generator().manual_seed(2901), Tq, S // 4, W)
    w.slot_idx[torch.rand(Tq, W, generator=torch.Generator().manual_seed(2902)) < 0.1] = -1
    w.block = 4
    rows = sorted(set(range(0, Tq, 9)) | {Tq - 1})
    got = run(w, dev(w, cuda_device), 1.0 / 16.0)
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, "e4m3 two-tile many waves block4")
    got, _ = _shards_combined(w, dev(w, cuda_device), 3, k_scale=w.k_scale, v_scale=w.v_scale,
                              record_dtype=torch.bfloat16)
    compare(w, got, oracle_lib, 1.0 / 16.0, rows, "e4m3 two-tile many waves block4, 3 shards")
