"""Seeded random shapes against the oracle: every kernel shape and path the launcher can
pick, on combinations the hand-written cases do not name.

Each case draws: KV heads (1, 2, 3, 4 or 8) and a group size G from 1 to 16; a cache of
up to ~140,000 slots (on both sides of the 65,536-row limit of the 16-bit row list); block
selection (1, 2, 4 or 16 slots per entry) or slot selection; a selection width up to
2,600 entries with masked entries and ragged per-row widths; bf16 or fp8_e4m3 caches;
the automatic split plan or a forced one; a strided Q view; a random scale.  The output
of every query row is compared with the CPU oracle at the parity gates, and rows with no
valid slot must be exactly zero.
"""
from __future__ import annotations

import pytest
import torch

import top_sparse_attention_index_b200 as qsa
from helpers import check_gates
from top_sparse_attention_index_b200 import workloads as wl

pytestmark = pytest.mark.gpu

D = 256
CASES = 24


def _draw(seed):
    g = torch.Generator().manual_seed(seed)
    ri = lambda lo, hi: int(torch.randint(lo, hi + 1, (1,), generator=g))  # noqa: E731
    rf = lambda: float(torch.rand(1, generator=g))  # noqa: E731
    Hkv = [1, 2, 3, 4, 8][ri(0, 4)]
    G = ri(1, 16)
    while G * Hkv > 48:
        G = ri(1, 16)
    Hq = G * Hkv
    S = [ri(16, 4096), ri(4097, 65536), ri(65537, 140000)][ri(0, 2)]
    while S * Hkv > 300000:          # host memory of the generated caches
        S //= 2
    block = [1, 1, 1, 1, 2, 4, 16][ri(0, 6)]
    n_ent = S // block
    if n_ent < 1:
        block, n_ent = 1, S
    W = min(ri(1, 2600), n_ent)
    budget = 4e9 / (Hq * 512.0)              # oracle work: Tq x W x block query-slot pairs
    Tq = max(1, min(ri(1, 200), int(budget / (W * block))))
    fp8 = rf() < 0.3
    nsplit = 0 if rf() < 0.7 else ri(1, 9)
    strided_q = rf() < 0.25
    scale = 0.03 + 0.07 * rf()
    minus1 = [0.0, 0.1, 0.5][ri(0, 2)]
    widths = rf() < 0.5
    q = torch.randn(Tq, 2 if strided_q else 1, Hq, D, generator=g).to(torch.bfloat16)[:, 0]
    k = torch.randn(S, Hkv, D, generator=g)
    v = torch.randn(S, Hkv, D, generator=g)
    idx = wl.uniform_distinct(g, Tq, n_ent, W)
    if minus1:
        idx[torch.rand(Tq, W, generator=g) < minus1] = -1
    if Tq > 2:
        idx[Tq // 2] = -1                                  # a fully masked row
    width = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32) if widths else None
    return dict(Tq=Tq, Hq=Hq, Hkv=Hkv, S=S, W=W, block=block, fp8=fp8, nsplit=nsplit,
                strided_q=strided_q, scale=scale, q=q, k=k, v=v, idx=idx, width=width)


def _empty_rows(c):
    W = c["idx"].shape[1]
    wt = torch.full((c["Tq"], 1), W) if c["width"] is None else c["width"].to(torch.int64)[:, None]
    ok = (torch.arange(W)[None, :] < wt) & (c["idx"] >= 0) & \
         ((c["idx"].to(torch.int64) + 1) * c["block"] <= c["S"])
    return (ok.sum(dim=1) == 0).nonzero().flatten().tolist()


@pytest.mark.parametrize("seed", range(7000, 7000 + CASES))
def test_random_shapes_match_oracle(cuda_device, oracle_lib, seed):
    c = _draw(seed)
    label = (f"seed {seed}: Tq={c['Tq']} Hq={c['Hq']} Hkv={c['Hkv']} S={c['S']} W={c['W']} "
             f"block={c['block']} fp8={c['fp8']} nsplit={c['nsplit']} strided_q={c['strided_q']}")
    if c["fp8"]:
        ks, vs = wl.E4M3_K_SCALE, wl.E4M3_V_SCALE
        k, v = wl.to_e4m3_cache(c["k"], ks), wl.to_e4m3_cache(c["v"], vs)
        ref = oracle_lib.forward_fp8kv(c["q"], k, v, c["idx"], c["width"], c["scale"], ks, vs,
                                       block=c["block"])
    else:
        ks = vs = 1.0
        k, v = c["k"].to(torch.bfloat16), c["v"].to(torch.bfloat16)
        ref = oracle_lib.forward(c["q"], k, v, c["idx"], c["width"], c["scale"], block=c["block"])
    if c["strided_q"]:
        base = c["q"].as_strided((c["Tq"], 2, c["Hq"], D), (2 * c["Hq"] * D, c["Hq"] * D, D, 1))
        q = base.to(cuda_device)[:, 0]
    else:
        q = c["q"].contiguous().to(cuda_device)
    err = torch.zeros(1, dtype=torch.int32, device=cuda_device)
    out = qsa.sparse_prefill(q, k.to(cuda_device), v.to(cuda_device), c["idx"].to(cuda_device),
                             None if c["width"] is None else c["width"].to(cuda_device),
                             scale=c["scale"], nsplit=c["nsplit"], block=c["block"],
                             k_scale=ks, v_scale=vs, err_word=err)
    torch.cuda.synchronize()
    assert int(err.item()) == 0, label
    check_gates(out.cpu().float(), torch.from_numpy(ref), _empty_rows(c), label)


@pytest.mark.parametrize("seed", range(7100, 7108))
def test_random_context_parallel_shards_match_oracle(cuda_device, oracle_lib, seed):
    """The same random draws split by slot range over 2-6 emulated ranks (shard boundaries
    on block multiples), bf16 or fp32 records, combined both ways: stacked (as after an
    all-gather) and through one pointer per record (as the peer exchange reads them).  The
    two combines agree bitwise; the result meets the gates against the whole-cache oracle."""
    c = _draw(seed)
    g = torch.Generator().manual_seed(seed + 1)
    R = int(torch.randint(2, 7, (1,), generator=g))
    rec = torch.bfloat16 if int(torch.randint(0, 2, (1,), generator=g)) else torch.float32
    label = (f"seed {seed}: R={R} {rec} Tq={c['Tq']} Hq={c['Hq']} Hkv={c['Hkv']} S={c['S']} "
             f"W={c['W']} block={c['block']} fp8={c['fp8']}")
    if c["fp8"]:
        ks, vs = wl.E4M3_K_SCALE, wl.E4M3_V_SCALE
        k, v = wl.to_e4m3_cache(c["k"], ks), wl.to_e4m3_cache(c["v"], vs)
        ref = oracle_lib.forward_fp8kv(c["q"], k, v, c["idx"], c["width"], c["scale"], ks, vs,
                                       block=c["block"])
    else:
        ks = vs = 1.0
        k, v = c["k"].to(torch.bfloat16), c["v"].to(torch.bfloat16)
        ref = oracle_lib.forward(c["q"], k, v, c["idx"], c["width"], c["scale"], block=c["block"])
    q = c["q"].contiguous().to(cuda_device)
    kd, vd, idx = k.to(cuda_device), v.to(cuda_device), c["idx"].to(cuda_device)
    width = None if c["width"] is None else c["width"].to(cuda_device)
    recs = [qsa.sparse_prefill_partial(q, kd[lo:hi], vd[lo:hi], idx, lo, c["S"], width=width,
                                       scale=c["scale"], block=c["block"], k_scale=ks,
                                       v_scale=vs, record_dtype=rec)
            for lo, hi in qsa.shard_ranges(c["S"], R, c["block"])]
    stacked = qsa.combine_partials(torch.stack([r[0] for r in recs]),
                                   torch.stack([r[1] for r in recs]))
    peer = torch.empty_like(stacked)
    qsa.combine_peer_records([r[0].data_ptr() for r in recs], [r[1].data_ptr() for r in recs],
                             rec, c["Tq"], c["Hq"], [peer])
    torch.cuda.synchronize()
    assert torch.equal(peer.view(torch.int16), stacked.view(torch.int16)), label
    check_gates(stacked.cpu().float(), torch.from_numpy(ref), _empty_rows(c), label)
