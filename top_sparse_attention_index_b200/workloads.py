"""Seeded synthetic inputs for the QSA sparse-prefill workloads.

This module only draws random numbers and lays them out; it contains none of the
attention arithmetic.  Both the CUDA path (tests, bench) and the CPU oracle consume
exactly these tensors, so it is the one module the two sides share.

The shapes follow the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's
opt-in CANN prefill PR" (orcarouter.ai blog):
  * "What the pull request actually adds", head-shapes bullet: local (Q heads, KV heads)
    pairs (16,2), (24,2), (12,1), (6,1), (3,1); BF16; head dimension 256.
  * "Nine tests that passed, ...": widths 1/63/64/65/2051, fully masked rows, zero
    selection width, non-contiguous tensors, compression-ratio-4 causal tail remainders,
    two requests sharing a prefix mapped to the same physical slots, 1 and 257 query
    rows, and the long prefill of 7,810 queries x 2,051 slots over 65,536 cache slots.
  * sizing bullet: the referenced extent is capped at 262,144 tokens.
The article uses no dataset: every value here is N(0,1) noise cast to bf16 and every
selection is drawn uniformly (or with the stated locality), which stands in for the
indexer's Top-K output.

All generators are CPU ``torch.Generator`` based and deterministic given the seed
(default seed = 1234 + config number).
"""
from __future__ import annotations

from dataclasses import dataclass, field

import torch

D = 256
DEFAULT_SCALE = 1.0 / 16.0  # 1/sqrt(256): the original head-dim-256 scale


@dataclass
class Workload:
    name: str
    q: torch.Tensor            # bf16 [Tq, Hq, D] (possibly a strided view)
    k_cache: torch.Tensor      # bf16 [S, Hkv, D]
    v_cache: torch.Tensor      # bf16 [S, Hkv, D]
    slot_idx: torch.Tensor     # int32 [Tq, W]
    width: torch.Tensor | None  # int32 [Tq] or None (= W)
    scales: tuple = (DEFAULT_SCALE,)
    notes: dict = field(default_factory=dict)
    block: int = 1              # slots named by one entry of slot_idx (block selection)
    kv_format: str = "bf16"     # "bf16", or "e4m3": k_cache / v_cache hold float8_e4m3fn codes
    k_scale: float = 1.0        # dequantisation scales of an e4m3 cache
    v_scale: float = 1.0

    @property
    def Tq(self) -> int:
        return self.q.shape[0]

    @property
    def Hq(self) -> int:
        return self.q.shape[1]

    @property
    def Hkv(self) -> int:
        return self.k_cache.shape[1]

    @property
    def S(self) -> int:
        return self.k_cache.shape[0]

    @property
    def W(self) -> int:
        return self.slot_idx.shape[1]


def _normal_bf16(gen: torch.Generator, *shape) -> torch.Tensor:
    return torch.randn(*shape, generator=gen, dtype=torch.float32).to(torch.bfloat16)


def _qkv(gen, Tq, Hq, Hkv, S):
    q = _normal_bf16(gen, Tq, Hq, D)
    k = _normal_bf16(gen, S, Hkv, D)
    v = _normal_bf16(gen, S, Hkv, D)
    return q, k, v


def uniform_distinct(gen: torch.Generator, rows: int, S: int, W: int) -> torch.Tensor:
    """int32 [rows, W]: each row is W distinct slots drawn uniformly from [0, S), in the
    order they were drawn (already a uniformly random order).

    Sequential draws that reject repeats give a uniform random subset in a uniform
    random order; done here in bulk: draw a surplus of candidates per row, drop every
    candidate equal to an earlier one in the same row, keep the first W survivors.
    Rows left short (vanishingly rare) fall back to a random permutation."""
    assert 0 <= W <= S
    if W == 0:
        return torch.empty(rows, 0, dtype=torch.int32)
    if 4 * W > S:
        return torch.stack([torch.randperm(S, generator=gen)[:W] for _ in range(rows)]).to(torch.int32)
    out = torch.empty(rows, W, dtype=torch.int32)
    R = W + W // 4 + 64
    block = max(1, (1 << 22) // R)
    for r0 in range(0, rows, block):
        r1 = min(rows, r0 + block)
        cand = torch.randint(0, S, (r1 - r0, R), generator=gen, dtype=torch.int64)
        srt, order = torch.sort(cand, dim=1, stable=True)
        dup_sorted = torch.zeros_like(srt, dtype=torch.bool)
        dup_sorted[:, 1:] = srt[:, 1:] == srt[:, :-1]
        dup = torch.empty_like(dup_sorted)
        dup.scatter_(1, order, dup_sorted)
        keep = ~dup
        rank = torch.cumsum(keep.to(torch.int64), dim=1)
        ok = rank[:, -1] >= W
        sel = keep & (rank <= W)
        for i in range(r1 - r0):
            if ok[i]:
                out[r0 + i] = cand[i][sel[i]].to(torch.int32)
            else:
                out[r0 + i] = torch.randperm(S, generator=gen)[:W].to(torch.int32)
    return out


def _shuffle_rows(gen, idx: torch.Tensor) -> torch.Tensor:
    keys = torch.rand(idx.shape, generator=gen)
    return torch.gather(idx, 1, torch.argsort(keys, dim=1))


# --------------------------------------------------------------------------------------
# The five configurations.
# --------------------------------------------------------------------------------------

def tiny(seed: int = 1235) -> Workload:
    """Hq=16, Hkv=2, S=1,024, Tq=128, W=64 distinct unordered slots shared across KV
    heads; rows 0, 37, 64 and 127 are all -1 (must output exactly zero); scale 1/16."""
    gen = torch.Generator().manual_seed(seed)
    Tq, Hq, Hkv, S, W = 128, 16, 2, 1024, 64
    q, k, v = _qkv(gen, Tq, Hq, Hkv, S)
    idx = uniform_distinct(gen, Tq, S, W)
    for t in (0, 37, 64, 127):
        idx[t] = -1
    return Workload("tiny_hq16_hkv2_s1024_tq128_w64", q, k, v, idx, None,
                    notes={"masked_rows": [0, 37, 64, 127]})


WIDTH_CYCLE = (0, 1, 63, 64, 65, 2051)


def width_sweep(seed: int = 1236) -> Workload:
    """Hq=12, Hkv=1, S=4,096, Tq=257, W=2,051; width[t] cycles over 0/1/63/64/65/2051
    with -1 filling every entry past the width; every 5th non-empty row additionally has
    a quarter of its in-width entries replaced by interior -1s; Q is a non-contiguous
    view with row stride 2*Hq*D; run at scale 1/16 and 0.05."""
    gen = torch.Generator().manual_seed(seed)
    Tq, Hq, Hkv, S, W = 257, 12, 1, 4096, 2051
    q_full = _normal_bf16(gen, Tq, 2, Hq, D)
    q = q_full[:, 0]  # row stride 2*Hq*D elements
    k = _normal_bf16(gen, S, Hkv, D)
    v = _normal_bf16(gen, S, Hkv, D)
    width = torch.tensor([WIDTH_CYCLE[t % len(WIDTH_CYCLE)] for t in range(Tq)], dtype=torch.int32)
    idx = torch.full((Tq, W), -1, dtype=torch.int32)
    nonempty = 0
    interior_rows = []
    for t in range(Tq):
        wt = int(width[t])
        if wt == 0:
            continue
        idx[t, :wt] = torch.randperm(S, generator=gen)[:wt].to(torch.int32)
        if nonempty % 5 == 0 and wt >= 4:
            holes = torch.randperm(wt, generator=gen)[: wt // 4]
            idx[t, holes] = -1
            interior_rows.append(t)
        nonempty += 1
    return Workload("width_sweep_hq12_hkv1_s4096_tq257_w2051", q, k, v, idx, width,
                    scales=(DEFAULT_SCALE, 0.05), notes={"interior_minus1_rows": interior_rows})


def causal_two_request(seed: int = 1237, suffix_only: bool = False) -> Workload:
    """Hq=24, Hkv=2, S=12,288: two requests of 8,192 positions; request A maps position
    p to slot p, request B maps p < 4,096 to slot p (the shared prefix) and p >= 4,096 to
    slot 8,192 + (p - 4,096).  The query at position p selects min(2,051, p+1) slots:
    its last min(128, p+1) positions always, the rest uniformly without replacement from
    positions [0, p-128]; slot order shuffled; width[t] = the number selected and -1
    pads the row to W = 2,051.  Tq = 16,384 (both requests' full rows) unless
    suffix_only, where request B only prefills its 4,096-token suffix (Tq = 12,288)."""
    gen = torch.Generator().manual_seed(seed)
    Hq, Hkv, S, W, L, P = 24, 2, 12288, 2051, 8192, 4096
    rows = [(0, p) for p in range(L)] + [(1, p) for p in range(P if suffix_only else 0, L)]
    Tq = len(rows)
    q, k, v = _qkv(gen, Tq, Hq, Hkv, S)
    idx = torch.full((Tq, W), -1, dtype=torch.int32)
    width = torch.empty(Tq, dtype=torch.int32)
    for t, (r, p) in enumerate(rows):
        n_sel = min(W, p + 1)
        tail = min(128, p + 1)
        recent = torch.arange(p - tail + 1, p + 1, dtype=torch.int64)
        rest = n_sel - tail
        if rest > 0:
            older = torch.randperm(p - 127, generator=gen)[:rest]
            pos = torch.cat([recent, older])
        else:
            pos = recent
        pos = pos[torch.randperm(n_sel, generator=gen)]
        slot = pos if r == 0 else torch.where(pos < P, pos, pos - P + L)
        idx[t, :n_sel] = slot.to(torch.int32)
        width[t] = n_sel
    return Workload("causal_two_request_hq24_hkv2_s12288_tq%d_w2051" % Tq, q, k, v, idx, width,
                    notes={"rows": "A: 0..8191, B: %s" % ("4096..8191" if suffix_only else "0..8191")})


def long_prefill(seed: int = 1238) -> Workload:
    """The long-prefill case: Hq=16, Hkv=2, S=65,536, Tq=7,810, W=2,051 distinct
    unordered slots per row uniform over [0, S), shared across KV heads; scale 1/16."""
    gen = torch.Generator().manual_seed(seed)
    Tq, Hq, Hkv, S, W = 7810, 16, 2, 65536, 2051
    q, k, v = _qkv(gen, Tq, Hq, Hkv, S)
    idx = uniform_distinct(gen, Tq, S, W)
    return Workload("long_prefill_hq16_hkv2_s65536_tq7810_w2051", q, k, v, idx, None)


def long_prefill_block4(seed: int = 1244) -> Workload:
    """Block selection at the indexer's budget ("Why QSA is the awkward part, in
    numbers": 2,048 selected micro-blocks per query, compression ratio 4): Hq=16, Hkv=2,
    S=65,536, Tq=7,810, W=2,048 distinct blocks of 4 consecutive slots per row (8,192
    slots), uniform over the 16,384 blocks of the cache."""
    gen = torch.Generator().manual_seed(seed)
    Tq, Hq, Hkv, S, W, B = 7810, 16, 2, 65536, 2048, 4
    q, k, v = _qkv(gen, Tq, Hq, Hkv, S)
    idx = uniform_distinct(gen, Tq, S // B, W)
    return Workload("long_prefill_block4_hq16_hkv2_s65536_tq7810_w2048x4", q, k, v, idx, None,
                    block=B)


def max_extent(Hq: int = 6, clustered: bool = False, seed: int | None = None) -> Workload:
    """Hq=6 or 3 with Hkv=1, S=262,144, Tq=4,096, W=2,048.  Uniform: 2,048 distinct
    slots uniform over [0, S).  Clustered: 1,024 slots = the whole window
    [(t*64) mod S, +1,024) (mod S) plus 1,024 distinct uniform slots outside it,
    shuffled."""
    assert Hq in (6, 3)
    if seed is None:
        seed = 1239 + (0 if Hq == 6 else 10) + (1 if clustered else 0)
    gen = torch.Generator().manual_seed(seed)
    Tq, Hkv, S, W, WIN = 4096, 1, 262144, 2048, 1024
    q, k, v = _qkv(gen, Tq, Hq, Hkv, S)
    if not clustered:
        idx = uniform_distinct(gen, Tq, S, W)
    else:
        far = uniform_distinct(gen, Tq, S - WIN, W - WIN)  # positions relative to window end
        start = (torch.arange(Tq, dtype=torch.int64) * 64) % S
        window = (start[:, None] + torch.arange(WIN)[None, :]) % S
        outside = (start[:, None] + WIN + far.to(torch.int64)) % S
        idx = _shuffle_rows(gen, torch.cat([window, outside], dim=1)).to(torch.int32)
    return Workload("max_extent_hq%d_hkv1_s262144_tq4096_w2048_%s" % (Hq, "clustered" if clustered else "uniform"),
                    q, k, v, idx, None)


# --------------------------------------------------------------------------------------
# fp8_e4m3 KV cache ("Where this sits in the Qwen4Exp serving build-out": fp8_e4m3 is the
# KV-cache format that performed better for this attention's decode).
# --------------------------------------------------------------------------------------

# Per-tensor scales for N(0,1) data: |x| / scale stays below the largest finite E4M3
# magnitude (448) for |x| < 6, and the smallest |x| land in the subnormal codes.
E4M3_K_SCALE = 0.0135
E4M3_V_SCALE = 0.0125


def to_e4m3_cache(x: torch.Tensor, scale: float) -> torch.Tensor:
    """float8_e4m3fn codes of x / scale (round to nearest, clamped to +-448): how a KV
    writer stores a cache with one scale per tensor."""
    return (x.float() / scale).clamp(-448.0, 448.0).to(torch.float8_e4m3fn)


def with_e4m3_cache(w: Workload, k_scale: float = E4M3_K_SCALE,
                    v_scale: float = E4M3_V_SCALE) -> Workload:
    """The same workload with its K and V caches stored as E4M3 codes."""
    return Workload(w.name + "_e4m3kv", w.q, to_e4m3_cache(w.k_cache, k_scale),
                    to_e4m3_cache(w.v_cache, v_scale), w.slot_idx, w.width, scales=w.scales,
                    notes=dict(w.notes), block=w.block, kv_format="e4m3", k_scale=k_scale,
                    v_scale=v_scale)


def long_prefill_e4m3kv(seed: int = 1238) -> Workload:
    """The long-prefill case with an fp8_e4m3 K/V cache (the bf16 case's values, scaled
    by 1/0.0135 for K and 1/0.0125 for V and rounded to E4M3)."""
    return with_e4m3_cache(long_prefill(seed))


CONFIGS = {
    1: tiny,
    2: width_sweep,
    3: causal_two_request,
    4: long_prefill,
    5: max_extent,
}
