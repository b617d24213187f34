"""Test helpers: the golden closed-form cases, an independent float64 brute force, and
the parity gates.

The gates are the ones stated in the article "Qwen4-Exp QSA comes to Huawei's Ascend:
inside SGLang's opt-in CANN prefill PR", section "Nine tests that passed, and a speed
number that did not come from this branch": atol = 0.025, rtol = 0.025, relative L2
error below 0.008, empty rows exactly zero, every output finite.
"""
from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np
import torch

GOLDEN = Path(__file__).resolve().parent / "golden" / "closed_form_cases.json"

ATOL = 0.025
RTOL = 0.025
REL_L2_MAX = 0.008

_SCALES = {"ln3": math.log(3.0), "ln2": math.log(2.0), "1/16": 1.0 / 16.0}


def load_golden():
    """The hand-derived cases as dicts of CPU tensors (bf16 q/k/v, int32 indices)."""
    spec = json.loads(GOLDEN.read_text())
    D = spec["D"]
    cases = []
    for c in spec["cases"]:
        Tq, Hq, Hkv, S, W = c["Tq"], c["Hq"], c["Hkv"], c["S"], c["W"]
        q = torch.zeros(Tq, Hq, D)
        for t, h, d, val in c["q"]:
            q[t, h, d] = val
        k = torch.zeros(S, Hkv, D)
        for s, j, d, val in c["k"]:
            k[s, j, d] = val
        v = torch.zeros(S, Hkv, D)
        for s, j, d, val in c["v"]:
            v[s, j, d] = val
        exp = torch.zeros(Tq, Hq, D, dtype=torch.float64)
        for t, h, d, val in c["expected"]:
            exp[t, h, d] = val
        cases.append(dict(
            name=c["name"], q=q.to(torch.bfloat16), k=k.to(torch.bfloat16), v=v.to(torch.bfloat16),
            slot_idx=torch.tensor(c["slot_idx"], dtype=torch.int32),
            width=None if c["width"] is None else torch.tensor(c["width"], dtype=torch.int32),
            scale=_SCALES[c["scale"]], S=S, expected=exp))
    return cases


def brute_force_fp64(q, k, v, slot_idx, width, scale, S=None):
    """float64 numpy evaluation of the definition, one (t, h) at a time, for tiny inputs.
    Written independently of the C oracle (vectorised over slots with numpy)."""
    q = q.to(torch.float64).numpy()
    k = k.to(torch.float64).numpy()
    v = v.to(torch.float64).numpy()
    idx = slot_idx.numpy()
    Tq, Hq, D = q.shape
    S = k.shape[0] if S is None else S
    Hkv = k.shape[1]
    G = Hq // Hkv
    out = np.zeros((Tq, Hq, D))
    for t in range(Tq):
        wt = idx.shape[1] if width is None else int(width[t])
        sel = [int(s) for s in idx[t, :wt] if 0 <= s < S]
        if not sel:
            continue
        for h in range(Hq):
            kj = k[sel, h // G]          # [n, D]
            vj = v[sel, h // G]
            s = scale * (kj @ q[t, h])   # [n]
            p = np.exp(s - s.max())
            out[t, h] = (p @ vj) / p.sum()
    return out


def valid_counts(slot_idx: torch.Tensor, width, S: int) -> torch.Tensor:
    """Number of valid selected slots per query row (int64 [Tq])."""
    W = slot_idx.shape[1]
    pos = torch.arange(W)[None, :]
    wt = torch.full((slot_idx.shape[0], 1), W) if width is None else width.to(torch.int64)[:, None]
    ok = (pos < wt) & (slot_idx >= 0) & (slot_idx < S)
    return ok.sum(dim=1)


def check_gates(got: torch.Tensor, ref: torch.Tensor, empty_rows=None, label=""):
    """Apply the parity gates: elementwise |got-ref| <= ATOL + RTOL*|ref|, rel-L2 below
    REL_L2_MAX, all finite, and rows listed in empty_rows bitwise zero.  got/ref are
    [rows, Hq, D]; returns (max_abs_err, rel_l2)."""
    got = got.to(torch.float64)
    ref = ref.to(torch.float64)
    assert got.shape == ref.shape, (got.shape, ref.shape)
    assert torch.isfinite(got).all(), f"{label}: non-finite outputs"
    err = (got - ref).abs()
    bound = ATOL + RTOL * ref.abs()
    bad = err > bound
    if bad.any():
        i = bad.nonzero()[0].tolist()
        raise AssertionError(f"{label}: {int(bad.sum())} elements outside atol/rtol; first at "
                             f"{i}: got {got[tuple(i)].item()} ref {ref[tuple(i)].item()}")
    nref = ref.norm().item()
    rel = (got - ref).norm().item() / nref if nref > 0 else (0.0 if got.norm().item() == 0 else math.inf)
    assert rel < REL_L2_MAX, f"{label}: rel-L2 {rel:.5f} >= {REL_L2_MAX}"
    if empty_rows is not None and len(empty_rows):
        z = got[list(empty_rows)]
        assert (z == 0).all(), f"{label}: empty rows are not exactly zero"
    max_err = err.max().item() if err.numel() else 0.0
    print(f"PARITY {label}: rows={got.shape[0]} max_abs_err={max_err:.3e} rel_l2={rel:.3e}")
    return max_err, rel
