"""Pins for the CPU oracle: checks against things other than itself.

Each pin is a plain function taking an ``oracle.Oracle`` so that the mutation test at
the bottom can run the same pins against copies of the oracle with a planted mistake.

Pins (the article, "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in CANN
prefill PR", prints no worked example, so the pins are closed forms, a library routine,
the article's packed-embedding identity and brute force):
  * hand-derived closed-form cases stored under tests/golden/;
  * dense special case: selecting every slot equals dense attention computed by
    torch.nn.functional.scaled_dot_product_attention (float64, GQA);
  * permutation invariance of the slot order, with -1s interleaved;
  * the packed-embedding identity of section "What the pull request actually adds":
    softmax(scale * Q' C^T) C = [P K, P V] with C = [K, V] and Q' = [Q, 0];
  * closed forms: width 1 returns v[slot] exactly; a zero query row returns the mean of
    the valid V rows; equal K rows return the mean of V; all -1 or width 0 returns +0;
    a very large scale returns the V row of the best-scoring slot;
  * float64 brute force on tiny random inputs.
"""
from __future__ import annotations

import math
import re
import subprocess
from pathlib import Path

import numpy as np
import pytest
import torch
import torch.nn.functional as F

import oracle
from helpers import brute_force_fp64, load_golden
from top_sparse_attention_index_b200 import workloads as wl

D = 256


def _rand_case(seed, Tq=6, Hq=4, Hkv=2, S=40, W=12, minus1=0.2, width=True):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    idx = torch.stack([torch.randperm(S, generator=g)[:W] for _ in range(Tq)]).to(torch.int32)
    idx[torch.rand(Tq, W, generator=g) < minus1] = -1
    wd = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32) if width else None
    return q, k, v, idx, wd


# ------------------------------------------------------------------------------------
# Pin functions (raise AssertionError on failure)
# ------------------------------------------------------------------------------------

def pin_golden(o):
    for c in load_golden():
        got = o.forward(c["q"], c["k"], c["v"], c["slot_idx"], c["width"], c["scale"], S=c["S"])
        np.testing.assert_allclose(got, c["expected"].numpy(), rtol=0, atol=2e-6, err_msg=c["name"])
        empty = (c["expected"].abs().sum(dim=(1, 2)) == 0).nonzero().flatten().tolist()
        for t in empty:
            assert np.all(got[t] == 0) and not np.signbit(got[t]).any(), c["name"]


def pin_brute_force(o):
    for seed, (Hq, Hkv) in enumerate([(4, 2), (16, 2), (12, 1), (6, 1), (3, 1), (24, 2)]):
        q, k, v, idx, wd = _rand_case(100 + seed, Hq=Hq, Hkv=Hkv)
        for scale in (1.0 / 16.0, 0.05, 0.3):
            got = o.forward(q, k, v, idx, wd, scale)
            ref = brute_force_fp64(q, k, v, idx, wd, scale)
            np.testing.assert_allclose(got, ref, rtol=2e-5, atol=2e-6)


def pin_dense_sdpa(o):
    g = torch.Generator().manual_seed(7)
    for Hq, Hkv, S, Tq in [(16, 2, 64, 5), (12, 1, 33, 3), (24, 2, 17, 2)]:
        q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
        k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
        v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
        idx = torch.stack([torch.randperm(S, generator=g) for _ in range(Tq)]).to(torch.int32)
        scale = 1.0 / 16.0
        got = o.forward(q, k, v, idx, None, scale)
        qd = q.to(torch.float64).permute(1, 0, 2)[None]      # [1, Hq, Tq, D]
        kd = k.to(torch.float64).permute(1, 0, 2)[None]      # [1, Hkv, S, D]
        vd = v.to(torch.float64).permute(1, 0, 2)[None]
        ref = F.scaled_dot_product_attention(qd, kd, vd, scale=scale, enable_gqa=True)
        ref = ref[0].permute(1, 0, 2).numpy()
        np.testing.assert_allclose(got, ref, rtol=2e-5, atol=2e-6)


def pin_permutation_invariance(o):
    g = torch.Generator().manual_seed(11)
    q, k, v, idx, _ = _rand_case(12, Tq=8, Hq=8, Hkv=1, S=300, W=200, minus1=0.0, width=False)
    base = o.forward(q, k, v, idx, None, 1.0 / 16.0)
    # shuffle each row and interleave -1s (the width grows to hold them)
    W2 = 260
    idx2 = torch.full((idx.shape[0], W2), -1, dtype=torch.int32)
    for t in range(idx.shape[0]):
        pos = torch.randperm(W2, generator=g)[:200].sort().values
        idx2[t, pos] = idx[t, torch.randperm(200, generator=g)]
    got = o.forward(q, k, v, idx2, None, 1.0 / 16.0)
    np.testing.assert_allclose(got, base, rtol=1e-5, atol=1e-6)


def pin_packed_identity(o):
    """softmax(scale * Q' C^T) C with C = [K, V] (512 wide) and Q' = [Q, 0] returns
    [P K, P V]: the V half must equal the oracle, the K half the oracle run with V := K."""
    q, k, v, idx, wd = _rand_case(21, Tq=8, Hq=8, Hkv=2, S=64, W=16)
    scale = 1.0 / 16.0
    G = q.shape[1] // k.shape[1]
    got_v = o.forward(q, k, v, idx, wd, scale)
    got_k = o.forward(q, k, k, idx, wd, scale)
    qd, kd, vd = q.double(), k.double(), v.double()
    for t in range(q.shape[0]):
        sel = [int(s) for s in idx[t, : int(wd[t])] if s >= 0]
        for h in range(q.shape[1]):
            if not sel:
                assert np.all(got_v[t, h] == 0) and np.all(got_k[t, h] == 0)
                continue
            C = torch.cat([kd[sel, h // G], vd[sel, h // G]], dim=1)         # [n, 512]
            Qp = torch.cat([qd[t, h], torch.zeros(D, dtype=torch.float64)])   # [512]
            P = torch.softmax(scale * (C @ Qp), dim=0)
            PC = P @ C
            np.testing.assert_allclose(got_v[t, h], PC[D:].numpy(), rtol=2e-5, atol=2e-6)
            np.testing.assert_allclose(got_k[t, h], PC[:D].numpy(), rtol=2e-5, atol=2e-6)


def pin_closed_forms(o):
    g = torch.Generator().manual_seed(31)
    S, Hq, Hkv, Tq, W = 50, 6, 2, 5, 9
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    G = Hq // Hkv
    # width 1 -> exactly v[slot]
    idx = torch.stack([torch.randperm(S, generator=g)[:W] for _ in range(Tq)]).to(torch.int32)
    one = torch.ones(Tq, dtype=torch.int32)
    got = o.forward(q, k, v, idx, one, 0.7)
    for t in range(Tq):
        for h in range(Hq):
            assert np.array_equal(got[t, h], v[int(idx[t, 0]), h // G].float().numpy())
    # zero query rows -> mean of the valid V rows
    qz = torch.zeros_like(q)
    idxm = idx.clone()
    idxm[:, 3] = -1
    got = o.forward(qz, k, v, idxm, None, 1.0 / 16.0)
    for t in range(Tq):
        sel = [int(s) for s in idxm[t] if s >= 0]
        for h in range(Hq):
            ref = v[sel, h // G].double().mean(dim=0).numpy()
            np.testing.assert_allclose(got[t, h], ref, rtol=1e-5, atol=1e-6)
    # all K rows equal -> mean of V
    ke = k[:1].expand(S, Hkv, D).clone()
    got = o.forward(q, ke, v, idx, None, 1.0 / 16.0)
    for t in range(Tq):
        for h in range(Hq):
            ref = v[idx[t].long(), h // G].double().mean(dim=0).numpy()
            np.testing.assert_allclose(got[t, h], ref, rtol=1e-5, atol=1e-6)
    # all -1, and width 0 -> exact +0
    allm = torch.full_like(idx, -1)
    got = o.forward(q, k, v, allm, None, 1.0 / 16.0)
    assert np.all(got == 0) and not np.signbit(got).any()
    got = o.forward(q, k, v, idx, torch.zeros(Tq, dtype=torch.int32), 1.0 / 16.0)
    assert np.all(got == 0) and not np.signbit(got).any()
    # very large scale -> the V row of the best-scoring slot (hard-max limit), finite
    got = o.forward(q, k, v, idx, None, 1000.0)
    assert np.isfinite(got).all()
    for t in range(Tq):
        for h in range(Hq):
            sc = k[idx[t].long(), h // G].double() @ q[t, h].double()
            top2 = torch.topk(sc, 2).values
            if float(top2[0] - top2[1]) * 1000.0 < 50:   # skip near-ties
                continue
            best = int(idx[t, int(torch.argmax(sc))])
            np.testing.assert_allclose(got[t, h], v[best, h // G].float().numpy(), rtol=1e-6, atol=1e-6)


def pin_error_flags(o):
    q, k, v, idx, _ = _rand_case(41, Tq=3, Hq=2, Hkv=1, S=20, W=5, minus1=0.0, width=False)
    bad = idx.clone()
    bad[1, 2] = 20      # == S: out of range
    bad[2, 0] = -7      # below -1
    got, err = o.forward(q, k, v, bad, None, 1.0 / 16.0, return_err=True)
    assert err & 1
    ref = o.forward(q, k, v, torch.where((bad >= 20) | (bad < -1), -1, bad), None, 1.0 / 16.0)
    assert np.array_equal(got, ref)
    wd = torch.tensor([5, 9, -1], dtype=torch.int32)
    got, err = o.forward(q, k, v, idx, wd, 1.0 / 16.0, return_err=True)
    assert err & 2
    ref = o.forward(q, k, v, idx, torch.tensor([5, 5, 0], dtype=torch.int32), 1.0 / 16.0)
    assert np.array_equal(got, ref)


def pin_block_selection(o):
    """Block selection: each entry b names slots b*block .. b*block+block-1.  Expanded
    here with numpy and compared with the slot-level oracle; a zero query over one block
    gives the mean of its V rows; a block reaching past S is masked and flagged."""
    g = torch.Generator().manual_seed(51)
    S, Hq, Hkv, Tq, W = 64, 8, 2, 6, 7
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    k = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    v = torch.randn(S, Hkv, D, generator=g).to(torch.bfloat16)
    for block in (2, 4):
        nb = S // block
        idx = torch.stack([torch.randperm(nb, generator=g)[:W] for _ in range(Tq)]).to(torch.int32)
        idx[1, 3] = -1
        wd = torch.tensor([7, 7, 0, 3, 1, 7], dtype=torch.int32)
        got = o.forward(q, k, v, idx, wd, 0.0625, block=block)
        rows = []
        for t in range(Tq):
            sl = [int(b) * block + e for b in idx[t, : int(wd[t])] if b >= 0 for e in range(block)]
            rows.append(sl + [-1] * (W * block - len(sl)))
        ref = o.forward(q, k, v, torch.tensor(rows, dtype=torch.int32), None, 0.0625)
        assert np.array_equal(got, ref)
        one = torch.tensor([[5] + [-1] * (W - 1)] * Tq, dtype=torch.int32)
        got = o.forward(torch.zeros_like(q), k, v, one, None, 0.0625, block=block)
        for h in range(Hq):
            mean = v[5 * block: 6 * block, h // (Hq // Hkv)].double().mean(dim=0).numpy()
            np.testing.assert_allclose(got[0, h], mean, rtol=1e-5, atol=1e-6)
        past = one.clone()
        past[:, 1] = nb          # the block starting at S: out of range
        got2, err = o.forward(q, k, v, past, None, 0.0625, block=block, return_err=True)
        assert err & 1
        assert np.array_equal(got2, o.forward(q, k, v, one, None, 0.0625, block=block))


PINS = [pin_golden, pin_brute_force, pin_dense_sdpa, pin_permutation_invariance,
        pin_packed_identity, pin_closed_forms, pin_error_flags, pin_block_selection]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


def test_oracle_strided_inputs_match_contiguous(oracle_lib):
    """The width-sweep workload's non-contiguous Q view gives the same result as a
    contiguous copy (strides are honoured)."""
    w = wl.width_sweep()
    assert not w.q.is_contiguous()
    rows = list(range(0, w.Tq, 7))
    a = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, w.width, 0.05, rows=rows)
    b = oracle_lib.forward(w.q.contiguous(), w.k_cache, w.v_cache, w.slot_idx, w.width, 0.05, rows=rows)
    assert np.array_equal(a, b)


def test_oracle_row_subset(oracle_lib):
    w = wl.tiny()
    full = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0)
    rows = [5, 0, 127, 64, 3]
    sub = oracle_lib.forward(w.q, w.k_cache, w.v_cache, w.slot_idx, None, 1.0 / 16.0, rows=rows)
    assert np.array_equal(sub, full[rows])
    for t in w.notes["masked_rows"]:
        assert np.all(full[t] == 0)


# ------------------------------------------------------------------------------------
# Planted mistakes: each mutant copy of the oracle must fail at least one pin.
# ------------------------------------------------------------------------------------

MUTANTS = {
    "wrong_head_map": ("const int32_t j = h / G;", "const int32_t j = h % Hkv;"),
    "dropped_scale": ("scratch_s[i] = scale * acc;", "scratch_s[i] = acc;"),
    "dropped_normalisation": ("out_row[d] = out_row[d] / l;", "out_row[d] = out_row[d];"),
    "width_ignored": ("int32_t width_t = width ? width[t] : W;", "int32_t width_t = W;"),
    "minus1_as_slot0": ("if (slot == -1) continue;", "if (slot == -1) slot = 0;"),
    "k_for_v_transposed_operand": (
        "const uint16_t* k_row = k_cache + scratch_i[i] * k_stride_s + (int64_t)j * k_stride_h;",
        "const uint16_t* k_row = v_cache + scratch_i[i] * v_stride_s + (int64_t)j * v_stride_h;"),
    "sign_flip_in_exponent": ("scratch_s[i] = expf(scratch_s[i] - m);", "scratch_s[i] = expf(m - scratch_s[i]);"),
    "max_not_subtracted": ("scratch_s[i] = expf(scratch_s[i] - m);", "scratch_s[i] = expf(scratch_s[i]);"),
    "off_by_one_width": ("for (int32_t w = 0; w < width_t; ++w) {", "for (int32_t w = 0; w + 1 < width_t; ++w) {"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.SOURCE.read_text()
    assert src.count(old) >= 1, f"mutation anchor not found: {old!r}"
    mutant_src = tmp_path / "qsa_oracle_mutant.c"
    mutant_src.write_text(src.replace(old, new))
    lib = oracle.build(mutant_src, tmp_path / "libqsa_oracle_mutant.so", force=True)
    mutant = oracle.Oracle(lib)
    failed = []
    with np.errstate(all="ignore"):
        for pin in PINS:
            try:
                pin(mutant)
            except AssertionError:
                failed.append(pin.__name__)
    assert failed, f"mutant {name} passed every pin"
