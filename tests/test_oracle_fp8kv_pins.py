"""Pins for the oracle's fp8_e4m3 KV-cache path: checks against things other than itself.

The fp8_e4m3 cache is the format named in the article "Qwen4-Exp QSA comes to Huawei's
Ascend: inside SGLang's opt-in CANN prefill PR", section "Where this sits in the
Qwen4Exp serving build-out".  The reading: one E4M3 code per element and one float scale
per tensor, dequantised value = code value x scale, then the plain attention definition.

Pins:
  * the E4M3 decoder against hand-worked code values (tests/golden/e4m3_codes.json) and
    against torch's float8_e4m3fn conversion for all 256 codes (a library routine);
  * hand-worked forward cases (tests/golden/e4m3_forward_cases.json: weights 3/4 and 1/4
    from a ln 3 score gap, subnormal and negative codes with scales);
  * with power-of-two scales every dequantised element is exactly a bf16 value, so the
    fp8 path must reproduce the (separately pinned) bf16 oracle on those bf16 tensors;
  * float64 brute force on tiny inputs with general scales (decoded by torch);
  * closed forms: width 1 returns the dequantised V row; a zero query returns the mean
    of the dequantised V rows; v_scale scales the output linearly; all -1 returns +0;
  * block selection equals the slot-level call on the expanded slots;
  * the error bits of the slot-level definition.
A mutation test plants mistakes in the fp8 code of the oracle and checks that each one
fails at least one pin.
"""
from __future__ import annotations

import json
import math
from pathlib import Path

import numpy as np
import pytest
import torch

import oracle

D = 256
GOLDEN = Path(__file__).resolve().parent / "golden" / "e4m3_codes.json"


def _codes(gen, *shape, lo=0, hi=256):
    """Random E4M3 codes as a uint8 tensor, NaN codes (0x7F, 0xFF) excluded."""
    c = torch.randint(lo, hi, shape, generator=gen, dtype=torch.int64)
    c = torch.where((c & 0x7F) == 0x7F, c - 1, c)
    return c.to(torch.uint8)


def _decode_lib(codes: torch.Tensor) -> torch.Tensor:
    return codes.view(torch.float8_e4m3fn).to(torch.float64)


def _case(seed, Tq=5, Hq=4, Hkv=2, S=40, W=12, minus1=0.2):
    g = torch.Generator().manual_seed(seed)
    q = torch.randn(Tq, Hq, D, generator=g).to(torch.bfloat16)
    # codes of moderate magnitude (|value| <= 15) keep the scores O(1) for scale 1/16
    k = _codes(g, S, Hkv, D, hi=256)
    k = torch.where((k & 0x78) >= 0x58, k & 0x87, k)   # exponent field >= 11 -> small
    v = _codes(g, S, Hkv, D)
    idx = torch.stack([torch.randperm(S, generator=g)[:W] for _ in range(Tq)]).to(torch.int32)
    idx[torch.rand(Tq, W, generator=g) < minus1] = -1
    wd = torch.randint(0, W + 1, (Tq,), generator=g, dtype=torch.int32)
    return q, k, v, idx, wd


def _brute_fp64(q, kq, vq, idx, wd, scale, ks, vs):
    qd = q.to(torch.float64)
    kd = _decode_lib(kq) * ks
    vd = _decode_lib(vq) * vs
    Tq, Hq, _ = q.shape
    G = Hq // kq.shape[1]
    out = np.zeros((Tq, Hq, D))
    for t in range(Tq):
        w = idx.shape[1] if wd is None else int(wd[t])
        sel = [int(s) for s in idx[t, :w] if s >= 0]
        if not sel:
            continue
        for h in range(Hq):
            s = scale * (kd[sel, h // G] @ qd[t, h])
            p = torch.exp(s - s.max())
            out[t, h] = ((p[:, None] * vd[sel, h // G]).sum(0) / p.sum()).numpy()
    return out


# ------------------------------------------------------------------------------------
# Pin functions
# ------------------------------------------------------------------------------------

def pin_decode_golden(o):
    spec = json.loads(GOLDEN.read_text())
    codes = np.array([int(c["code"], 16) for c in spec["codes"]], dtype=np.uint8)
    got = o.decode_e4m3(codes)
    for c, g in zip(spec["codes"], got):
        if c["value"] == "nan":
            assert math.isnan(g), c
        else:
            assert g == c["value"] and math.copysign(1.0, g) == math.copysign(1.0, c["value"]), (c, g)


def pin_decode_library(o):
    codes = np.arange(256, dtype=np.uint8)
    got = o.decode_e4m3(codes)
    ref = torch.from_numpy(codes).view(torch.float8_e4m3fn).float().numpy()
    nan = np.isnan(ref)
    assert np.array_equal(np.isnan(got), nan)
    assert np.array_equal(got[~nan].view(np.uint32), ref[~nan].view(np.uint32))


def pin_matches_bf16_oracle(o):
    for seed, (Hq, Hkv) in enumerate([(4, 2), (16, 2), (12, 1), (3, 1)]):
        q, k, v, idx, wd = _case(300 + seed, Hq=Hq, Hkv=Hkv)
        for ks, vs in ((1.0, 1.0), (2.0 ** -4, 2.0 ** -3), (4.0, 0.5)):
            kb = (_decode_lib(k) * ks).to(torch.bfloat16)
            vb = (_decode_lib(v) * vs).to(torch.bfloat16)
            assert torch.equal(kb.double(), _decode_lib(k) * ks)   # exact in bf16
            got = o.forward_fp8kv(q, k, v, idx, wd, 1.0 / 16.0, ks, vs)
            ref = o.forward(q, kb, vb, idx, wd, 1.0 / 16.0)
            np.testing.assert_allclose(got, ref, rtol=1e-6, atol=1e-7)


def pin_brute_force(o):
    for seed, (Hq, Hkv) in enumerate([(4, 2), (16, 2), (6, 1)]):
        q, k, v, idx, wd = _case(400 + seed, Hq=Hq, Hkv=Hkv)
        for scale, ks, vs in ((1.0 / 16.0, 0.0135, 0.0125), (0.05, 0.3, 1.7), (0.2, 0.07, 0.01)):
            got = o.forward_fp8kv(q, k, v, idx, wd, scale, ks, vs)
            ref = _brute_fp64(q, k, v, idx, wd, scale, ks, vs)
            np.testing.assert_allclose(got, ref, rtol=2e-5, atol=2e-6 * max(vs * 448, 1.0))


def pin_closed_forms(o):
    q, k, v, idx, _ = _case(500, Tq=4, Hq=6, Hkv=2, S=30, W=8, minus1=0.0)
    G = 3
    ks, vs = 0.0135, 0.0125
    # width 1 -> the dequantised V row, exactly
    one = torch.ones(4, dtype=torch.int32)
    got = o.forward_fp8kv(q, k, v, idx, one, 0.7, ks, vs)
    for t in range(4):
        for h in range(6):
            ref = (_decode_lib(v[int(idx[t, 0]), h // G]).float() * np.float32(vs)).numpy()
            assert np.array_equal(got[t, h], ref)
    # zero query -> mean of the dequantised V rows
    got = o.forward_fp8kv(torch.zeros_like(q), k, v, idx, None, 1.0 / 16.0, ks, vs)
    for t in range(4):
        for h in range(6):
            ref = (_decode_lib(v[idx[t].long(), h // G]) * vs).mean(dim=0).numpy()
            np.testing.assert_allclose(got[t, h], ref, rtol=1e-5, atol=1e-6)
    # v_scale is a linear factor of the output (exact for a power of two)
    a = o.forward_fp8kv(q, k, v, idx, None, 1.0 / 16.0, ks, 0.25)
    b = o.forward_fp8kv(q, k, v, idx, None, 1.0 / 16.0, ks, 1.0)
    assert np.array_equal(a, b * np.float32(0.25))
    # k_scale multiplies the scores like the softmax scale does
    c = o.forward_fp8kv(q, k, v, idx, None, 0.125, 1.0, vs)
    d = o.forward_fp8kv(q, k, v, idx, None, 1.0, 0.125, vs)
    np.testing.assert_allclose(c, d, rtol=1e-5, atol=1e-6)
    # all -1 -> exact +0
    got = o.forward_fp8kv(q, k, v, torch.full_like(idx, -1), None, 1.0 / 16.0, ks, vs)
    assert np.all(got == 0) and not np.signbit(got).any()


def pin_block_selection(o):
    g = torch.Generator().manual_seed(510)
    q, k, v, _, _ = _case(511, Tq=4, Hq=8, Hkv=2, S=64, W=8)
    for block in (2, 4):
        nb = 64 // block
        idx = torch.stack([torch.randperm(nb, generator=g)[:6] for _ in range(4)]).to(torch.int32)
        idx[2, 1] = -1
        got = o.forward_fp8kv(q, k, v, idx, None, 0.0625, 0.0135, 0.0125, block=block)
        rows = [[int(b) * block + e for b in idx[t] if b >= 0 for e in range(block)] for t in range(4)]
        rows = [r + [-1] * (6 * block - len(r)) for r in rows]
        ref = o.forward_fp8kv(q, k, v, torch.tensor(rows, dtype=torch.int32), None, 0.0625,
                              0.0135, 0.0125)
        assert np.array_equal(got, ref)


def pin_error_flags(o):
    q, k, v, idx, _ = _case(520, Tq=3, Hq=2, Hkv=1, S=20, W=5, minus1=0.0)
    bad = idx.clone()
    bad[1, 2] = 20
    bad[2, 0] = -5
    got, err = o.forward_fp8kv(q, k, v, bad, None, 0.0625, 0.0135, 0.0125, return_err=True)
    assert err & 1
    clean = torch.where((bad >= 20) | (bad < -1), -1, bad)
    assert np.array_equal(got, o.forward_fp8kv(q, k, v, clean, None, 0.0625, 0.0135, 0.0125))
    _, err = o.forward_fp8kv(q, k, v, idx, torch.tensor([5, 6, 0], dtype=torch.int32), 0.0625,
                             0.0135, 0.0125, return_err=True)
    assert err & 2


FORWARD_GOLDEN = Path(__file__).resolve().parent / "golden" / "e4m3_forward_cases.json"
_SCALES = {"ln3": math.log(3.0), "ln2": math.log(2.0), "1": 1.0}


def load_forward_golden():
    """The hand-worked fp8 forward cases: bf16 q, E4M3 code caches, expected outputs."""
    spec = json.loads(FORWARD_GOLDEN.read_text())
    cases = []
    for c in spec["cases"]:
        Tq, Hq, Hkv, S = c["Tq"], c["Hq"], c["Hkv"], c["S"]
        q = torch.zeros(Tq, Hq, D)
        for t, h, d, val in c["q"]:
            q[t, h, d] = val
        kc = torch.zeros(S, Hkv, D, dtype=torch.uint8)
        for s_, j, d, code in c["k_codes"]:
            kc[s_, j, d] = int(code, 16)
        vc = torch.zeros(S, Hkv, D, dtype=torch.uint8)
        for s_, j, d, code in c["v_codes"]:
            vc[s_, j, d] = int(code, 16)
        exp = torch.zeros(Tq, Hq, D, dtype=torch.float64)
        for t, h, d, val in c["expected"]:
            exp[t, h, d] = val
        cases.append(dict(name=c["name"], q=q.to(torch.bfloat16), k=kc, v=vc,
                          slot_idx=torch.tensor(c["slot_idx"], dtype=torch.int32),
                          scale=_SCALES[c["scale"]], k_scale=c["k_scale"], v_scale=c["v_scale"],
                          expected=exp))
    return cases


def pin_forward_golden(o):
    for c in load_forward_golden():
        got = o.forward_fp8kv(c["q"], c["k"], c["v"], c["slot_idx"], None, c["scale"],
                              c["k_scale"], c["v_scale"])
        np.testing.assert_allclose(got, c["expected"].numpy(), rtol=0, atol=2e-6, err_msg=c["name"])
        empty = (c["expected"].abs().sum(dim=(1, 2)) == 0).nonzero().flatten().tolist()
        for t in empty:
            assert np.all(got[t] == 0) and not np.signbit(got[t]).any(), c["name"]


PINS = [pin_decode_golden, pin_decode_library, pin_forward_golden, pin_matches_bf16_oracle,
        pin_brute_force, pin_closed_forms, pin_block_selection, pin_error_flags]


@pytest.mark.parametrize("pin", PINS, ids=lambda f: f.__name__)
def test_fp8kv_oracle_pin(pin, oracle_lib):
    pin(oracle_lib)


MUTANTS = {
    "e4m3_bias_8": ("mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);",
                    "mag = ldexpf(1.0f + (float)m / 8.0f, e - 8);"),
    "e4m3_subnormal_as_normal": ("mag = ldexpf((float)m / 8.0f, 1 - 7);",
                                 "mag = ldexpf(1.0f + (float)m / 8.0f, 0 - 7);"),
    "e4m3_sign_ignored": ("return sign ? -mag : mag;", "return mag;"),
    "e4m3_mantissa_width": ("mag = ldexpf(1.0f + (float)m / 8.0f, e - 7);",
                            "mag = ldexpf(1.0f + (float)m / 16.0f, e - 7);"),
    "e4m3_nan_not_special": ("if (e == 15 && m == 7) return NAN;", ""),
    "kv_scales_swapped": ("kf[i * D + d] = e4m3_value(k_row[d]) * k_scale;",
                          "kf[i * D + d] = e4m3_value(k_row[d]) * v_scale;"),
    "v_scale_dropped": ("vf[i * D + d] = e4m3_value(v_row[d]) * v_scale;",
                        "vf[i * D + d] = e4m3_value(v_row[d]);"),
    "v_rows_from_k": ("const uint8_t* v_row = v_cache + sel[i] * v_stride_s + (int64_t)j * v_stride_h;",
                      "const uint8_t* v_row = k_cache + sel[i] * k_stride_s + (int64_t)j * k_stride_h;"),
    "block_offset_unscaled": ("for (int32_t e = 0; e < block; ++e) sel[n++] = (int64_t)b * block + e;",
                              "for (int32_t e = 0; e < block; ++e) sel[n++] = (int64_t)b + e;"),
    "group_heads_shifted": ("for (int32_t h = j * G; h < (j + 1) * G; ++h) {",
                            "for (int32_t h = j; h < Hq; h += Hkv) {"),
}


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_fp8kv_planted_mistake_is_caught(name, tmp_path):
    old, new = MUTANTS[name]
    src = oracle.SOURCE.read_text()
    assert src.count(old) == 1, f"mutation anchor must occur once: {old!r}"
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
