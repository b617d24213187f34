"""CPU oracle for selected-slot sparse attention (QSA prefill).

TEST INFRASTRUCTURE ONLY.  Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU
baseline leg of ``bench.py`` may import this package.  The CUDA library in
``top_sparse_attention_index_b200`` never imports it and shares no code with it.

The arithmetic lives in ``qsa_oracle.c`` (plain C, fp32, OpenMP over query rows) and
follows the article "Qwen4-Exp QSA comes to Huawei's Ascend: inside SGLang's opt-in
CANN prefill PR", section "What the pull request actually adds" (softmax(scale*QK^T)V
over the selected slots, -1 masked, fully masked rows zero) and section "Nine tests
that passed, ..." (FP32 CPU reference from the same BF16 inputs), plus block selection
and the fp8_e4m3 KV cache (sections "Why QSA is the awkward part, in numbers" and "Where
this sits in the Qwen4Exp serving build-out").  This module only compiles that file with
gcc and marshals numpy / torch CPU arrays into it.
"""
from __future__ import annotations

import ctypes
import subprocess
import sys
from pathlib import Path

import numpy as np

_HERE = Path(__file__).resolve().parent
SOURCE = _HERE / "qsa_oracle.c"
LIBRARY = _HERE / "libqsa_oracle.so"

GCC_FLAGS = ["-O2", "-std=c11", "-fPIC", "-shared", "-fopenmp", "-ffp-contract=off",
             "-fno-fast-math", "-Wall", "-Wextra"]


def build(source: Path | str = SOURCE, output: Path | str = LIBRARY, force: bool = False) -> Path:
    """Compile the oracle C file into a shared library (gcc, fp32, OpenMP)."""
    source, output = Path(source), Path(output)
    if not force and output.exists() and output.stat().st_mtime >= source.stat().st_mtime:
        return output
    cmd = ["gcc", *GCC_FLAGS, str(source), "-o", str(output), "-lm"]
    subprocess.run(cmd, check=True)
    return output


class Oracle:
    """ctypes wrapper around one compiled copy of the oracle library."""

    def __init__(self, library: Path | str | None = None):
        path = Path(library) if library is not None else build()
        self._lib = ctypes.CDLL(str(path))
        f = self._lib.qsa_oracle_forward
        f.restype = ctypes.c_int
        p, i64, i32 = ctypes.c_void_p, ctypes.c_int64, ctypes.c_int32
        f.argtypes = [p, i64, i64, p, i64, i64, p, i64, i64, p, i64, p,
                      i32, i32, i32, i32, i64, i32, ctypes.c_float, p, i64, p, p]
        fb = self._lib.qsa_oracle_forward_block
        fb.restype = ctypes.c_int
        fb.argtypes = [p, i64, i64, p, i64, i64, p, i64, i64, p, i64, p,
                       i32, i32, i32, i32, i64, i32, i32, ctypes.c_float, p, i64, p, p]
        f8 = self._lib.qsa_oracle_forward_fp8kv
        f8.restype = ctypes.c_int
        f8.argtypes = [p, i64, i64, p, i64, i64, p, i64, i64, p, i64, p,
                       i32, i32, i32, i32, i64, i32, i32, ctypes.c_float, ctypes.c_float,
                       ctypes.c_float, p, i64, p, p]
        dec = self._lib.qsa_oracle_decode_e4m3
        dec.restype = None
        dec.argtypes = [p, i64, p]
        self._lib.qsa_oracle_num_threads.restype = ctypes.c_int
        self.path = path

    def num_threads(self) -> int:
        return int(self._lib.qsa_oracle_num_threads())

    def forward(self, q, k_cache, v_cache, slot_idx, width=None, scale=1.0 / 16.0, rows=None,
                S=None, return_err=False, block=1):
        """fp32 oracle output for query rows ``rows`` (all rows when None).

        q: bf16 bits as uint16 array [Tq, Hq, D] (any strides, d contiguous) or a torch
        bf16 CPU tensor; k_cache / v_cache: [S, Hkv, D] likewise; slot_idx: int32
        [Tq, W] (row-strided, column-contiguous); width: int32 [Tq] or None.
        Returns float32 [len(rows) or Tq, Hq, D] (and the error bits when asked).
        With block > 1 every entry of slot_idx names `block` consecutive slots.
        """
        q, k_cache, v_cache = (_as_bf16_bits(x) for x in (q, k_cache, v_cache))
        slot_idx = _as_i32(slot_idx)
        Tq, Hq, D = q.shape
        S_, Hkv, Dk = k_cache.shape
        assert Dk == D and v_cache.shape == k_cache.shape
        S = S_ if S is None else S
        W = slot_idx.shape[1]
        for a in (q, k_cache, v_cache):
            assert a.strides[-1] == 2, "innermost dimension must be contiguous"
        assert slot_idx.strides[1] == 4
        if width is not None:
            width = np.ascontiguousarray(_as_i32(width))
            assert width.shape == (Tq,)
        if rows is not None:
            rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            nrows = rows.shape[0]
        else:
            nrows = Tq
        out = np.zeros((nrows, Hq, D), dtype=np.float32)
        err = ctypes.c_uint32(0)
        common = (q.ctypes.data, q.strides[0] // 2, q.strides[1] // 2,
                  k_cache.ctypes.data, k_cache.strides[0] // 2, k_cache.strides[1] // 2,
                  v_cache.ctypes.data, v_cache.strides[0] // 2, v_cache.strides[1] // 2,
                  slot_idx.ctypes.data, slot_idx.strides[0] // 4,
                  None if width is None else width.ctypes.data, Tq, Hq, Hkv, D, S, W)
        tail = (ctypes.c_float(scale), None if rows is None else rows.ctypes.data, nrows,
                out.ctypes.data, ctypes.byref(err))
        if block == 1:
            rc = self._lib.qsa_oracle_forward(*common, *tail)
        else:
            rc = self._lib.qsa_oracle_forward_block(*common, block, *tail)
        if rc != 0:
            raise ValueError("oracle rejected the sizes")
        return (out, int(err.value)) if return_err else out


    def decode_e4m3(self, codes) -> np.ndarray:
        """float32 values of E4M3 codes (uint8 array or float8_e4m3fn / uint8 tensor)."""
        c = np.ascontiguousarray(_as_u8(codes))
        out = np.empty(c.shape, dtype=np.float32)
        self._lib.qsa_oracle_decode_e4m3(c.ctypes.data, c.size, out.ctypes.data)
        return out

    def forward_fp8kv(self, q, k_cache, v_cache, slot_idx, width=None, scale=1.0 / 16.0,
                      k_scale=1.0, v_scale=1.0, rows=None, S=None, return_err=False, block=1):
        """fp32 oracle output with an fp8_e4m3 K/V cache.

        k_cache / v_cache: E4M3 codes [S, Hkv, D] as a uint8 array or a float8_e4m3fn /
        uint8 CPU tensor (d contiguous); a dequantised element is its code's value times
        k_scale (v_scale).  Everything else as ``forward``.
        """
        q = _as_bf16_bits(q)
        k_cache, v_cache = _as_u8(k_cache), _as_u8(v_cache)
        slot_idx = _as_i32(slot_idx)
        Tq, Hq, D = q.shape
        S_, Hkv, Dk = k_cache.shape
        assert Dk == D and v_cache.shape == k_cache.shape
        S = S_ if S is None else S
        W = slot_idx.shape[1]
        assert q.strides[-1] == 2 and k_cache.strides[-1] == 1 and v_cache.strides[-1] == 1
        assert slot_idx.strides[1] == 4
        if width is not None:
            width = np.ascontiguousarray(_as_i32(width))
            assert width.shape == (Tq,)
        if rows is not None:
            rows = np.ascontiguousarray(np.asarray(rows, dtype=np.int64))
            nrows = rows.shape[0]
        else:
            nrows = Tq
        out = np.zeros((nrows, Hq, D), dtype=np.float32)
        err = ctypes.c_uint32(0)
        rc = self._lib.qsa_oracle_forward_fp8kv(
            q.ctypes.data, q.strides[0] // 2, q.strides[1] // 2,
            k_cache.ctypes.data, k_cache.strides[0], k_cache.strides[1],
            v_cache.ctypes.data, v_cache.strides[0], v_cache.strides[1],
            slot_idx.ctypes.data, slot_idx.strides[0] // 4,
            None if width is None else width.ctypes.data, Tq, Hq, Hkv, D, S, W, block,
            ctypes.c_float(scale), ctypes.c_float(k_scale), ctypes.c_float(v_scale),
            None if rows is None else rows.ctypes.data, nrows, out.ctypes.data,
            ctypes.byref(err))
        if rc != 0:
            raise ValueError("oracle rejected the sizes")
        return (out, int(err.value)) if return_err else out


def _as_u8(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint8
        return x
    import torch
    assert isinstance(x, torch.Tensor) and x.device.type == "cpu"
    assert x.dtype in (torch.uint8, torch.float8_e4m3fn)
    return _strided_view(x.view(torch.uint8), np.uint8)


def _as_bf16_bits(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        assert x.dtype == np.uint16
        return x
    import torch  # local: torch is only needed for tensor inputs
    assert isinstance(x, torch.Tensor) and x.dtype == torch.bfloat16 and x.device.type == "cpu"
    return _strided_view(x.view(torch.int16), np.uint16)


def _as_i32(x) -> np.ndarray:
    if isinstance(x, np.ndarray):
        assert x.dtype == np.int32
        return x
    import torch
    assert isinstance(x, torch.Tensor) and x.dtype == torch.int32 and x.device.type == "cpu"
    return _strided_view(x, np.int32)


def _strided_view(t, dtype) -> np.ndarray:
    """numpy view of a (possibly non-contiguous) torch CPU tensor, same strides."""
    base = t.numpy() if t.is_contiguous() else None
    if base is not None:
        return base.view(dtype)
    itemsize = np.dtype(dtype).itemsize
    storage = t.untyped_storage()
    buf = (ctypes.c_char * storage.nbytes()).from_address(storage.data_ptr())
    arr = np.frombuffer(buf, dtype=dtype)
    return np.lib.stride_tricks.as_strided(
        arr[t.storage_offset():], shape=tuple(t.shape),
        strides=tuple(s * itemsize for s in t.stride()))


_default: Oracle | None = None


def default() -> Oracle:
    """The oracle built from the committed source (built on first use)."""
    global _default
    if _default is None:
        _default = Oracle()
    return _default


if __name__ == "__main__":  # python -m oracle [--force] : build the library
    print(build(force="--force" in sys.argv))
