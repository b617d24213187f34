"""ctypes binding of libqsa.so: argument marshalling only.

Every step of the computation runs in the CUDA kernels behind the C ABI declared in
include/qsa.h; this module converts torch tensors into pointers, strides and the
current CUDA stream, and turns status codes into exceptions.  There is no fallback:
if the library is missing or a GPU is absent, the calls raise.
"""
from __future__ import annotations

import ctypes
from pathlib import Path

import torch

LIBRARY = Path(__file__).resolve().parent / "libqsa.so"

QSA_OK = 0
QSA_ERR_INVALID_ARG = 1
QSA_ERR_UNSUPPORTED = 2
QSA_ERR_WORKSPACE = 3
QSA_ERR_CUDA = 4
QSA_ERRBIT_SLOT_RANGE = 0x1
QSA_ERRBIT_WIDTH_RANGE = 0x2
QSA_ERRBIT_Q_RANGE = 0x4
QSA_MAX_SLOTS_PER_SPLIT = 2240
QSA_MAX_BLOCK = 16
QSA_STATIC_SCRATCH_BYTES = 16 << 20
QSA_MAX_PEERS = 16
QSA_IPC_HANDLE_BYTES = 64

# Every symbol include/qsa.h declares, with its ctypes signature (restype, argtypes).
_p, _i32, _i64, _sz, _f = ctypes.c_void_p, ctypes.c_int32, ctypes.c_int64, ctypes.c_size_t, ctypes.c_float
SIGNATURES = {
    "qsa_abi_version": (_i32, []),
    "qsa_sparse_prefill_plan": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, ctypes.POINTER(_sz)]),
    "qsa_sparse_prefill_workspace_bytes": (_sz, [_i32, _i32, _i32, _i32, _i32, _i32]),
    "qsa_sparse_prefill": (_i32, [_p, _i64, _i64, _p, _i64, _i64, _p, _i64, _i64, _p, _i64, _p,
                                  _i32, _i32, _i32, _i32, _i64, _i32, _f, _p, _i64, _i64, _i32,
                                  _p, _sz, _p, _p]),
    "qsa_sparse_prefill_block_plan": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i32, _i32,
                                             ctypes.POINTER(_sz)]),
    "qsa_sparse_prefill_block": (_i32, [_p, _i64, _i64, _p, _i64, _i64, _p, _i64, _i64, _p, _i64,
                                        _p, _i32, _i32, _i32, _i32, _i64, _i32, _i32, _f, _p, _i64,
                                        _i64, _i32, _p, _sz, _p, _p]),
    "qsa_sparse_prefill_fp8kv": (_i32, [_p, _i64, _i64, _p, _i64, _i64, _p, _i64, _i64, _p, _i64,
                                        _p, _i32, _i32, _i32, _i32, _i64, _i32, _i32, _f, _f, _f,
                                        _p, _i64, _i64, _i32, _p, _sz, _p, _p]),
    "qsa_sparse_prefill_partial": (_i32, [_p, _i64, _i64, _p, _i64, _i64, _p, _i64, _i64, _p,
                                          _i64, _p, _i32, _i32, _i32, _i32, _i64, _i32, _i32,
                                          _i64, _i64, _i32, _f, _f, _f, _p, _p, _i32, _i32, _p,
                                          _sz, _p, _p]),
    "qsa_sparse_prefill_partial_plan": (_i32, [_i32, _i32, _i32, _i32, _i32, _i32, _i64, _i64,
                                               _i32, _i32, ctypes.POINTER(_sz)]),
    "qsa_combine_partials": (_i32, [_p, _p, _i32, _i32, _i32, _i32, _i32, _p, _i64, _i64, _p]),
    "qsa_sparse_prefill_noalloc": (_i32, [_p, _i64, _i64, _p, _i64, _i64, _p, _i64, _i64, _p,
                                          _i64, _p, _i32, _i32, _i32, _i32, _i64, _i32, _f, _p,
                                          _i64, _i64, _i32, _p, _p]),
    "qsa_probe_gather": (_i32, [_i32, _i32, _p, _i64, _i64, _i32, _i32, _i32, _i32, _i32,
                                ctypes.c_uint32, _p, _p]),
    "qsa_probe_mma_operands": (_i32, [_i32, _i32, _i32, _i32, _p, _p]),
    "qsa_combine_peer_records": (_i32, [ctypes.POINTER(_p), ctypes.POINTER(_p), _i32, _i32, _i32,
                                        _i32, _i32, _i32, _i32, ctypes.POINTER(_p), _i32, _i64,
                                        _i64, _p]),
    "qsa_ipc_export": (_i32, [_p, _p, ctypes.POINTER(ctypes.c_uint64)]),
    "qsa_ipc_import": (_i32, [_p, ctypes.POINTER(_p)]),
    "qsa_ipc_close": (_i32, [_p]),
    "qsa_status_string": (ctypes.c_char_p, [_i32]),
    "qsa_last_error_detail": (ctypes.c_char_p, []),
}


class QSAError(RuntimeError):
    def __init__(self, status: int, detail: str):
        super().__init__(f"{qsa_status_string(status)}: {detail}")
        self.status = status


_lib = None


def load_library(path: Path | str | None = None):
    """Load libqsa.so (built in-tree by build_lib.py); raises if it is missing."""
    global _lib
    if _lib is not None and path is None:
        return _lib
    path = Path(path) if path is not None else LIBRARY
    if not path.exists():
        raise RuntimeError(f"{path} is missing: build it with "
                           "`python -m top_sparse_attention_index_b200.build_lib`")
    lib = ctypes.CDLL(str(path))
    for name, (res, args) in SIGNATURES.items():
        fn = getattr(lib, name)
        fn.restype = res
        fn.argtypes = args
    if path == LIBRARY:
        _lib = lib
    return lib


# ---- names of the C ABI -------------------------------------------------------------

def qsa_abi_version() -> int:
    return int(load_library().qsa_abi_version())


def qsa_status_string(status: int) -> str:
    return load_library().qsa_status_string(int(status)).decode()


def qsa_last_error_detail() -> str:
    return load_library().qsa_last_error_detail().decode()


def qsa_sparse_prefill_plan(Tq, Hq, Hkv, D, W, num_sms, nsplit_request=0):
    """(nsplit, workspace_bytes) for this shape; raises QSAError for invalid shapes."""
    ws = ctypes.c_size_t(0)
    n = int(load_library().qsa_sparse_prefill_plan(Tq, Hq, Hkv, D, W, num_sms, nsplit_request,
                                                   ctypes.byref(ws)))
    if n < 0:
        raise QSAError(-n, qsa_last_error_detail())
    return n, int(ws.value)


def qsa_sparse_prefill_workspace_bytes(Tq, Hq, Hkv, W, D, num_sms) -> int:
    """Workspace bytes of the automatic plan; raises QSAError for invalid shapes."""
    n = int(load_library().qsa_sparse_prefill_workspace_bytes(Tq, Hq, Hkv, W, D, num_sms))
    if n == ctypes.c_size_t(-1).value:
        qsa_sparse_prefill_plan(Tq, Hq, Hkv, D, W, num_sms)  # raises with the status
        raise QSAError(QSA_ERR_INVALID_ARG, qsa_last_error_detail())
    return n


def qsa_probe_gather(method, read_back, src, rows, pitch_bytes, row_bytes, warps_per_cta, stages,
                     ctas, iters, seed, sink, stream) -> int:
    """Raw call of the gather-rate probe (include/qsa_probe.h); returns the status code."""
    return int(load_library().qsa_probe_gather(method, read_back, src, rows, pitch_bytes,
                                               row_bytes, warps_per_cta, stages, ctas, iters,
                                               seed, sink, stream))


def qsa_probe_mma_operands(method, n, rounds, ctas, out, stream) -> int:
    """Raw call of the MMA operand-rate probe (include/qsa_probe.h); returns the status."""
    return int(load_library().qsa_probe_mma_operands(method, n, rounds, ctas, out, stream))


def qsa_sparse_prefill(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                       v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S,
                       W, scale, out, out_stride_t, out_stride_h, nsplit, workspace,
                       workspace_bytes, err_word, stream) -> int:
    """Raw call with integer pointers; returns the status code unchanged."""
    return int(load_library().qsa_sparse_prefill(
        q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache, v_stride_s,
        v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W, ctypes.c_float(scale),
        out, out_stride_t, out_stride_h, nsplit, workspace, workspace_bytes, err_word, stream))


def qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, D, W, block, num_sms, nsplit_request=0):
    """(nsplit, workspace_bytes) for block selection; raises QSAError for invalid shapes."""
    ws = ctypes.c_size_t(0)
    n = int(load_library().qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, D, W, block, num_sms,
                                                         nsplit_request, ctypes.byref(ws)))
    if n < 0:
        raise QSAError(-n, qsa_last_error_detail())
    return n, int(ws.value)


def qsa_sparse_prefill_block(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                             v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv,
                             D, S, W, block, scale, out, out_stride_t, out_stride_h, nsplit,
                             workspace, workspace_bytes, err_word, stream) -> int:
    """Raw call of block selection (each entry names `block` consecutive slots)."""
    return int(load_library().qsa_sparse_prefill_block(
        q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache, v_stride_s,
        v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W, block,
        ctypes.c_float(scale), out, out_stride_t, out_stride_h, nsplit, workspace,
        workspace_bytes, err_word, stream))


def qsa_sparse_prefill_fp8kv(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache,
                             v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv,
                             D, S, W, block, scale, k_scale, v_scale, out, out_stride_t,
                             out_stride_h, nsplit, workspace, workspace_bytes, err_word,
                             stream) -> int:
    """Raw call with an E4M3 K/V cache (strides in bytes) and its two scales."""
    return int(load_library().qsa_sparse_prefill_fp8kv(
        q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache, v_stride_s,
        v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W, block,
        ctypes.c_float(scale), ctypes.c_float(k_scale), ctypes.c_float(v_scale), out,
        out_stride_t, out_stride_h, nsplit, workspace, workspace_bytes, err_word, stream))


def qsa_sparse_prefill_partial(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h,
                               v_cache, v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq,
                               Hq, Hkv, D, S, W, block, slot_lo, S_total, kv_fp8, scale, k_scale,
                               v_scale, part_o, part_lse, record_bf16, nsplit, workspace,
                               workspace_bytes, err_word, stream) -> int:
    """Raw call of one slot-range shard's partial record (context parallelism)."""
    return int(load_library().qsa_sparse_prefill_partial(
        q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache, v_stride_s,
        v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W, block, slot_lo, S_total,
        kv_fp8, ctypes.c_float(scale), ctypes.c_float(k_scale), ctypes.c_float(v_scale), part_o,
        part_lse, record_bf16, nsplit, workspace, workspace_bytes, err_word, stream))


def qsa_sparse_prefill_partial_plan(Tq, Hq, Hkv, D, W, block, S, S_total, num_sms,
                                    nsplit_request=0):
    """(nsplit, workspace_bytes) of a slot-range shard's call; raises QSAError for invalid
    shapes."""
    ws = ctypes.c_size_t(0)
    n = int(load_library().qsa_sparse_prefill_partial_plan(Tq, Hq, Hkv, D, W, block, S, S_total,
                                                           num_sms, nsplit_request,
                                                           ctypes.byref(ws)))
    if n < 0:
        raise QSAError(-n, qsa_last_error_detail())
    return n, int(ws.value)


def qsa_combine_partials(part_o, part_lse, record_bf16, R, Tq, Hq, D, out, out_stride_t,
                         out_stride_h, stream) -> int:
    """Raw call of the log-sum-exp combine of R stacked partial records."""
    return int(load_library().qsa_combine_partials(part_o, part_lse, record_bf16, R, Tq, Hq, D,
                                                   out, out_stride_t, out_stride_h, stream))


def qsa_sparse_prefill_noalloc(q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h,
                               v_cache, v_stride_s, v_stride_h, slot_idx, idx_stride_t, width, Tq,
                               Hq, Hkv, D, S, W, scale, out, out_stride_t, out_stride_h, nsplit,
                               err_word, stream) -> int:
    """Raw call of the entry point that takes its split scratch from the library's static
    device array instead of a caller workspace; returns the status code unchanged."""
    return int(load_library().qsa_sparse_prefill_noalloc(
        q, q_stride_t, q_stride_h, k_cache, k_stride_s, k_stride_h, v_cache, v_stride_s,
        v_stride_h, slot_idx, idx_stride_t, width, Tq, Hq, Hkv, D, S, W, ctypes.c_float(scale),
        out, out_stride_t, out_stride_h, nsplit, err_word, stream))


# ---- torch-facing wrapper ------------------------------------------------------------

def _ptr(t):
    return None if t is None else t.data_ptr()


def _check_dev(name, t, dtype, device):
    if t.device != device:
        raise ValueError(f"{name} must live on {device}, got {t.device}")
    if t.dtype != dtype:
        raise ValueError(f"{name} must be {dtype}, got {t.dtype}")
    if t.dim() > 0 and t.shape[-1] > 1 and t.stride(-1) != 1:
        raise ValueError(f"{name} must be contiguous in its last dimension")


def sparse_prefill(q, k_cache, v_cache, slot_idx, width=None, scale=None, out=None, nsplit=0,
                   err_word=None, stream=None, block=1, k_scale=1.0, v_scale=1.0):
    """Selected-slot sparse attention on the GPU.

    q [Tq, Hq, 256] bf16, k_cache / v_cache [S, Hkv, 256] bf16, slot_idx [Tq, W] int32
    (-1 = masked), width [Tq] int32 or None; scale defaults to 1/sqrt(256) = 1/16.
    Returns out [Tq, Hq, 256] bf16 (allocated unless given).  Work is enqueued on
    ``stream`` (default: torch's current stream); nothing is synchronised.  With
    block > 1 every entry of slot_idx names `block` consecutive slots.  K/V caches of
    dtype float8_e4m3fn are an fp8_e4m3 cache dequantised as code value x k_scale
    (x v_scale); the scales are ignored for bf16 caches.
    """
    device = q.device
    if device.type != "cuda":
        raise ValueError("sparse_prefill runs on CUDA tensors only")
    Tq, Hq, D = q.shape
    S, Hkv, Dk = k_cache.shape
    if Dk != D or tuple(v_cache.shape) != (S, Hkv, D):
        raise ValueError("k_cache and v_cache must both be [S, Hkv, D]")
    if slot_idx.dim() != 2 or slot_idx.shape[0] != Tq:
        raise ValueError("slot_idx must be [Tq, W]")
    W = slot_idx.shape[1]
    kv_fp8 = k_cache.dtype == torch.float8_e4m3fn
    kv_dt = torch.float8_e4m3fn if kv_fp8 else torch.bfloat16
    for name, t, dt in (("q", q, torch.bfloat16), ("k_cache", k_cache, kv_dt),
                        ("v_cache", v_cache, kv_dt), ("slot_idx", slot_idx, torch.int32)):
        _check_dev(name, t, dt, device)
    if width is not None:
        _check_dev("width", width, torch.int32, device)
        if tuple(width.shape) != (Tq,) or (Tq > 1 and width.stride(0) != 1):
            raise ValueError("width must be a contiguous [Tq] int32 tensor")
    if out is None:
        out = torch.empty(Tq, Hq, D, dtype=torch.bfloat16, device=device)
    else:
        _check_dev("out", out, torch.bfloat16, device)
        if tuple(out.shape) != (Tq, Hq, D):
            raise ValueError("out must be [Tq, Hq, D]")
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    num_sms = torch.cuda.get_device_properties(device).multi_processor_count
    ns, ws_bytes = qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, D, W, block, num_sms, nsplit)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device) if ws_bytes else None
    with torch.cuda.device(device):
        head = (_ptr(q), q.stride(0), q.stride(1), _ptr(k_cache), k_cache.stride(0), k_cache.stride(1),
                _ptr(v_cache), v_cache.stride(0), v_cache.stride(1), _ptr(slot_idx) if W else None,
                slot_idx.stride(0), _ptr(width), Tq, Hq, Hkv, D, S, W, block, float(scale))
        tail = (_ptr(out), out.stride(0), out.stride(1), ns, _ptr(ws), ws_bytes, _ptr(err_word),
                stream.cuda_stream)
        if kv_fp8:
            st = qsa_sparse_prefill_fp8kv(*head, float(k_scale), float(v_scale), *tail)
        else:
            st = qsa_sparse_prefill_block(*head, *tail)
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())
    return out


def sparse_prefill_partial(q, k_cache, v_cache, slot_idx, slot_lo, S_total, width=None,
                           scale=None, part_o=None, part_lse=None, nsplit=0, err_word=None,
                           stream=None, block=1, k_scale=1.0, v_scale=1.0,
                           record_dtype=torch.float32, compact=True):
    """One device's partial record for a cache split by slot range (context parallel).

    k_cache / v_cache hold the global slots [slot_lo, slot_lo + S) of a cache of S_total
    slots (bf16, or float8_e4m3fn codes with k_scale / v_scale); slot_idx holds global
    slot numbers.  Returns (part_o [Tq, Hq, 256] of record_dtype (float32 or bfloat16),
    part_lse fp32 [Tq, Hq]): the output normalised over this device's valid slots and the
    base-2 log-sum-exp of their scaled scores (-inf where there are none).  Combine the
    records of all devices with combine_partials.  compact=True gives the call the
    workspace in which it first gathers each row's local entries (same result, fewer
    entries for the fused kernel to scan); False gives it only the split workspace.
    """
    device = q.device
    if device.type != "cuda":
        raise ValueError("sparse_prefill_partial runs on CUDA tensors only")
    Tq, Hq, D = q.shape
    S, Hkv, Dk = k_cache.shape
    if Dk != D or tuple(v_cache.shape) != (S, Hkv, D):
        raise ValueError("k_cache and v_cache must both be [S, Hkv, D]")
    if slot_idx.dim() != 2 or slot_idx.shape[0] != Tq:
        raise ValueError("slot_idx must be [Tq, W]")
    W = slot_idx.shape[1]
    kv_fp8 = k_cache.dtype == torch.float8_e4m3fn
    kv_dt = torch.float8_e4m3fn if kv_fp8 else torch.bfloat16
    for name, t, dt in (("q", q, torch.bfloat16), ("k_cache", k_cache, kv_dt),
                        ("v_cache", v_cache, kv_dt), ("slot_idx", slot_idx, torch.int32)):
        _check_dev(name, t, dt, device)
    if width is not None:
        _check_dev("width", width, torch.int32, device)
    if record_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("record_dtype must be torch.float32 or torch.bfloat16")
    if part_o is None:
        part_o = torch.empty(Tq, Hq, D, dtype=record_dtype, device=device)
    if part_lse is None:
        part_lse = torch.empty(Tq, Hq, dtype=torch.float32, device=device)
    for name, t, shape, dt in (("part_o", part_o, (Tq, Hq, D), record_dtype),
                               ("part_lse", part_lse, (Tq, Hq), torch.float32)):
        if tuple(t.shape) != shape or t.dtype != dt or not t.is_contiguous() or t.device != device:
            raise ValueError(f"{name} must be a contiguous {dt} {shape} tensor on {device}")
    if scale is None:
        scale = 1.0 / (D ** 0.5)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    num_sms = torch.cuda.get_device_properties(device).multi_processor_count
    if compact:
        ns, ws_bytes = qsa_sparse_prefill_partial_plan(Tq, Hq, Hkv, D, W, block, S,
                                                       int(S_total), num_sms, nsplit)
    else:
        ns, ws_bytes = qsa_sparse_prefill_block_plan(Tq, Hq, Hkv, D, W, block, num_sms, nsplit)
    ws = torch.empty(max(ws_bytes, 1), dtype=torch.uint8, device=device) if ws_bytes else None
    with torch.cuda.device(device):
        st = qsa_sparse_prefill_partial(
            _ptr(q), q.stride(0), q.stride(1), _ptr(k_cache), k_cache.stride(0), k_cache.stride(1),
            _ptr(v_cache), v_cache.stride(0), v_cache.stride(1), _ptr(slot_idx) if W else None,
            slot_idx.stride(0), _ptr(width), Tq, Hq, Hkv, D, S, W, block, int(slot_lo),
            int(S_total), 1 if kv_fp8 else 0, float(scale), float(k_scale), float(v_scale),
            _ptr(part_o), _ptr(part_lse), 1 if record_dtype == torch.bfloat16 else 0, ns,
            _ptr(ws), ws_bytes, _ptr(err_word), stream.cuda_stream)
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())
    return part_o, part_lse


def combine_partials(part_o, part_lse, out=None, stream=None):
    """bf16 [Tq, Hq, 256]: the log-sum-exp combine of R stacked partial records
    (part_o float32 or bfloat16 [R, Tq, Hq, 256], part_lse float32 [R, Tq, Hq], both
    contiguous)."""
    device = part_o.device
    if device.type != "cuda":
        raise ValueError("combine_partials runs on CUDA tensors only")
    if part_o.dim() != 4 or part_lse.shape != part_o.shape[:3]:
        raise ValueError("part_o must be [R, Tq, Hq, D] and part_lse [R, Tq, Hq]")
    R, Tq, Hq, D = part_o.shape
    if part_o.dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("part_o must be float32 or bfloat16")
    for name, t in (("part_o", part_o), ("part_lse", part_lse)):
        dt = part_o.dtype if name == "part_o" else torch.float32
        if t.dtype != dt or not t.is_contiguous() or t.device != device:
            raise ValueError(f"{name} must be a contiguous {dt} tensor on {device}")
    if out is None:
        out = torch.empty(Tq, Hq, D, dtype=torch.bfloat16, device=device)
    else:
        _check_dev("out", out, torch.bfloat16, device)
    if stream is None:
        stream = torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        st = qsa_combine_partials(_ptr(part_o), _ptr(part_lse),
                                  1 if part_o.dtype == torch.bfloat16 else 0, R, Tq, Hq, D,
                                  _ptr(out), out.stride(0), out.stride(1), stream.cuda_stream)
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())
    return out


# ---- records addressed one pointer each (include/qsa_peer.h) --------------------------

def _ptr_array(ptrs):
    arr = (ctypes.c_void_p * len(ptrs))()
    for i, v in enumerate(ptrs):
        arr[i] = int(v)
    return arr


def qsa_combine_peer_records(rec_o, rec_lse, R, record_bf16, Tq, Hq, D, t0, t1, out, n_out,
                             out_stride_t, out_stride_h, stream) -> int:
    """Raw call: rec_o, rec_lse and out are sequences of integer device pointers (the
    host arrays of the C call); returns the status code."""
    return int(load_library().qsa_combine_peer_records(
        _ptr_array(rec_o), _ptr_array(rec_lse), R, record_bf16, Tq, Hq, D, t0, t1,
        _ptr_array(out), n_out, out_stride_t, out_stride_h, stream))


def combine_peer_records(rec_o_ptrs, rec_lse_ptrs, record_dtype, Tq, Hq, outs, t0=0, t1=None,
                         stream=None, device=None):
    """The log-sum-exp combine of R records given as device pointers (this device's memory
    or peer memory mapped into this process), rows [t0, t1) stored as bf16 to every tensor
    in `outs` (bf16 [Tq, Hq, 256] tensors, or (pointer, stride_t, stride_h) triples that
    share the strides of the first).  Returns nothing; the work is enqueued on `stream`."""
    device = torch.device(device) if device is not None else None
    t1 = Tq if t1 is None else t1
    if record_dtype not in (torch.float32, torch.bfloat16):
        raise ValueError("record_dtype must be torch.float32 or torch.bfloat16")
    if len(rec_o_ptrs) != len(rec_lse_ptrs):
        raise ValueError("one O pointer and one lse pointer per record")
    out_ptrs, strides = [], None
    for o in outs:
        if isinstance(o, torch.Tensor):
            _check_dev("out", o, torch.bfloat16, o.device)
            if tuple(o.shape) != (Tq, Hq, 256):
                raise ValueError("every out must be [Tq, Hq, 256]")
            device = device or o.device
            st = (o.stride(0), o.stride(1))
            out_ptrs.append(_ptr(o))
        else:
            ptr, st_t, st_h = o
            st = (st_t, st_h)
            out_ptrs.append(int(ptr))
        if strides is not None and st != strides:
            raise ValueError("every out must have the same strides")
        strides = st
    if strides is None:
        raise ValueError("at least one out")
    if device is None:
        device = torch.device("cuda", torch.cuda.current_device())
    if stream is None:
        stream = torch.cuda.current_stream(device)
    with torch.cuda.device(device):
        st = qsa_combine_peer_records(rec_o_ptrs, rec_lse_ptrs, len(rec_o_ptrs),
                                      1 if record_dtype == torch.bfloat16 else 0, Tq, Hq, 256,
                                      t0, t1, out_ptrs, len(out_ptrs), strides[0], strides[1],
                                      stream.cuda_stream)
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())


def ipc_export(t: torch.Tensor):
    """(handle bytes, byte offset) that let another process map the memory of `t`."""
    h = ctypes.create_string_buffer(QSA_IPC_HANDLE_BYTES)
    off = ctypes.c_uint64(0)
    with torch.cuda.device(t.device):
        st = int(load_library().qsa_ipc_export(_ptr(t), h, ctypes.byref(off)))
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())
    return h.raw, int(off.value)


def ipc_import(handle: bytes, device) -> int:
    """Maps another process's exported allocation on `device`; returns its base pointer."""
    if len(handle) != QSA_IPC_HANDLE_BYTES:
        raise ValueError("an IPC handle is %d bytes" % QSA_IPC_HANDLE_BYTES)
    base = ctypes.c_void_p(0)
    with torch.cuda.device(device):
        st = int(load_library().qsa_ipc_import(ctypes.create_string_buffer(handle, len(handle)),
                                               ctypes.byref(base)))
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())
    return int(base.value)


def ipc_close(base: int, device) -> None:
    with torch.cuda.device(device):
        st = int(load_library().qsa_ipc_close(ctypes.c_void_p(base)))
    if st != QSA_OK:
        raise QSAError(st, qsa_last_error_detail())


_COPY_STREAMS = {}


def _copy_streams(device):
    """The two side streams of the host-buffer path, one pair per device, created once:
    reusing them lets the caching allocator recycle the staging buffers of earlier
    calls instead of allocating (and synchronising) anew."""
    key = torch.device(device).index if torch.device(device).index is not None else torch.cuda.current_device()
    if key not in _COPY_STREAMS:
        _COPY_STREAMS[key] = (torch.cuda.Stream(key), torch.cuda.Stream(key))
    return _COPY_STREAMS[key]


def sparse_prefill_from_host(q, k_cache, v_cache, slot_idx, width=None, scale=None, out=None,
                             device=None, chunk_rows=None, nsplit=0, block=1, k_scale=1.0,
                             v_scale=1.0):
    """Host-buffer form of sparse_prefill: copies the inputs to `device`, runs the kernels
    and copies the result back, overlapping the transfers with the computation.

    Inputs are CPU tensors (pinned memory makes the copies asynchronous); the result is
    written to `out` (a CPU bf16 [Tq, Hq, 256] tensor, allocated pinned when None) and
    is complete when the returned CUDA event has completed (``event.synchronize()``).
    K and V are copied first (every query row may read any slot); then query rows go in
    chunks of `chunk_rows`: chunk c+1's Q and indices cross the bus while chunk c is
    computed and chunk c-1's output returns on a third stream.  With nsplit = 0 every
    chunk uses the split plan of the whole batch, so the result is bitwise that of
    sparse_prefill on the whole batch when the chunks launch the same kernel shape (a
    launch of fewer waves may take another shape, which changes only the order of the
    sums).
    """
    device = torch.device(device if device is not None else "cuda")
    if device.type != "cuda":
        raise ValueError("sparse_prefill_from_host needs a CUDA device")
    Tq, Hq, D = q.shape
    if out is None:
        out = torch.empty(Tq, Hq, D, dtype=torch.bfloat16).pin_memory()
    if chunk_rows is None:
        # eight chunks: measured best for the long prefill (5.46 ms; 16 chunks 5.61, four
        # 5.83; chunks shrinking towards the end were slower still)
        chunk_rows = max(-(-Tq // 8), 256)
    if nsplit == 0:
        # every chunk uses the whole batch's split plan (the kernel shape of a launch
        # may still differ with its size, which changes only the order of the sums)
        num_sms = torch.cuda.get_device_properties(device).multi_processor_count
        nsplit, _ = qsa_sparse_prefill_block_plan(Tq, Hq, k_cache.shape[1], D, slot_idx.shape[1],
                                                  block, num_sms, 0)
    h2d, d2h = _copy_streams(device)
    comp = torch.cuda.current_stream(device)
    h2d.wait_stream(comp)  # ordered after work already queued on the caller's stream
    with torch.cuda.device(device):
        with torch.cuda.stream(h2d):
            k_d = k_cache.to(device, non_blocking=True)
            v_d = v_cache.to(device, non_blocking=True)
            kv_ready = torch.cuda.Event()
            kv_ready.record(h2d)
        out_d = torch.empty(Tq, Hq, D, dtype=torch.bfloat16, device=device)
        comp.wait_event(kv_ready)
        done = None
        for r0 in range(0, max(Tq, 1), chunk_rows):
            r1 = min(Tq, r0 + chunk_rows)
            with torch.cuda.stream(h2d):
                q_c = q[r0:r1].to(device, non_blocking=True)
                i_c = slot_idx[r0:r1].to(device, non_blocking=True)
                w_c = None if width is None else width[r0:r1].to(device, non_blocking=True)
                ready = torch.cuda.Event()
                ready.record(h2d)
            comp.wait_event(ready)
            # the chunk's device buffers were allocated on h2d and are used on comp
            for t in (q_c, i_c, w_c):
                if t is not None:
                    t.record_stream(comp)
            sparse_prefill(q_c, k_d, v_d, i_c, w_c, scale=scale, out=out_d[r0:r1], nsplit=nsplit,
                           stream=comp, block=block, k_scale=k_scale, v_scale=v_scale)
            done = torch.cuda.Event()
            done.record(comp)
            d2h.wait_event(done)
            with torch.cuda.stream(d2h):
                out[r0:r1].copy_(out_d[r0:r1], non_blocking=True)
        for t in (k_d, v_d):
            t.record_stream(comp)
        out_d.record_stream(d2h)
        finished = torch.cuda.Event()
        finished.record(d2h)
    return out, finished
