"""B200-native (sm_100a) Top-K-selected sparse attention for QSA prefill.

The computation lives in libqsa.so (hand-written CUDA behind the C ABI in
include/qsa.h); this package is its thin Python binding plus seeded workload
generators.  Importing the package does not load the library; the first call does,
and raises if the library is missing (there is no CPU fallback).
"""
from ._binding import (  # noqa: F401
    QSA_ERR_CUDA,
    QSA_ERR_INVALID_ARG,
    QSA_ERR_UNSUPPORTED,
    QSA_ERR_WORKSPACE,
    QSA_ERRBIT_SLOT_RANGE,
    QSA_ERRBIT_Q_RANGE,
    QSA_ERRBIT_WIDTH_RANGE,
    QSA_MAX_BLOCK,
    QSA_MAX_SLOTS_PER_SPLIT,
    QSA_STATIC_SCRATCH_BYTES,
    QSA_OK,
    QSAError,
    load_library,
    qsa_abi_version,
    qsa_last_error_detail,
    qsa_sparse_prefill,
    qsa_sparse_prefill_block,
    qsa_combine_partials,
    qsa_probe_gather,
    qsa_probe_mma_operands,
    qsa_sparse_prefill_block_plan,
    qsa_sparse_prefill_fp8kv,
    qsa_sparse_prefill_partial,
    qsa_sparse_prefill_partial_plan,
    qsa_sparse_prefill_noalloc,
    qsa_sparse_prefill_plan,
    qsa_sparse_prefill_workspace_bytes,
    qsa_status_string,
    combine_partials,
    combine_peer_records,
    qsa_combine_peer_records,
    sparse_prefill,
    sparse_prefill_from_host,
    sparse_prefill_partial,
)
from .context_parallel import (  # noqa: F401
    PeerExchange,
    release_peer_exchanges,
    shard_ranges,
    sparse_prefill_context_parallel,
)

__all__ = [
    "sparse_prefill", "sparse_prefill_from_host", "qsa_sparse_prefill", "qsa_sparse_prefill_noalloc",
    "qsa_sparse_prefill_block", "qsa_sparse_prefill_block_plan", "qsa_sparse_prefill_fp8kv",
    "qsa_sparse_prefill_partial", "qsa_sparse_prefill_partial_plan", "qsa_combine_partials", "sparse_prefill_partial",
    "combine_partials", "sparse_prefill_context_parallel", "shard_ranges",
    "qsa_combine_peer_records", "combine_peer_records", "PeerExchange", "release_peer_exchanges",
    "qsa_sparse_prefill_plan", "qsa_sparse_prefill_workspace_bytes", "qsa_status_string", "qsa_last_error_detail", "qsa_abi_version",
    "load_library", "QSAError", "qsa_probe_gather", "qsa_probe_mma_operands",
]
