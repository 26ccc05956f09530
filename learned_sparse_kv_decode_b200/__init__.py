"""Lookahead Sparse Attention (LSA) decode step for B200 (sm_100a).

The chunk-scoring, top-k, gather and sparse flash-decode kernels live in
``liblsa_b200.so`` (sources in ``csrc/``, C ABI in ``include/lsa.h``);
``abi`` is the thin ctypes binding with the same entry-point names. The library
must be built (``learned_sparse_kv_decode_b200.build.build()``): there is no
fallback when it is missing.

Importing the package first brings the in-tree library up to date: a missing library, or one
older than its sources, is compiled with nvcc (no GPU needed); a current one is only
checked by modification time. Without nvcc and without a current library the import fails.
"""
from . import build as _build

_build.build()

from .abi import (  # noqa: E402,F401
    Dims, LsaError, alloc_workspace, header_symbols, lsa_abi_version, lsa_decode_step,
    lsa_gather_kv, lsa_get_device_status, lsa_score_chunks, lsa_sparse_decode_attn,
    lsa_topk_select, lsa_sparse_decode_attn_noalloc, lsa_refresh_resident,
    lsa_threshold_select, lsa_decode_step_threshold, lsa_indexer_score_fp8, lsa_decode_step_fp8,
    LSA_ENSEMBLE_MAX, LSA_ENSEMBLE_MEAN, LSA_INDEX_DIM, lsa_sparse_decode_attn_counts, lsa_shard_candidates,
    lsa_shard_global_select, lsa_merge_partials, lsa_read_stream, lsa_workspace_init, lsa_workspace_size, string,
    lsa_sparse_decode_attn_lookahead, lsa_decode_step_lookahead, lsa_lookahead_partition,
    LSA_OK, LSA_ERR_INVALID_ARG, LSA_ERR_WORKSPACE, LSA_ERR_CUDA, LSA_ERR_NONFINITE,
    LSA_ERR_TIMEOUT, LSA_ERR_UNSUPPORTED, LSA_ERR_BAD_ID, LSA_F32, LSA_BF16,
)
