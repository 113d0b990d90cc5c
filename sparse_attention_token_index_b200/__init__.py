"""B200 (sm_100a) DSA lightning indexer: dense, group-shared (PIVOT) and decode.

A thin Python binding over the C ABI in ``include/dsa_index.h``
(``libdsa_index.so``, built in-tree by ``sparse_attention_token_index_b200.build``).
The functions here only marshal arguments: torch provides device memory and
the current CUDA stream; every step of the indexer runs in the library's
CUDA kernels.  There is no CPU path: without the library or a CUDA device
these functions raise.
"""
from __future__ import annotations

from ._binding import (  # noqa: F401
    DSA_DTYPE_BF16,
    DSA_DTYPE_FP32,
    DSA_DTYPE_FP8_E4M3,
    DSA_GROUP_REFINE,
    DSA_GROUP_REUSE,
    DSA_GROUP_REFINE_LOCAL,
    DsaError,
    lib,
    lib_path,
    dsa_index_dense,
    dsa_index_group,
    dsa_index_decode,
    dsa_index_decode_group,
    dsa_index_block_routed,
    dsa_ivf_build,
    dsa_index_ivf_routed,
    IvfIndex,
    dsa_debug_scores,
    dsa_index_dense_static,
    dsa_index_dense_host,
    dsa_index_group_host,
    dsa_index_decode_host,
    dense_host_staging_bytes,
    group_host_staging_bytes,
    decode_host_staging_bytes,
    dsa_kernel_timer_start,
    dsa_kernel_timer_stop,
    dsa_check_status,
    dsa_debug_set_wait,
    dense_workspace_bytes,
    group_workspace_bytes,
    decode_workspace_bytes,
    decode_group_workspace_bytes,
    block_routed_workspace_bytes,
    ivf_routed_workspace_bytes,
    EXPORTED_SYMBOLS,
)
