"""B200 (sm_100a) lightning-indexer selection: Python binding of libls_indexer.so.

The binding only marshals arguments (torch tensors for device memory and the
current CUDA stream) into the library's C ABI (include/ls_indexer.h); every
step of the selection path runs in the library's CUDA kernels.  The library
is loaded on first use; a missing or stale libls_indexer.so raises
ImportError there (build it with `python -m
sparse_attention_indexer_lightning_b200.build`).  There is no fallback.
"""

from ._lib import (  # noqa: F401
    EXPORTED,
    LIB_PATH,
    LSError,
    ls_bucket_select,
    ls_decode_select,
    ls_decode_select_noalloc,
    ls_decode_two_stage_pq_select,
    ls_decode_two_stage_select,
    ls_device_status,
    ls_indexer_score,
    ls_indexer_score_fp8,
    ls_indexer_score_pq,
    ls_lsa_flat_select,
    ls_lsa_tree_levels_select,
    ls_lsa_tree_levels_workspace_size,
    ls_lsa_tree_select,
    ls_merge_select,
    ls_sparse_attention,
    ls_attention_merge,
    ls_prefill_select_stream,
    ls_prefill_select_stream_fp8,
    ls_profile_begin,
    ls_profile_end,
    ls_selftest_wait_probe,
    ls_topk_select,
    lib,
    shard_plan,
)
