"""The pages' size and time arithmetic, recomputed from their stated shapes.

* Indexer cache entry: 128 B fp8 key + 4 B scale = 132 B per compressed
  position; MLA latent KV entry 576 B ("03 long context", section "The
  Architectural Answer: Read Less of the Past").
* Per (query, key) indexer FLOPs = 2 * heads * 128 (same section: 16.4 KFLOP
  at 64 heads).
* LeanSparse: fp8 indexer keys at 512K tokens vs a 4K-entry hot KV buffer,
  "7.2 times the space" per indexed layer (podcast transcript, 02:59-03:30);
  the layer-streamed prefill loads history in about 2.9 ms at 32 GB/s
  (05:36-06:44 and 06:44-07:09), stride-4 CSA entries (02:36-02:56).
* LSA at 10M tokens ("Latent Sparse Attention", "The method, term by term",
  holding cost): 1,310,720 buckets, 64-d bf16 centroids, 16-slot int32 member
  tables, 2,621,440 GLM indexer keys of 128 B.
"""

from __future__ import annotations

KEY_BYTES = 128
SCALE_BYTES = 4
INDEXER_ENTRY_BYTES = KEY_BYTES + SCALE_BYTES  # 132
KV_ENTRY_BYTES = 576
CSA_STRIDE = 4
HOT_BUFFER_ENTRIES = 4096


def indexer_flops_per_pair(heads: int, d: int = 128) -> int:
    return 2 * heads * d


def indexer_bytes(tokens: int, stride: int = 1, entry: int = INDEXER_ENTRY_BYTES) -> int:
    return (tokens // stride) * entry


def key_to_hot_buffer_ratio(tokens: int, with_scale: bool = True) -> float:
    """Stride-4 fp8 indexer keys over a 4K-entry buffer of 576 B KV entries."""
    entry = INDEXER_ENTRY_BYTES if with_scale else KEY_BYTES
    return indexer_bytes(tokens, CSA_STRIDE, entry) / (HOT_BUFFER_ENTRIES * KV_ENTRY_BYTES)


def prefill_history_load_ms(tokens: int, gbps: float = 32.0) -> float:
    """One layer's stride-4 indexer keys plus compressed KV over the host link."""
    entries = tokens // CSA_STRIDE
    return entries * (INDEXER_ENTRY_BYTES + KV_ENTRY_BYTES) / (gbps * 1e9) * 1e3


def lsa_holding(tokens: int, block_keys: int = 512, block_buckets: int = 64, dim: int = 64,
                slots: int = 16):
    """LSA per-layer holding sizes: one index key per token, clustered in blocks
    of 512 keys into 64 buckets; GLM's indexer keeps one key per 4 tokens."""
    buckets = tokens // block_keys * block_buckets
    glm_keys = tokens // CSA_STRIDE
    return {
        "buckets": buckets,
        "centroid_bytes": buckets * dim * 2,
        "member_bytes": buckets * slots * 4,
        "glm_keys": glm_keys,
        "glm_key_bytes": glm_keys * KEY_BYTES,
    }
