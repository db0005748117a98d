"""Shapes of the indexer workloads.

Five full-size workloads follow the shapes the pages use:

* ``decode_tiny``   -- 4 sequences x 8192 tokens (2048 stride-4 compressed
  positions), one query each.
* ``decode_batch``  -- 64 sequences x 131072 tokens (32768 positions each).
* ``prefill_chunk`` -- one 4096-query chunk at token positions
  126976..131071 against 131072 history tokens (32768 positions), history
  streamed in 8192-key tiles through two device buffers (LeanSparse podcast
  transcript, 05:36-06:44).
* ``prefill_chunk_fp8`` -- the same chunk with fp8 e4m3 queries (one scale
  per query head) and an fp8 history (one scale per key), quantised from the
  same draws: the indexer's FP8 form ("03 long context" lecture, section
  "Sparsity Is a Systems Feature: The Blast Radius", kernel layer).
* ``two_stage``     -- 32 sequences x 524288 tokens (131072 positions each):
  compact int8 scan, 4096-entry shortlist, exact re-rank of fp8 originals
  (LeanSparse podcast transcript, 07:12-08:00).
* ``lsa_flat``      -- the native LSA flat search over one sequence of
  1048576 tokens: 131072 buckets (64 per 512-key block) with 64-d unit
  centroids, 256 index queries, top 1024 buckets expanded to 4096 long-range
  keys plus 4 sinks and the window ("Latent Sparse Attention", "How LSA finds
  the keys").
* ``lsa_tree_10m``  -- the tree search at 10485760 tokens: three node
  levels over 1310720 buckets, 256 index queries ("Latent Sparse Attention",
  "The tree, step by step").
* ``lsa_prefill_10m`` -- the sampled-threshold flat search for one prefill
  chunk of 32768 queries at 10485760 tokens ("Latent Sparse Attention",
  "What the kernels do about the top-p").
* ``bucket``        -- one sequence of 1048576 tokens (262144 keys) built as
  32768 clusters of 8 keys; 256 decode queries keep 64 buckets and expand them
  to 512 keys ("Latent Sparse Attention", "How LSA finds the keys").

Indexer geometry everywhere: H = 32 heads, d = 128, top-k = 512 (the
GLM-shaped indexer of "Latent Sparse Attention", "Where the time goes"; k = 512
as in the LeanSparse transcript, 01:33-02:06).

Reduced variants (suffix ``_s``) keep every structural feature (several tiles,
ragged tails, causal prefix, planted keys, clusters) at sizes the fp64 oracle
finishes in seconds; they are parity cases.
"""

from __future__ import annotations

from dataclasses import dataclass, field, replace
from typing import Dict


@dataclass(frozen=True)
class Workload:
    name: str
    kind: str  # "decode" | "prefill" | "two_stage" | "bucket" | "lsa" | "attention"
    H: int = 32
    d: int = 128
    k: int = 512
    seed: int = 0
    # decode / two_stage
    B: int = 0
    N: int = 0
    # ragged decode: per-sequence valid lengths drawn in [N - ragged, N]
    ragged: int = 0
    # prefill
    T: int = 0
    q_pos0: int = 0
    stride: int = 4
    tile_keys: int = 8192
    # two_stage
    shortlist: int = 0
    plant_frac: float = 0.0
    plant_cos: float = 0.6
    # bucket
    clusters: int = 0
    cluster_size: int = 0
    noise_rel: float = 0.3
    top_p: int = 0
    budget: int = 0
    extra: Dict[str, int] = field(default_factory=dict)

    def with_(self, **kw) -> "Workload":
        return replace(self, **kw)

    # ---- sizes used by the benchmark and the tests -------------------------
    @property
    def n_keys(self) -> int:
        if self.kind == "bucket":
            return self.clusters * self.cluster_size
        return self.N


WORKLOADS: Dict[str, Workload] = {
    "decode_tiny": Workload("decode_tiny", "decode", B=4, N=2048),
    "decode_batch": Workload("decode_batch", "decode", B=64, N=32768),
    "prefill_chunk": Workload(
        "prefill_chunk", "prefill", T=4096, q_pos0=126976, N=32768, stride=4, tile_keys=8192
    ),
    # the same chunk with fp8 queries (one scale per query head) and an fp8
    # history (one scale per key): the indexer's FP8 form
    "prefill_chunk_fp8": Workload(
        "prefill_chunk_fp8", "prefill", T=4096, q_pos0=126976, N=32768, stride=4, tile_keys=8192,
        extra={"fp8": 1},
    ),
    "two_stage": Workload(
        "two_stage", "two_stage", B=32, N=131072, shortlist=4096, plant_frac=0.05, plant_cos=0.6
    ),
    # the same search with 32-byte PQ compact keys (LeanSparse podcast
    # transcript, 07:12-07:34) in place of the int8 ones
    "two_stage_pq": Workload(
        "two_stage_pq", "two_stage", B=32, N=131072, shortlist=4096, plant_frac=0.05, plant_cos=0.6,
        extra={"pq": 1},
    ),
    "bucket": Workload(
        "bucket", "bucket", T=256, clusters=32768, cluster_size=8, noise_rel=0.3, top_p=64, budget=512
    ),
    # native LSA flat search: one sequence of 1048576 tokens (2048 blocks of
    # 512 keys, 64 buckets each), 256 index queries at positions spread over
    # its second half; top 1024 buckets, 4096 long-range keys, 4 sinks
    # ("Latent Sparse Attention", "How LSA finds the keys")
    "lsa_flat": Workload(
        "lsa_flat", "lsa", T=256, N=1048576, top_p=1024, budget=4096,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "spread": 2053},
    ),
    # its tree search: 32768 node buckets (4 buckets each), beam 2048
    # ("Latent Sparse Attention", "The tree, step by step")
    "lsa_tree": Workload(
        "lsa_tree", "lsa", T=256, N=1048576, top_p=1024, budget=4096,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "spread": 2053, "node_block": 4096, "fanout": 4,
               "beam": 2048},
    ),
    # the tree at 10485760 tokens: 1310720 buckets under three node levels
    # (327680, 81920, 20480 node buckets); the beam starts at level 3, the
    # lowest with at most 32768 node buckets, and scores 20480 + 3 x 8192
    # vectors per query ("Latent Sparse Attention", "The tree, step by step")
    "lsa_tree_10m": Workload(
        "lsa_tree_10m", "lsa", T=256, N=10485760, top_p=1024, budget=4096,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "spread": 20531, "node_block": 4096, "fanout": 4,
               "beam": 2048, "levels": 3, "start_nodes": 32768},
    ),
    # the sampled-threshold flat search on one prefill chunk: 32768 queries
    # (the sequence's last 32768 tokens) against 1310720 buckets at
    # 10485760 tokens, top 1024 buckets each ("Latent Sparse Attention",
    # "What the kernels do about the top-p")
    "lsa_prefill_10m": Workload(
        "lsa_prefill_10m", "lsa", T=32768, N=10485760, top_p=1024, budget=4096,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "chunk": 1},
    ),
    # a 4096-query chunk of the same sequence (the scan's profile case: the
    # 168 MB of centroids still exceed L2, the workspace stays near 1.5 GB)
    "lsa_prefill_10m_q4096": Workload(
        "lsa_prefill_10m_q4096", "lsa", T=4096, N=10485760, top_p=1024, budget=4096,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "chunk": 1},
    ),
    # sparse main attention after the decode selection: 64 decode queries of
    # 128 heads, each over its 512 selected rows of a latent cache of
    # 262144 rows x 576 bf16 (302 MB, larger than L2); H, d = heads, latent
    # width ("03 long context", "The Architectural Answer: Read Less of the
    # Past", stage 2)
    "attn_decode": Workload("attn_decode", "attention", T=64, H=128, d=576, N=262144, k=512),
    # ---- reduced parity cases: several tiles, ragged tails ------------------
    "decode_s": Workload("decode_s", "decode", B=5, N=3000, ragged=700),
    "prefill_s": Workload(
        "prefill_s", "prefill", T=77, q_pos0=4000, N=1019, stride=4, tile_keys=256
    ),
    "prefill_fp8_s": Workload(
        "prefill_fp8_s", "prefill", T=77, q_pos0=4000, N=1019, stride=4, tile_keys=256, extra={"fp8": 1}
    ),
    "two_stage_s": Workload(
        "two_stage_s", "two_stage", B=3, N=9000, shortlist=1024, plant_frac=0.05, plant_cos=0.6, ragged=1500
    ),
    "two_stage_pq_s": Workload(
        "two_stage_pq_s", "two_stage", B=3, N=9000, shortlist=1024, plant_frac=0.05, plant_cos=0.6, ragged=1500,
        extra={"pq": 1},
    ),
    "lsa_flat_s": Workload(
        "lsa_flat_s", "lsa", T=37, N=40000, top_p=64, budget=512,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "edge": 1, "node_block": 4096, "fanout": 4, "beam": 96},
    ),
    # the tree with three node levels at a reduced size: node blocks of 128
    # entries (two key blocks' buckets, so a query can see half a node
    # block), 4992 buckets, 1248 / 288 / 64 node buckets
    "lsa_tree_levels_s": Workload(
        "lsa_tree_levels_s", "lsa", T=37, N=40000, top_p=64, budget=512,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "edge": 1, "node_block": 128, "fanout": 4, "beam": 24,
               "levels": 3, "start_nodes": 500},
    ),
    # a prefill chunk at a reduced size: 3000 queries (the last 3000 tokens of
    # 262144) against 32768 buckets
    "lsa_prefill_s": Workload(
        "lsa_prefill_s", "lsa", T=3000, N=262144, top_p=256, budget=1024,
        extra={"block_keys": 512, "bpb": 64, "n_sink": 4, "chunk": 1},
    ),
    # 7 queries, 2 head groups, 300 slots (5 chunks, the last ragged); rows 0
    # and 1 select nothing and one row, the others a ragged prefix
    "attn_s": Workload("attn_s", "attention", T=7, H=16, d=576, N=3000, k=300, ragged=250),
    "bucket_s": Workload(
        "bucket_s", "bucket", T=19, clusters=1500, cluster_size=8, noise_rel=0.3, top_p=64, budget=512,
        extra={"min_size": 4, "max_size": 16},
    ),
}


def get_workload(name: str) -> Workload:
    try:
        return WORKLOADS[name]
    except KeyError:
        raise KeyError(f"unknown workload {name!r}; known: {sorted(WORKLOADS)}") from None
