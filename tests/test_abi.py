"""The C ABI without a GPU: the shared library loads, exports every entry
point the header declares, and rejects bad arguments before touching CUDA."""

import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ls_indexer.h")


@pytest.fixture(scope="module")
def lib():
    from sparse_attention_indexer_lightning_b200 import build
    build.build()
    from sparse_attention_indexer_lightning_b200 import _lib
    return _lib.load_library()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ls_[a-z0-9_]+)\s*\(", text)))


def test_header_declares_the_calls():
    names = declared_functions()
    for n in ("ls_indexer_score", "ls_topk_select", "ls_prefill_select_stream", "ls_decode_two_stage_select",
              "ls_bucket_select", "ls_decode_select", "ls_last_error", "ls_device_status", "ls_indexer_score_fp8",
              "ls_prefill_select_stream_fp8", "ls_lsa_flat_select", "ls_lsa_tree_select", "ls_indexer_score_pq",
              "ls_decode_two_stage_pq_select", "ls_merge_select", "ls_sparse_attention", "ls_attention_merge",
              "ls_lsa_tree_levels_select"):
        assert n in names


def test_every_declared_symbol_is_exported(lib):
    for n in declared_functions():
        assert hasattr(lib, n), n
    from sparse_attention_indexer_lightning_b200._lib import EXPORTED
    assert set(EXPORTED) == set(declared_functions())


def test_version_and_workspace_queries(lib):
    assert lib.ls_version() == 100
    assert lib.ls_decode_select_workspace_size(64, 32768) == 64 * 32768 * 4   # the score rows only
    # one 8192-key tile of scores plus lists of k + 2k entries per later tile (values and labels)
    assert lib.ls_prefill_select_workspace_size(4096, 32768, 8192, 512, 0) >= 4096 * 8192 * 4 + 4096 * (512 + 3 * 1024) * 8
    assert lib.ls_prefill_select_workspace_size(4096, 8192, 8192, 512, 0) < 4096 * 8192 * 4 + 4096 * 64
    # full_scores: the whole T x N matrix
    assert lib.ls_prefill_select_workspace_size(4096, 32768, 8192, 512, 1) >= 4096 * 32768 * 4
    assert lib.ls_two_stage_workspace_size(32, 131072, 4096) >= 32 * 131072 * 4 + 2 * 32 * 4096 * 4
    assert lib.ls_bucket_workspace_size(256, 32768, 64, 512) >= 256 * 32768 * 4
    assert lib.ls_decode_select_workspace_size(0, 10) == 0
    # fp8: w * q_scale per (query, head); the fp8 prefill adds it to the bf16 prefill's workspace
    assert lib.ls_indexer_score_fp8_workspace_size(2, 9) >= 2 * 9 * 32 * 4
    assert (lib.ls_prefill_select_fp8_workspace_size(4096, 32768, 8192, 512, 1)
            >= lib.ls_prefill_select_workspace_size(4096, 32768, 8192, 512, 1) + 4096 * 32 * 4)
    # LSA: the T x P bucket scores, visible counts and picks
    assert lib.ls_lsa_flat_workspace_size(256, 131072, 1024, 0, 0) >= 256 * 131072 * 4 + 256 * 1024 * 4
    # LSA tree: node scores, beam and candidates (beam * fanout + node_block per row)
    assert lib.ls_lsa_tree_workspace_size(256, 32768, 2048, 4, 4096, 1024) >= 256 * 32768 * 4 + 256 * 12288 * 8
    # LSA tree over three node levels at 10M tokens: starts at level 3 (20480 nodes); candidate rows of
    # beam * fanout + node_block - 1 entries; invalid level sizes answer 0
    import ctypes
    sizes = (ctypes.c_int * 3)(327680, 81920, 20480)
    ws3 = lib.ls_lsa_tree_levels_workspace_size(256, 1310720, sizes, 3, 4096, 4, 2048, 32768, 1024)
    assert ws3 >= 256 * 20480 * 4 + 256 * (8192 + 4095) * 8 + 2 * 256 * 2048 * 4 + 4 * 256 * 4
    assert ws3 < 256 * 81920 * 4                # the level-2 scores are never held
    bad = (ctypes.c_int * 3)(327681, 81920, 20480)
    assert lib.ls_lsa_tree_levels_workspace_size(256, 1310720, bad, 3, 4096, 4, 2048, 32768, 1024) == 0
    assert lib.ls_lsa_tree_levels_workspace_size(256, 1310720, sizes, 0, 4096, 4, 2048, 32768, 1024) == 0
    # shard merge: the packed S * k_in candidates per row (values and positions) and the row counts
    assert lib.ls_merge_select_workspace_size(4, 4096, 512) >= 4096 * 4 * 512 * 8 + 4096 * 4
    assert lib.ls_merge_select_workspace_size(0, 4096, 512) == 0
    # the threshold form adds the samples and the candidate lists (4 * top_p per row, segments of twice that)
    assert (lib.ls_lsa_flat_workspace_size(256, 131072, 1024, 1, 0)
            >= lib.ls_lsa_flat_workspace_size(256, 131072, 1024, 0, 0) + 256 * 8192 * 8)
    # ... but never the T x P matrix at prefill scale: 32768 queries x 1310720 buckets (172 GB) fit in
    # about 20 GB, the fallback's scores within 4 GiB (or fallback_rows x P)
    big = lib.ls_lsa_flat_workspace_size(32768, 1310720, 1024, 1, 0)
    assert 0 < big < 20 * 2 ** 30
    assert big - lib.ls_lsa_flat_workspace_size(32768, 1310720, 1024, 1, 256) >= (768 - 256) * 1310720 * 4 - 4096


def test_argument_checks_without_gpu(lib):
    P = ctypes.c_void_p
    dummy = P(16)
    # H != 32 is not built
    st = lib.ls_indexer_score(dummy, dummy, dummy, 0, None, None, None, 4, 1, 1, 16, 128, 64, dummy, None, None)
    assert st == 3
    assert b"H=32" in lib.ls_last_error()
    # k out of range
    assert lib.ls_topk_select(dummy, 10, None, None, 1, 10, 0, dummy, None, None) == 1
    assert lib.ls_topk_select(dummy, 10, None, None, 1, 10, 5000, dummy, None, None) == 1
    # ld < N
    assert lib.ls_topk_select(dummy, 5, None, None, 1, 10, 3, dummy, None, None) == 1
    # short workspace
    st = lib.ls_decode_select(dummy, dummy, dummy, None, 2, 32, 128, 100, 8, dummy, None, dummy, 10, None)
    assert st == 2
    # unknown key dtype / misaligned pointers
    st = lib.ls_indexer_score(dummy, dummy, dummy, 9, None, None, None, 4, 1, 1, 32, 128, 64, dummy, None, None)
    assert st == 1
    st = lib.ls_indexer_score(P(17), dummy, dummy, 0, None, None, None, 4, 1, 1, 32, 128, 64, dummy, None, None)
    assert st == 1
    # the selection histogram is built for one query per sequence
    st = lib.ls_indexer_score(dummy, dummy, dummy, 0, None, None, None, 4, 1, 2, 32, 128, 64, dummy, dummy, None)
    assert st == 3
    # two-stage: shortlist shorter than k
    st = lib.ls_decode_two_stage_select(dummy, dummy, dummy, dummy, dummy, dummy, None, 1, 32, 128, 100, 256, 512,
                                        dummy, None, None, dummy, 1 << 30, None)
    assert st == 1
    # PQ two-stage: shortlist shorter than k; PQ scores: null codebooks, H != 32
    st = lib.ls_decode_two_stage_pq_select(dummy, dummy, dummy, dummy, dummy, dummy, None, 1, 32, 128, 100, 256, 512,
                                           dummy, None, None, dummy, 1 << 30, None)
    assert st == 1
    assert lib.ls_indexer_score_pq(dummy, dummy, dummy, None, None, 1, 32, 128, 64, dummy, None) == 1
    assert lib.ls_indexer_score_pq(dummy, dummy, dummy, dummy, None, 1, 16, 128, 64, dummy, None) == 3
    # fp8 indexer: H != 32, null scale, short workspace
    assert lib.ls_indexer_score_fp8(dummy, dummy, dummy, dummy, dummy, None, None, 4, 1, 8, 16, 128, 64, dummy,
                                    dummy, 1 << 20, None) == 3
    assert lib.ls_indexer_score_fp8(dummy, None, dummy, dummy, dummy, None, None, 4, 1, 8, 32, 128, 64, dummy,
                                    dummy, 1 << 20, None) == 1
    assert lib.ls_indexer_score_fp8(dummy, dummy, dummy, dummy, dummy, None, None, 4, 1, 8, 32, 128, 64, dummy,
                                    dummy, 16, None) == 2
    # fp8 prefill: k out of range; LSA: d != 64, top_p too large, short workspace
    assert lib.ls_prefill_select_stream_fp8(dummy, dummy, dummy, dummy, 4, 32, 128, dummy, dummy, 100, 4, 64,
                                            dummy, dummy, 5000, 0, dummy, None, dummy, 1 << 30, None, None) == 1
    assert lib.ls_lsa_flat_select(dummy, dummy, dummy, dummy, dummy, 4, 128, 64, 512, 64, 4, 16, 64, 1, 0, dummy,
                                  dummy, None, dummy, 1 << 30, None) == 3
    assert lib.ls_lsa_flat_select(dummy, dummy, dummy, dummy, dummy, 4, 64, 64, 512, 64, 4, 5000, 64, 1, 0, dummy,
                                  dummy, None, dummy, 1 << 30, None) == 1
    assert lib.ls_lsa_flat_select(dummy, dummy, dummy, dummy, dummy, 4, 64, 64, 512, 64, 4, 16, 64, 1, 0, dummy,
                                  dummy, None, dummy, 8, None) == 2
    assert lib.ls_lsa_flat_select(None, None, None, None, None, 0, 64, 64, 512, 64, 4, 16, 64, 1, 0, None, None,
                                  None, None, 0, None) == 0
    # LSA tree: d != 64, beam too large, more node children than buckets, short workspace, empty batch
    tree = lib.ls_lsa_tree_select
    assert tree(dummy, dummy, dummy, dummy, dummy, dummy, 4, 128, 4096, 1024, 512, 64, 4096, 4, 96, 4, 64, 512, dummy,
                dummy, None, None, dummy, 1 << 30, None) == 3
    assert tree(dummy, dummy, dummy, dummy, dummy, dummy, 4, 64, 4096, 1024, 512, 64, 4096, 4, 5000, 4, 64, 512, dummy,
                dummy, None, None, dummy, 1 << 30, None) == 1
    assert tree(dummy, dummy, dummy, dummy, dummy, dummy, 4, 64, 4096, 1025, 512, 64, 4096, 4, 96, 4, 64, 512, dummy,
                dummy, None, None, dummy, 1 << 30, None) == 1
    assert tree(dummy, dummy, dummy, dummy, dummy, dummy, 4, 64, 4096, 1024, 512, 64, 4096, 4, 96, 4, 64, 512, dummy,
                dummy, None, None, dummy, 16, None) == 2
    assert tree(None, None, None, None, None, None, 0, 64, 4096, 1024, 512, 64, 4096, 4, 96, 4, 64, 512, None, None,
                None, None, None, 0, None) == 0
    # shard merge: no shards, k above the limit, short workspace, empty batch
    assert lib.ls_merge_select(dummy, dummy, dummy, 0, 4, 512, 512, dummy, None, dummy, 1 << 30, None) == 1
    assert lib.ls_merge_select(dummy, dummy, dummy, 2, 4, 512, 100000, dummy, None, dummy, 1 << 30, None) == 1
    assert lib.ls_merge_select(dummy, dummy, dummy, 2, 4, 512, 512, dummy, None, dummy, 16, None) == 2
    assert lib.ls_merge_select(None, None, None, 2, 0, 512, 512, None, None, None, 0, None) == 0
    # sparse attention: latent width not built, heads not a multiple of 8, k above 2048, misaligned q,
    # empty batch
    att = lib.ls_sparse_attention
    assert att(dummy, dummy, dummy, None, 4, 128, 128, 512, 1000, 512, 0.04, 0, dummy, None, None) == 3
    assert att(dummy, dummy, dummy, None, 4, 12, 576, 512, 1000, 512, 0.04, 0, dummy, None, None) == 1
    assert att(dummy, dummy, dummy, None, 4, 128, 576, 512, 1000, 100000, 0.04, 0, dummy, None, None) == 1
    assert att(P(8), dummy, dummy, None, 4, 128, 576, 512, 1000, 512, 0.04, 0, dummy, None, None) == 1
    assert att(dummy, dummy, dummy, None, 4, 128, 576, 512, 1000, 512, float("nan"), 0, dummy, None, None) == 1
    assert att(None, None, None, None, 0, 128, 576, 512, 1000, 512, 0.04, 0, None, None, None) == 0
    assert att(dummy, dummy, dummy, None, 4, 128, 576, 512, 1000, 512, 0.04, 6, dummy, None, None) == 1
    # attention merge: no parts, odd value width, empty
    mg = lib.ls_attention_merge
    assert mg(dummy, dummy, 0, 10, 512, dummy, None, None) == 1
    assert mg(dummy, dummy, 2, 10, 511, dummy, None, None) == 1
    assert mg(None, None, 2, 0, 512, None, None, None) == 0
    # bucket: budget below k
    st = lib.ls_bucket_select(dummy, dummy, dummy, dummy, dummy, dummy, 1, 32, 128, 10, 80, 4, 100, 512, dummy,
                              None, None, dummy, 1 << 30, None)
    assert st == 1
    # empty problems are a no-op
    assert lib.ls_indexer_score(None, None, None, 0, None, None, None, 4, 0, 1, 32, 128, 64, None, None, None) == 0
    # profiling with nothing recorded
    n = ctypes.c_int(-1)
    assert lib.ls_profile_begin() == 0
    assert lib.ls_profile_end(ctypes.byref(n)) == 0 and n.value == 0
    assert lib.ls_profile_kernel(0, None, None, None) == 1


def test_tree_levels_argument_checks(lib):
    """ls_lsa_tree_levels_select and its workspace query refuse bad trees
    before touching CUDA: the host arrays are read, nothing is launched."""
    P = ctypes.c_void_p
    dummy = P(16)
    sizes = (ctypes.c_int * 3)(32768, 8192, 2048)
    nodes = (ctypes.c_void_p * 3)(16, 32, 48)

    def call(L=3, d=64, Pb=131072, beam=2048, start=32768, ws_bytes=1 << 40, level_sizes=sizes, node_ptrs=nodes,
             T=4, node_block=4096, fanout=4):
        return lib.ls_lsa_tree_levels_select(dummy, dummy, dummy, ctypes.cast(node_ptrs, P),
                                             ctypes.cast(level_sizes, P), L, dummy, dummy, T, d, Pb, 512, 64,
                                             node_block, fanout, beam, start, 4, 1024, 4096, dummy, dummy, None,
                                             None, dummy, ws_bytes, None)

    ws_size = lib.ls_lsa_tree_levels_workspace_size
    good = ws_size(4, 131072, ctypes.cast(sizes, P), 3, 4096, 4, 2048, 32768, 1024)
    assert good > 0
    assert call(d=128) == 3                                      # the index space is 64-d
    assert call(L=0) == 1 and call(L=17) == 1                    # 1 .. 16 levels
    big = (ctypes.c_int * 3)(32768, 8193, 2048)                  # 8193 nodes of 4 exceed 32768 below
    assert call(level_sizes=big) == 1
    assert ws_size(4, 131072, ctypes.cast(big, P), 3, 4096, 4, 2048, 32768, 1024) == 0
    assert call(beam=0) == 1 and call(beam=5000) == 1 and call(start=0) == 1
    assert call(node_block=4098) == 1                            # not a multiple of fanout
    assert call(Pb=100000) == 1                                  # level 1 needs 4 * 32768 buckets
    assert "level 1" in lib.ls_last_error().decode()
    null_level = (ctypes.c_void_p * 3)(16, None, 48)
    assert call(node_ptrs=null_level) == 1 and b"level 2" in lib.ls_last_error()
    odd_level = (ctypes.c_void_p * 3)(16, 32, 40)                # level 3's centroids 8-byte aligned only
    assert call(node_ptrs=odd_level) == 1
    assert call(ws_bytes=good - 1) == 2
    assert call(T=0, ws_bytes=0) == 0                            # an empty batch is a no-op
    assert ws_size(0, 131072, ctypes.cast(sizes, P), 3, 4096, 4, 2048, 32768, 1024) == 0


def test_missing_library_fails_loudly(tmp_path):
    from sparse_attention_indexer_lightning_b200 import _lib
    with pytest.raises(ImportError):
        _lib.load_library(str(tmp_path / "libls_indexer.so"))


def _host_calls():
    """One call of each Python entry point with host (CPU) tensors of the
    right dtypes and shapes."""
    import torch
    import sparse_attention_indexer_lightning_b200 as L
    bf, f32, i32, i64 = torch.bfloat16, torch.float32, torch.int32, torch.int64
    z = torch.zeros
    B, T, H, d, N, P = 2, 3, 32, 128, 64, 16
    e4 = torch.float8_e4m3fn
    return {
        "ls_indexer_score": lambda: L.ls_indexer_score(z(B, T, H, d, dtype=bf), z(B, T, H), z(B, N, d, dtype=bf)),
        "ls_topk_select": lambda: L.ls_topk_select(z(B, N), 8),
        "ls_decode_select": lambda: L.ls_decode_select(z(B, H, d, dtype=bf), z(B, H), z(B, N, d, dtype=bf), k=8),
        "ls_decode_select_noalloc": lambda: L.ls_decode_select_noalloc(z(B, H, d, dtype=bf), z(B, H),
                                                                       z(B, N, d, dtype=bf), k=8),
        "ls_indexer_score_fp8": lambda: L.ls_indexer_score_fp8(z(B, T, H, d, dtype=e4), z(B, T, H), z(B, T, H),
                                                               z(B, N, d, dtype=e4), z(B, N)),
        "ls_decode_two_stage_select": lambda: L.ls_decode_two_stage_select(
            z(B, H, d, dtype=bf), z(B, H), z(B, N, d, dtype=torch.int8), z(B, N), z(B, N, d, dtype=e4), z(B, N),
            shortlist=16, k=8),
        "ls_indexer_score_pq": lambda: L.ls_indexer_score_pq(z(B, H, d, dtype=bf), z(B, H),
                                                             z(B, N, 32, dtype=torch.uint8),
                                                             z(32, 256, 4, dtype=torch.float16)),
        "ls_bucket_select": lambda: L.ls_bucket_select(z(B, H, d, dtype=bf), z(B, H), z(P, d, dtype=bf),
                                                       z(P + 1, dtype=i32), z(N, dtype=i32), z(N, d, dtype=bf),
                                                       top_p=4, budget=16, k=8),
        "ls_lsa_flat_select": lambda: L.ls_lsa_flat_select(z(T, 64, dtype=bf), z(T, dtype=i64), z(P, 64, dtype=bf),
                                                           z(P + 1, dtype=i32), z(N, dtype=i32), top_p=4, budget=8),
        "ls_lsa_tree_select": lambda: L.ls_lsa_tree_select(z(T, 64, dtype=bf), z(T, dtype=i64), z(P, 64, dtype=bf),
                                                           z(P // 4, 64, dtype=bf), z(P + 1, dtype=i32),
                                                           z(N, dtype=i32), node_block=8, beam=2, top_p=4, budget=8),
        "ls_lsa_tree_levels_select": lambda: L.ls_lsa_tree_levels_select(
            z(T, 64, dtype=bf), z(T, dtype=i64), z(P, 64, dtype=bf), [z(P // 4, 64, dtype=bf)],
            z(P + 1, dtype=i32), z(N, dtype=i32), node_block=8, beam=2, start_nodes=4, top_p=4, budget=8),
        "ls_prefill_select_stream": lambda: L.ls_prefill_select_stream(
            z(T, H, d, dtype=bf), z(T, H), z(T, dtype=i64), z(N, d, dtype=bf), z(16, d, dtype=bf),
            z(16, d, dtype=bf), k=8),
        "ls_prefill_select_stream_fp8": lambda: L.ls_prefill_select_stream_fp8(
            z(T, H, d, dtype=e4), z(T, H), z(T, H), z(T, dtype=i64), z(N, d, dtype=e4), z(N), z(16, d, dtype=e4),
            z(16, d, dtype=e4), k=8),
        "ls_merge_select": lambda: L.ls_merge_select(z(2, T, 8), z(2, T, 8, dtype=i32), z(2, dtype=i32), k=8),
        "ls_sparse_attention": lambda: L.ls_sparse_attention(z(2, 8, 576, dtype=bf), z(10, 576, dtype=bf),
                                                             z(2, 4, dtype=i32)),
        "ls_attention_merge": lambda: L.ls_attention_merge(z(2, 3, 512), z(2, 3)),
    }


@pytest.mark.parametrize("name", sorted(_host_calls()))
def test_every_binding_refuses_host_tensors(name):
    """Each Python entry point checks its tensors before any CUDA call: host
    tensors give a ValueError naming CUDA, whatever the machine has."""
    with pytest.raises(ValueError, match="CUDA"):
        _host_calls()[name]()
