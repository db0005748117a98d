"""ctypes binding of libls_indexer.so (the C ABI in include/ls_indexer.h).

Argument marshalling only: the functions below check dtypes, devices and
shapes of torch tensors, allocate outputs and workspace through torch, and
call the library on the current CUDA stream.  Every step of the selection path
runs in the library's kernels; there is no fallback.  The first call loads the
shared library and raises ImportError when it is missing or stale.
"""

from __future__ import annotations

import ctypes
import math
import os
from typing import Optional

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "libls_indexer.so")

LS_OK = 0
LS_ERR_INVALID_ARG = 1
LS_ERR_WORKSPACE = 2
LS_ERR_UNSUPPORTED = 3
LS_ERR_CUDA = 4
LS_ERR_TIMEOUT = 5
LS_KEY_BF16 = 0
LS_KEY_FP8_E4M3 = 1
LS_KEY_INT8 = 2
LS_FAULT_WAIT_TIMEOUT = 1
LS_FAULT_BAD_INDEX = 2
LS_ATTN_FOREIGN_ROWS = 1
LS_ATTN_CUDA_CORES = 2

EXPORTED = (
    "ls_last_error", "ls_version", "ls_device_status", "ls_indexer_score", "ls_topk_select",
    "ls_decode_select_workspace_size", "ls_decode_select", "ls_prefill_select_workspace_size",
    "ls_prefill_select_stream", "ls_two_stage_workspace_size", "ls_decode_two_stage_select",
    "ls_bucket_workspace_size", "ls_bucket_select", "ls_selftest_wait_probe", "ls_profile_begin",
    "ls_profile_end", "ls_profile_kernel", "ls_decode_select_noalloc", "ls_decode_two_stage_pq_select",
    "ls_indexer_score_pq", "ls_indexer_score_fp8_workspace_size", "ls_indexer_score_fp8",
    "ls_prefill_select_fp8_workspace_size", "ls_prefill_select_stream_fp8", "ls_lsa_flat_workspace_size",
    "ls_lsa_flat_select", "ls_lsa_tree_workspace_size", "ls_lsa_tree_select", "ls_merge_select_workspace_size",
    "ls_merge_select", "ls_sparse_attention", "ls_attention_merge", "ls_lsa_tree_levels_workspace_size",
    "ls_lsa_tree_levels_select",
)
HIST_BINS = 2048


class LSError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"ls status {status}: {msg}")
        self.status = status


def load_library(path: str = LIB_PATH) -> ctypes.CDLL:
    if not os.path.exists(path):
        raise ImportError(
            f"{path} is missing: build it with `python -m sparse_attention_indexer_lightning_b200.build`"
        )
    lib = ctypes.CDLL(path)
    P, I, I64, SZ, U64 = ctypes.c_void_p, ctypes.c_int, ctypes.c_int64, ctypes.c_size_t, ctypes.c_uint64
    sig = {
        "ls_last_error": (ctypes.c_char_p, []),
        "ls_version": (I, []),
        "ls_device_status": (I, [P, P]),
        "ls_indexer_score": (I, [P, P, P, I, P, P, P, I, I, I, I, I, I, P, P, P]),
        "ls_topk_select": (I, [P, I64, P, P, I, I, I, P, P, P]),
        "ls_decode_select_workspace_size": (SZ, [I, I]),
        "ls_decode_select": (I, [P, P, P, P, I, I, I, I, I, P, P, P, SZ, P]),
        "ls_prefill_select_workspace_size": (SZ, [I, I, I, I, I]),
        "ls_prefill_select_stream": (I, [P, P, P, I, I, I, P, I, I, I, P, P, I, I, P, P, P, SZ, P, P]),
        "ls_two_stage_workspace_size": (SZ, [I, I, I]),
        "ls_decode_two_stage_select": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, SZ, P]),
        "ls_bucket_workspace_size": (SZ, [I, I, I, I]),
        "ls_bucket_select": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, I, P, P, P, P, SZ, P]),
        "ls_selftest_wait_probe": (I, [U64, P, P]),
        "ls_profile_begin": (I, []),
        "ls_profile_end": (I, [P]),
        "ls_profile_kernel": (I, [I, P, P, P]),
        "ls_decode_select_noalloc": (I, [P, P, P, P, I, I, I, I, I, P, P, P]),
        "ls_decode_two_stage_pq_select": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, P, P, SZ, P]),
        "ls_indexer_score_pq": (I, [P, P, P, P, P, I, I, I, I, P, P]),
        "ls_indexer_score_fp8_workspace_size": (SZ, [I, I]),
        "ls_indexer_score_fp8": (I, [P, P, P, P, P, P, P, I, I, I, I, I, I, P, P, SZ, P]),
        "ls_prefill_select_fp8_workspace_size": (SZ, [I, I, I, I, I]),
        "ls_prefill_select_stream_fp8": (I, [P, P, P, P, I, I, I, P, P, I, I, I, P, P, I, I, P, P, P, SZ, P, P]),
        "ls_lsa_flat_workspace_size": (SZ, [I, I, I, I, I]),
        "ls_lsa_flat_select": (I, [P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, P, P, P, P, SZ, P]),
        "ls_lsa_tree_workspace_size": (SZ, [I, I, I, I, I, I]),
        "ls_lsa_tree_select": (I, [P, P, P, P, P, P, I, I, I, I, I, I, I, I, I, I, I, I, P, P, P, P, P, SZ, P]),
        "ls_lsa_tree_levels_workspace_size": (SZ, [I, I, P, I, I, I, I, I, I]),
        "ls_lsa_tree_levels_select": (I, [P, P, P, P, P, I, P, P, I, I, I, I, I, I, I, I, I, I, I, I, P, P, P, P,
                                          P, SZ, P]),
        "ls_merge_select_workspace_size": (SZ, [I, I, I]),
        "ls_merge_select": (I, [P, P, P, I, I, I, I, P, P, P, SZ, P]),
        "ls_sparse_attention": (I, [P, P, P, P, I, I, I, I, I64, I, ctypes.c_float, I, P, P, P]),
        "ls_attention_merge": (I, [P, P, I, I64, I, P, P, P]),
    }
    for name, (res, args) in sig.items():
        try:
            fn = getattr(lib, name)
        except AttributeError:
            raise ImportError(f"{path} does not export {name}: it is stale, rebuild it") from None
        fn.restype = res
        fn.argtypes = args
    return lib


_lib: Optional[ctypes.CDLL] = None


def lib() -> ctypes.CDLL:
    global _lib
    if _lib is None:
        _lib = load_library()
    return _lib


def _check(status: int) -> None:
    if status != LS_OK:
        raise LSError(status, lib().ls_last_error().decode(errors="replace"))


def _ptr(t: Optional[torch.Tensor]):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _dev(t: torch.Tensor, dtype, name: str, ndim: Optional[int] = None) -> torch.Tensor:
    if t.device.type != "cuda":
        raise ValueError(f"{name} must be a CUDA tensor")
    if t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}, got {t.dtype}")
    if ndim is not None and t.dim() != ndim:
        raise ValueError(f"{name} must have {ndim} dims, got {tuple(t.shape)}")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    return t


def _opt(t, dtype, name):
    return None if t is None else _dev(t, dtype, name)


def _workspace(nbytes: int, device) -> torch.Tensor:
    return torch.empty(max(int(nbytes), 1), dtype=torch.uint8, device=device)


# --------------------------------------------------------------------------- #
# the library's calls, one Python function per C entry point
# --------------------------------------------------------------------------- #
def ls_indexer_score(q, w, keys, key_scale=None, n_valid=None, q_pos=None, stride: int = 4, hist_out=None,
                     stream=None):
    """q [B,T,H,d] bf16, w [B,T,H] f32, keys [B,N,d] (bf16 | float8_e4m3fn | int8) -> scores [B,T,N] f32.

    hist_out: optional zeroed int32 [B*T, 2048] tensor that receives the selection histogram (T == 1)."""
    _dev(q, torch.bfloat16, "q", 4)
    B, T, H, d = q.shape
    _dev(w, torch.float32, "w", 3)
    if keys.dtype == torch.bfloat16:
        kd = LS_KEY_BF16
    elif keys.dtype == torch.float8_e4m3fn:
        kd = LS_KEY_FP8_E4M3
    elif keys.dtype == torch.int8:
        kd = LS_KEY_INT8
    else:
        raise TypeError(f"unsupported key dtype {keys.dtype}")
    _dev(keys, keys.dtype, "keys", 3)
    N = keys.shape[1]
    _opt(key_scale, torch.float32, "key_scale")
    _opt(n_valid, torch.int32, "n_valid")
    _opt(q_pos, torch.int64, "q_pos")
    _opt(hist_out, torch.int32, "hist_out")
    out = torch.empty((B, T, N), dtype=torch.float32, device=q.device)
    _check(lib().ls_indexer_score(_ptr(q), _ptr(w), _ptr(keys), kd, _ptr(key_scale), _ptr(n_valid), _ptr(q_pos),
                                  stride, B, T, H, d, N, _ptr(out), _ptr(hist_out), _stream(stream)))
    return out


def ls_topk_select(scores, k: int, n_valid=None, hist=None, with_values: bool = True, stream=None):
    """scores [R,N] f32 (row-contiguous) -> (idx [R,k] int32, val [R,k] f32).

    hist: optional int32 [R, 2048] selection histogram of the rows (from ls_indexer_score)."""
    _dev(scores, torch.float32, "scores", 2)
    R, N = scores.shape
    _opt(n_valid, torch.int32, "n_valid")
    _opt(hist, torch.int32, "hist")
    idx = torch.empty((R, k), dtype=torch.int32, device=scores.device)
    val = torch.empty((R, k), dtype=torch.float32, device=scores.device) if with_values else None
    _check(lib().ls_topk_select(_ptr(scores), N, _ptr(n_valid), _ptr(hist), R, N, k, _ptr(idx), _ptr(val),
                                _stream(stream)))
    return idx, val


def ls_decode_select(q, w, keys, k: int = 512, n_valid=None, ws=None, out=None, stream=None):
    """q [B,H,d] bf16, w [B,H] f32, keys [B,N,d] bf16 -> (idx [B,k], val [B,k])."""
    _dev(q, torch.bfloat16, "q", 3)
    B, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    _dev(keys, torch.bfloat16, "keys", 3)
    N = keys.shape[1]
    _opt(n_valid, torch.int32, "n_valid")
    need = lib().ls_decode_select_workspace_size(B, N)
    if ws is None:
        ws = _workspace(need, q.device)
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=q.device),
               torch.empty((B, k), dtype=torch.float32, device=q.device))
    idx, val = out
    _check(lib().ls_decode_select(_ptr(q), _ptr(w), _ptr(keys), _ptr(n_valid), B, H, d, N, k, _ptr(idx), _ptr(val),
                                  _ptr(ws), ws.numel(), _stream(stream)))
    return idx, val


def ls_decode_select_noalloc(q, w, keys, k: int = 512, n_valid=None, out=None, stream=None):
    """ls_decode_select with the library's fixed device scratch instead of a workspace.

    For callers that cannot allocate device memory on this path; sizes above
    the fixed scratch raise LSError (LS_ERR_WORKSPACE).  Calls share the
    scratch, so calls that overlap on the GPU must be serialised."""
    _dev(q, torch.bfloat16, "q", 3)
    B, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    _dev(keys, torch.bfloat16, "keys", 3)
    N = keys.shape[1]
    _opt(n_valid, torch.int32, "n_valid")
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=q.device),
               torch.empty((B, k), dtype=torch.float32, device=q.device))
    idx, val = out
    _check(lib().ls_decode_select_noalloc(_ptr(q), _ptr(w), _ptr(keys), _ptr(n_valid), B, H, d, N, k, _ptr(idx),
                                          _ptr(val), _stream(stream)))
    return idx, val


def ls_prefill_select_stream(q, w, q_pos, hist_k, buf0, buf1, k: int = 512, stride: int = 4,
                             tile_keys: Optional[int] = None, full_scores: bool = False, ws=None, out=None,
                             copy_stream=None, stream=None):
    """Causal prefill selection with the history streamed from (pinned) host memory.

    q [T,H,d] bf16, w [T,H] f32, q_pos [T] int64 (device); hist_k [N,d] bf16 in
    pinned host memory (or on the device); buf0/buf1 [tile_keys, d] bf16 device.
    full_scores=False keeps a running top-k across the tiles (workspace: one
    tile of scores); True scores into a full T x N matrix and selects once.
    """
    _dev(q, torch.bfloat16, "q", 3)
    T, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    _dev(q_pos, torch.int64, "q_pos", 1)
    if hist_k.dtype != torch.bfloat16 or hist_k.dim() != 2 or not hist_k.is_contiguous():
        raise ValueError("hist_k must be a contiguous [N, d] bf16 tensor")
    if hist_k.device.type == "cpu" and not hist_k.is_pinned():
        raise ValueError("hist_k must be in pinned host memory")
    N = hist_k.shape[0]
    _dev(buf0, torch.bfloat16, "buf0", 2)
    _dev(buf1, torch.bfloat16, "buf1", 2)
    tk = buf0.shape[0] if tile_keys is None else tile_keys
    if buf0.shape[0] < tk or buf1.shape[0] < tk:
        raise ValueError("buffers are shorter than tile_keys")
    need = lib().ls_prefill_select_workspace_size(T, N, tk, k, int(full_scores))
    if ws is None:
        ws = _workspace(need, q.device)
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=q.device),
               torch.empty((T, k), dtype=torch.float32, device=q.device))
    idx, val = out
    cs = _stream(stream)
    xs = ctypes.c_void_p(copy_stream.cuda_stream) if copy_stream is not None else None
    _check(lib().ls_prefill_select_stream(_ptr(q), _ptr(w), _ptr(q_pos), T, H, d, _ptr(hist_k), N, stride, tk,
                                          _ptr(buf0), _ptr(buf1), k, int(full_scores), _ptr(idx), _ptr(val),
                                          _ptr(ws), ws.numel(), cs, xs))
    return idx, val


def _codes(t, name: str, ndim: int) -> torch.Tensor:
    """fp8 e4m3 codes as a uint8 view (float8_e4m3fn tensors are viewed, not converted)."""
    if t.dtype == torch.float8_e4m3fn:
        t = t.view(torch.uint8)
    return _dev(t, torch.uint8, name, ndim)


def ls_indexer_score_fp8(q8, q_scale, w, k8, k_scale, n_valid=None, q_pos=None, stride: int = 4, ws=None,
                         stream=None):
    """q8 [B,T,H,d] e4m3 (float8_e4m3fn or uint8 codes), q_scale [B,T,H] f32, w [B,T,H] f32,
    k8 [B,N,d] e4m3, k_scale [B,N] f32 -> scores [B,T,N] f32 (the fp8 indexer; scales >= 0)."""
    q8 = _codes(q8, "q8", 4)
    B, T, H, d = q8.shape
    _dev(q_scale, torch.float32, "q_scale", 3)
    _dev(w, torch.float32, "w", 3)
    k8 = _codes(k8, "k8", 3)
    N = k8.shape[1]
    _dev(k_scale, torch.float32, "k_scale", 2)
    _opt(n_valid, torch.int32, "n_valid")
    _opt(q_pos, torch.int64, "q_pos")
    need = lib().ls_indexer_score_fp8_workspace_size(B, T)
    if ws is None:
        ws = _workspace(need, q8.device)
    out = torch.empty((B, T, N), dtype=torch.float32, device=q8.device)
    _check(lib().ls_indexer_score_fp8(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(k8), _ptr(k_scale), _ptr(n_valid),
                                      _ptr(q_pos), stride, B, T, H, d, N, _ptr(out), _ptr(ws), ws.numel(),
                                      _stream(stream)))
    return out


def ls_prefill_select_stream_fp8(q8, q_scale, w, q_pos, hist_k8, hist_kscale, buf0, buf1, k: int = 512,
                                 stride: int = 4, tile_keys: Optional[int] = None, full_scores: bool = False,
                                 ws=None, out=None, copy_stream=None, stream=None):
    """Causal prefill selection with fp8 queries and an fp8 history streamed from (pinned) host memory.

    q8 [T,H,d] e4m3, q_scale [T,H] f32, w [T,H] f32, q_pos [T] int64 (device);
    hist_k8 [N,d] e4m3 codes and hist_kscale [N] f32 in pinned host memory (or
    on the device); buf0/buf1 uint8 device buffers of tile_keys * (d + 4) bytes.
    """
    q8 = _codes(q8, "q8", 3)
    T, H, d = q8.shape
    _dev(q_scale, torch.float32, "q_scale", 2)
    _dev(w, torch.float32, "w", 2)
    _dev(q_pos, torch.int64, "q_pos", 1)
    if hist_k8.dtype == torch.float8_e4m3fn:
        hist_k8 = hist_k8.view(torch.uint8)
    for t, dt, nd, name in ((hist_k8, torch.uint8, 2, "hist_k8"), (hist_kscale, torch.float32, 1, "hist_kscale")):
        if t.dtype != dt or t.dim() != nd or not t.is_contiguous():
            raise ValueError(f"{name} must be a contiguous {nd}-d {dt} tensor")
        if t.device.type == "cpu" and not t.is_pinned():
            raise ValueError(f"{name} must be in pinned host memory")
    N = hist_k8.shape[0]
    _dev(buf0, torch.uint8, "buf0", 1)
    _dev(buf1, torch.uint8, "buf1", 1)
    tk = buf0.numel() // (d + 4) if tile_keys is None else tile_keys
    if buf0.numel() < tk * (d + 4) or buf1.numel() < tk * (d + 4):
        raise ValueError("buffers are shorter than tile_keys * (d + 4) bytes")
    need = lib().ls_prefill_select_fp8_workspace_size(T, N, tk, k, int(full_scores))
    if ws is None:
        ws = _workspace(need, q8.device)
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=q8.device),
               torch.empty((T, k), dtype=torch.float32, device=q8.device))
    idx, val = out
    cs = _stream(stream)
    xs = ctypes.c_void_p(copy_stream.cuda_stream) if copy_stream is not None else None
    _check(lib().ls_prefill_select_stream_fp8(_ptr(q8), _ptr(q_scale), _ptr(w), _ptr(q_pos), T, H, d, _ptr(hist_k8),
                                              _ptr(hist_kscale), N, stride, tk, _ptr(buf0), _ptr(buf1), k,
                                              int(full_scores), _ptr(idx), _ptr(val), _ptr(ws), ws.numel(), cs, xs))
    return idx, val


def ls_decode_two_stage_select(q, w, ck, ck_scale, fk, fk_scale, n_valid=None, shortlist: int = 4096, k: int = 512,
                               want_shortlist: bool = False, ws=None, out=None, stream=None):
    """Two-stage decode search. ck int8 [B,N,d] + ck_scale [B,N]; fk e4m3 [B,N,d] + fk_scale [B,N]."""
    _dev(q, torch.bfloat16, "q", 3)
    B, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    _dev(ck, torch.int8, "ck", 3)
    N = ck.shape[1]
    _dev(ck_scale, torch.float32, "ck_scale", 2)
    if fk.dtype == torch.uint8:
        fk = fk.view(torch.float8_e4m3fn)
    _dev(fk, torch.float8_e4m3fn, "fk", 3)
    _dev(fk_scale, torch.float32, "fk_scale", 2)
    _opt(n_valid, torch.int32, "n_valid")
    need = lib().ls_two_stage_workspace_size(B, N, shortlist)
    if ws is None:
        ws = _workspace(need, q.device)
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=q.device),
               torch.empty((B, k), dtype=torch.float32, device=q.device))
    idx, val = out
    sl = torch.empty((B, shortlist), dtype=torch.int32, device=q.device) if want_shortlist else None
    _check(lib().ls_decode_two_stage_select(_ptr(q), _ptr(w), _ptr(ck), _ptr(ck_scale), _ptr(fk), _ptr(fk_scale),
                                            _ptr(n_valid), B, H, d, N, shortlist, k, _ptr(idx), _ptr(val), _ptr(sl),
                                            _ptr(ws), ws.numel(), _stream(stream)))
    if want_shortlist:
        return idx, val, sl
    return idx, val


def _pq_args(pq_codes, pq_books):
    _dev(pq_codes, torch.uint8, "pq_codes", 3)
    if pq_codes.shape[2] != 32:
        raise ValueError("pq_codes must be [B, N, 32]")
    if pq_books.dtype == torch.int16:
        pq_books = pq_books.view(torch.float16)
    _dev(pq_books, torch.float16, "pq_books", 3)
    if tuple(pq_books.shape) != (32, 256, 4):
        raise ValueError("pq_books must be [32, 256, 4] fp16")
    return pq_codes, pq_books


def ls_indexer_score_pq(q, w, pq_codes, pq_books, n_valid=None, stream=None):
    """q [B,H,d] bf16, w [B,H] f32, pq_codes [B,N,32] uint8, pq_books [32,256,4] fp16 -> scores [B,N] f32."""
    _dev(q, torch.bfloat16, "q", 3)
    B, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    pq_codes, pq_books = _pq_args(pq_codes, pq_books)
    N = pq_codes.shape[1]
    _opt(n_valid, torch.int32, "n_valid")
    out = torch.empty((B, N), dtype=torch.float32, device=q.device)
    _check(lib().ls_indexer_score_pq(_ptr(q), _ptr(w), _ptr(pq_codes), _ptr(pq_books), _ptr(n_valid), B, H, d, N,
                                     _ptr(out), _stream(stream)))
    return out


def ls_decode_two_stage_pq_select(q, w, pq_codes, pq_books, fk, fk_scale, n_valid=None, shortlist: int = 4096,
                                  k: int = 512, want_shortlist: bool = False, ws=None, out=None, stream=None):
    """Two-stage decode search with PQ compact keys (pq_codes [B,N,32] uint8, pq_books [32,256,4] fp16) and the
    fp8 originals fk e4m3 [B,N,d] + fk_scale [B,N] for the exact re-rank."""
    _dev(q, torch.bfloat16, "q", 3)
    B, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    pq_codes, pq_books = _pq_args(pq_codes, pq_books)
    N = pq_codes.shape[1]
    if fk.dtype == torch.uint8:
        fk = fk.view(torch.float8_e4m3fn)
    _dev(fk, torch.float8_e4m3fn, "fk", 3)
    _dev(fk_scale, torch.float32, "fk_scale", 2)
    _opt(n_valid, torch.int32, "n_valid")
    need = lib().ls_two_stage_workspace_size(B, N, shortlist)
    if ws is None:
        ws = _workspace(need, q.device)
    if out is None:
        out = (torch.empty((B, k), dtype=torch.int32, device=q.device),
               torch.empty((B, k), dtype=torch.float32, device=q.device))
    idx, val = out
    sl = torch.empty((B, shortlist), dtype=torch.int32, device=q.device) if want_shortlist else None
    _check(lib().ls_decode_two_stage_pq_select(_ptr(q), _ptr(w), _ptr(pq_codes), _ptr(pq_books), _ptr(fk),
                                               _ptr(fk_scale), _ptr(n_valid), B, H, d, N, shortlist, k, _ptr(idx),
                                               _ptr(val), _ptr(sl), _ptr(ws), ws.numel(), _stream(stream)))
    if want_shortlist:
        return idx, val, sl
    return idx, val


def ls_bucket_select(q, w, centroids, bucket_off, bucket_mem, keys, top_p: int = 64, budget: int = 512,
                     k: int = 512, want_picked: bool = False, ws=None, out=None, stream=None):
    """Bucket search. centroids [P,d] bf16, bucket_off [P+1] int32, bucket_mem [M] int32, keys [N,d] bf16."""
    _dev(q, torch.bfloat16, "q", 3)
    T, H, d = q.shape
    _dev(w, torch.float32, "w", 2)
    _dev(centroids, torch.bfloat16, "centroids", 2)
    P = centroids.shape[0]
    _dev(bucket_off, torch.int32, "bucket_off", 1)
    _dev(bucket_mem, torch.int32, "bucket_mem", 1)
    _dev(keys, torch.bfloat16, "keys", 2)
    N = keys.shape[0]
    need = lib().ls_bucket_workspace_size(T, P, top_p, budget)
    if ws is None:
        ws = _workspace(need, q.device)
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=q.device),
               torch.empty((T, k), dtype=torch.float32, device=q.device))
    idx, val = out
    picked = torch.empty((T, top_p), dtype=torch.int32, device=q.device) if want_picked else None
    _check(lib().ls_bucket_select(_ptr(q), _ptr(w), _ptr(centroids), _ptr(bucket_off), _ptr(bucket_mem), _ptr(keys),
                                  T, H, d, P, N, top_p, budget, k, _ptr(idx), _ptr(val), _ptr(picked), _ptr(ws),
                                  ws.numel(), _stream(stream)))
    if want_picked:
        return idx, val, picked
    return idx, val


def ls_lsa_flat_select(q_idx, q_pos, centroids, bucket_off, bucket_mem, block_keys: int = 512,
                       buckets_per_block: int = 64, n_sink: int = 4, top_p: int = 1024, budget: int = 4096,
                       threshold: bool = False, fallback_rows: int = 0, want_picked: bool = False, ws=None, out=None,
                       stream=None):
    """Native LSA flat search.  q_idx [T,64] bf16, q_pos [T] int64, centroids [P,64] bf16 (block-major),
    bucket_off [P+1] / bucket_mem int32 (members ascending) -> (keys [T, n_sink+block_keys+budget] int32,
    n [T] int32[, picked [T, top_p] int32]).  threshold: the sampled-threshold scan with candidate lists (else
    the full score matrix); both pick the same buckets.  fallback_rows: queries the threshold form's fallback
    scores in full at a time (0: the default bound)."""
    _dev(q_idx, torch.bfloat16, "q_idx", 2)
    T, d = q_idx.shape
    _dev(q_pos, torch.int64, "q_pos", 1)
    _dev(centroids, torch.bfloat16, "centroids", 2)
    P = centroids.shape[0]
    _dev(bucket_off, torch.int32, "bucket_off", 1)
    _dev(bucket_mem, torch.int32, "bucket_mem", 1)
    need = lib().ls_lsa_flat_workspace_size(T, P, top_p, int(threshold), int(fallback_rows))
    if ws is None:
        ws = _workspace(need, q_idx.device)
    if out is None:
        out = (torch.empty((T, n_sink + block_keys + budget), dtype=torch.int32, device=q_idx.device),
               torch.empty((T,), dtype=torch.int32, device=q_idx.device))
    keys, n = out
    picked = torch.empty((T, top_p), dtype=torch.int32, device=q_idx.device) if want_picked else None
    _check(lib().ls_lsa_flat_select(_ptr(q_idx), _ptr(q_pos), _ptr(centroids), _ptr(bucket_off), _ptr(bucket_mem),
                                    T, d, P, block_keys, buckets_per_block, n_sink, top_p, budget, int(threshold),
                                    int(fallback_rows), _ptr(keys), _ptr(n), _ptr(picked), _ptr(ws), ws.numel(),
                                    _stream(stream)))
    return (keys, n, picked) if want_picked else (keys, n)


def ls_lsa_tree_select(q_idx, q_pos, centroids, node_centroids, bucket_off, bucket_mem, block_keys: int = 512,
                       buckets_per_block: int = 64, node_block: int = 4096, fanout: int = 4, beam: int = 2048,
                       n_sink: int = 4, top_p: int = 1024, budget: int = 4096, want_picked: bool = False,
                       ws=None, out=None, stream=None):
    """LSA tree search over one level of node buckets.  As ls_lsa_flat_select, plus node_centroids [P1,64]
    bf16; with want_picked also returns (picked [T, top_p], beam [T, beam]) int32."""
    _dev(q_idx, torch.bfloat16, "q_idx", 2)
    T, d = q_idx.shape
    _dev(q_pos, torch.int64, "q_pos", 1)
    _dev(centroids, torch.bfloat16, "centroids", 2)
    _dev(node_centroids, torch.bfloat16, "node_centroids", 2)
    P, P1 = centroids.shape[0], node_centroids.shape[0]
    _dev(bucket_off, torch.int32, "bucket_off", 1)
    _dev(bucket_mem, torch.int32, "bucket_mem", 1)
    need = lib().ls_lsa_tree_workspace_size(T, P1, beam, fanout, node_block, top_p)
    if ws is None:
        ws = _workspace(need, q_idx.device)
    if out is None:
        out = (torch.empty((T, n_sink + block_keys + budget), dtype=torch.int32, device=q_idx.device),
               torch.empty((T,), dtype=torch.int32, device=q_idx.device))
    keys, n = out
    picked = torch.empty((T, top_p), dtype=torch.int32, device=q_idx.device) if want_picked else None
    bm = torch.empty((T, beam), dtype=torch.int32, device=q_idx.device) if want_picked else None
    _check(lib().ls_lsa_tree_select(_ptr(q_idx), _ptr(q_pos), _ptr(centroids), _ptr(node_centroids),
                                    _ptr(bucket_off), _ptr(bucket_mem), T, d, P, P1, block_keys, buckets_per_block,
                                    node_block, fanout, beam, n_sink, top_p, budget, _ptr(keys), _ptr(n),
                                    _ptr(picked), _ptr(bm), _ptr(ws), ws.numel(), _stream(stream)))
    return (keys, n, picked, bm) if want_picked else (keys, n)


def ls_lsa_tree_levels_workspace_size(T: int, P: int, level_sizes, node_block: int = 4096, fanout: int = 4,
                                      beam: int = 2048, start_nodes: int = 32768, top_p: int = 1024) -> int:
    L = len(level_sizes)
    sizes = (ctypes.c_int * max(L, 1))(*[int(x) for x in level_sizes])
    return lib().ls_lsa_tree_levels_workspace_size(T, P, sizes, L, node_block, fanout, beam, start_nodes, top_p)


def ls_lsa_tree_levels_select(q_idx, q_pos, centroids, node_levels, bucket_off, bucket_mem, block_keys: int = 512,
                              buckets_per_block: int = 64, node_block: int = 4096, fanout: int = 4,
                              beam: int = 2048, start_nodes: int = 32768, n_sink: int = 4, top_p: int = 1024,
                              budget: int = 4096, want_picked: bool = False, ws=None, out=None, stream=None):
    """LSA tree search over several node levels.  As ls_lsa_flat_select, plus node_levels: a list of L
    [P_l,64] bf16 tensors (levels 1..L); with want_picked also returns (picked [T, top_p],
    beams [L, T, beam]) int32 (levels above the start level are left unwritten)."""
    _dev(q_idx, torch.bfloat16, "q_idx", 2)
    T, d = q_idx.shape
    _dev(q_pos, torch.int64, "q_pos", 1)
    _dev(centroids, torch.bfloat16, "centroids", 2)
    for i, nc in enumerate(node_levels):
        _dev(nc, torch.bfloat16, f"node_levels[{i}]", 2)
    _dev(bucket_off, torch.int32, "bucket_off", 1)
    _dev(bucket_mem, torch.int32, "bucket_mem", 1)
    P, L = centroids.shape[0], len(node_levels)
    sizes = [int(nc.shape[0]) for nc in node_levels]
    need = ls_lsa_tree_levels_workspace_size(T, P, sizes, node_block, fanout, beam, start_nodes, top_p)
    if ws is None:
        ws = _workspace(need, q_idx.device)
    if out is None:
        out = (torch.empty((T, n_sink + block_keys + budget), dtype=torch.int32, device=q_idx.device),
               torch.empty((T,), dtype=torch.int32, device=q_idx.device))
    keys, n = out
    picked = torch.empty((T, top_p), dtype=torch.int32, device=q_idx.device) if want_picked else None
    beams = torch.full((max(L, 1), T, beam), -2, dtype=torch.int32, device=q_idx.device) if want_picked else None
    ptrs = (ctypes.c_void_p * max(L, 1))(*[nc.data_ptr() for nc in node_levels])
    csizes = (ctypes.c_int * max(L, 1))(*sizes)
    _check(lib().ls_lsa_tree_levels_select(_ptr(q_idx), _ptr(q_pos), _ptr(centroids), ptrs, csizes, L,
                                           _ptr(bucket_off), _ptr(bucket_mem), T, d, P, block_keys,
                                           buckets_per_block, node_block, fanout, beam, start_nodes, n_sink, top_p,
                                           budget, _ptr(keys), _ptr(n), _ptr(picked), _ptr(beams), _ptr(ws),
                                           ws.numel(), _stream(stream)))
    return (keys, n, picked, beams) if want_picked else (keys, n)


def ls_merge_select(vals, idx, offsets, k: int = 512, ws=None, out=None, stream=None):
    """Merge S shards' top-k lists of the same T queries into the global top-k.

    vals [S,T,k_in] f32 and idx [S,T,k_in] int32 (positions local to each shard, -1 padded),
    offsets [S] int32 (each shard's first history position) -> (idx [T,k] int32, val [T,k] f32)."""
    _dev(vals, torch.float32, "vals", 3)
    _dev(idx, torch.int32, "idx", 3)
    _dev(offsets, torch.int32, "offsets", 1)
    S, T, k_in = vals.shape
    need = lib().ls_merge_select_workspace_size(S, T, k_in)
    if ws is None:
        ws = _workspace(need, vals.device)
    if out is None:
        out = (torch.empty((T, k), dtype=torch.int32, device=vals.device),
               torch.empty((T, k), dtype=torch.float32, device=vals.device))
    io, vo = out
    _check(lib().ls_merge_select(_ptr(vals), _ptr(idx), _ptr(offsets), S, T, k_in, k, _ptr(io), _ptr(vo), _ptr(ws),
                                 ws.numel(), _stream(stream)))
    return io, vo




def ls_sparse_attention(q, latent, idx, scale: Optional[float] = None, row_off=None, want_lse: bool = True,
                        out=None, foreign_rows: bool = False, cuda_cores: bool = False, stream=None):
    """Sparse main attention over the selected latent rows.

    q [T,H,576] bf16, latent [R,576] bf16, idx [T,k] int32 (-1 = unused slot),
    row_off [T] int64 or None (row = idx + row_off[t]); scale defaults to
    1/sqrt(576) -> (out [T,H,512] f32, lse [T,H] f32 or None).  With
    ``foreign_rows`` latent holds one shard of the rows (row_off = -its first
    row) and rows outside it are skipped as another shard's.  ``cuda_cores``
    forces the fp32 CUDA-core kernel where the tensor-core one would run."""
    _dev(q, torch.bfloat16, "q", 3)
    _dev(latent, torch.bfloat16, "latent", 2)
    _dev(idx, torch.int32, "idx", 2)
    _opt(row_off, torch.int64, "row_off")
    T, H, d = q.shape
    R, d_lat = latent.shape
    if d_lat != d:
        raise ValueError(f"q has {d} elements per head, latent rows {d_lat}")
    if idx.shape[0] != T:
        raise ValueError(f"idx has {idx.shape[0]} rows for {T} queries")
    k = idx.shape[1]
    if scale is None:
        scale = 1.0 / math.sqrt(d)
    if out is None:
        out = torch.empty((T, H, 512), dtype=torch.float32, device=q.device)
    lse = torch.empty((T, H), dtype=torch.float32, device=q.device) if want_lse else None
    _check(lib().ls_sparse_attention(_ptr(q), _ptr(latent), _ptr(idx), _ptr(row_off), T, H, d, 512, R, k, float(scale),
                                     (LS_ATTN_FOREIGN_ROWS if foreign_rows else 0)
                                     | (LS_ATTN_CUDA_CORES if cuda_cores else 0), _ptr(out), _ptr(lse),
                                     _stream(stream)))
    return out, lse


def ls_attention_merge(o_parts, lse_parts, out=None, stream=None):
    """Combine S partial attentions over disjoint row sets (online softmax).

    o_parts [S,...,d_v] f32, lse_parts [S,...] f32 -> (o [...,d_v] f32, lse [...] f32)."""
    _dev(o_parts, torch.float32, "o_parts")
    _dev(lse_parts, torch.float32, "lse_parts")
    S, d_v = o_parts.shape[0], o_parts.shape[-1]
    if tuple(o_parts.shape[:-1]) != tuple(lse_parts.shape):
        raise ValueError(f"o_parts {tuple(o_parts.shape)} and lse_parts {tuple(lse_parts.shape)} disagree")
    rows = lse_parts[0].numel()
    if out is None:
        out = (torch.empty(o_parts.shape[1:], dtype=torch.float32, device=o_parts.device),
               torch.empty(lse_parts.shape[1:], dtype=torch.float32, device=o_parts.device))
    o, lse = out
    _check(lib().ls_attention_merge(_ptr(o_parts), _ptr(lse_parts), S, rows, d_v, _ptr(o), _ptr(lse),
                                    _stream(stream)))
    return o, lse


def shard_plan(n_keys: int, n_shards: int):
    """Contiguous shards of a history of n_keys compressed positions: [(first position, length), ...]."""
    base, out = 0, []
    for s in range(n_shards):
        length = n_keys // n_shards + (1 if s < n_keys % n_shards else 0)
        out.append((base, length))
        base += length
    return out


def ls_device_status(stream=None) -> int:
    """Fault bits of the device fault word (read and cleared).  Raises on none."""
    flags = ctypes.c_int(0)
    st = lib().ls_device_status(ctypes.byref(flags), _stream(stream))
    if st not in (LS_OK, LS_ERR_TIMEOUT, LS_ERR_INVALID_ARG):
        _check(st)
    return flags.value


def ls_selftest_wait_probe(limit_ns: int, stream=None) -> torch.Tensor:
    gave_up = torch.zeros(1, dtype=torch.int32, device="cuda")
    _check(lib().ls_selftest_wait_probe(limit_ns, _ptr(gave_up), _stream(stream)))
    return gave_up


def ls_profile_begin() -> None:
    _check(lib().ls_profile_begin())


def ls_profile_end() -> dict:
    """Stop recording; {kernel name: (total ms, launches)} of the library's launches."""
    n = ctypes.c_int(0)
    _check(lib().ls_profile_end(ctypes.byref(n)))
    out = {}
    for i in range(n.value):
        name = ctypes.c_char_p()
        ms = ctypes.c_double()
        cnt = ctypes.c_longlong()
        _check(lib().ls_profile_kernel(i, ctypes.byref(name), ctypes.byref(ms), ctypes.byref(cnt)))
        out[name.value.decode()] = (ms.value, cnt.value)
    return out
