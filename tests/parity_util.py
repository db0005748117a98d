"""Helpers shared by the GPU parity tests: host->device transfer of the seeded
inputs and the comparison rules.

Score tolerance (the stated bound: 2e-3 relative for bf16 inputs, 2e-2 for
fp8 inputs; the normaliser is this suite's reading):

    |s_gpu - s_ref| <= rtol * max(|s_ref|, m_row)

with m_row the median |s_ref| over the row's eligible positions, a floor for
scores that cancel to near zero.

Selection ("band") rule: with tau the k-th largest reference score of the
row and delta = rtol * max(|tau|, m_row), the GPU's selected set must contain
every eligible position whose reference score exceeds tau + delta and none
whose score is below tau - delta; the selected values must match the reference
within the score tolerance, be in canonical order (value desc, position asc)
and hold no duplicates.
"""

from __future__ import annotations

import numpy as np
import torch

RTOL_BF16 = 2e-3
RTOL_FP8 = 2e-2


def dev_bf16(bits: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(bits).view(np.int16)).view(torch.bfloat16).cuda()


def dev(a: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def dev_e4m3(codes: np.ndarray) -> torch.Tensor:
    return torch.from_numpy(np.ascontiguousarray(codes)).cuda().view(torch.float8_e4m3fn)


def row_floor(ref: np.ndarray) -> float:
    f = np.abs(ref[np.isfinite(ref)])
    return float(np.median(f)) if f.size else 0.0


def check_scores(gpu: np.ndarray, ref: np.ndarray, rtol: float, what: str = "") -> None:
    gpu = np.asarray(gpu, dtype=np.float64)
    ref = np.asarray(ref, dtype=np.float64)
    assert gpu.shape == ref.shape, (gpu.shape, ref.shape)
    m = row_floor(ref)
    tol = rtol * np.maximum(np.abs(ref), m)
    err = np.abs(gpu - ref)
    bad = ~(err <= tol)
    if bad.any():
        i = int(np.flatnonzero(bad)[0])
        raise AssertionError(f"{what}: {bad.sum()} scores off, first at {i}: gpu {gpu.flat[i]!r} ref {ref.flat[i]!r}")


def check_selection(idx: np.ndarray, val: np.ndarray, cand_pos: np.ndarray, cand_ref: np.ndarray, k: int,
                    rtol: float, what: str = "") -> None:
    """One row: GPU (idx, val) against reference scores of every candidate."""
    idx = np.asarray(idx, dtype=np.int64)
    val = np.asarray(val, dtype=np.float64)
    cand_pos = np.asarray(cand_pos, dtype=np.int64)
    cand_ref = np.asarray(cand_ref, dtype=np.float64)
    n = cand_pos.size
    want = min(k, n)
    sel = idx[idx >= 0]
    assert sel.size == want, f"{what}: selected {sel.size}, expected {want}"
    assert np.all(idx[want:] == -1), f"{what}: padding is not -1"
    assert np.all(np.isneginf(val[want:])), f"{what}: padding values are not -inf"
    assert len(set(sel.tolist())) == sel.size, f"{what}: duplicate positions"
    if want == 0:
        return
    ref_of = dict(zip(cand_pos.tolist(), cand_ref.tolist()))
    assert all(int(p) in ref_of for p in sel), f"{what}: selected a position outside the candidates"
    m = row_floor(cand_ref)
    ref_sel = np.array([ref_of[int(p)] for p in sel])
    tol = rtol * np.maximum(np.abs(ref_sel), m)
    assert np.all(np.abs(val[:want] - ref_sel) <= tol), f"{what}: selected values off the reference"
    # canonical order of the GPU's own values
    v = val[:want]
    for a in range(want - 1):
        assert v[a] > v[a + 1] or (v[a] == v[a + 1] and sel[a] < sel[a + 1]), f"{what}: order broken at {a}"
    if want < n:
        tau = np.sort(cand_ref)[::-1][want - 1]
        delta = rtol * max(abs(tau), m)
        sset = set(sel.tolist())
        must = cand_pos[cand_ref > tau + delta]
        never = cand_pos[cand_ref < tau - delta]
        missing = [int(p) for p in must if int(p) not in sset]
        wrong = [int(p) for p in never if int(p) in sset]
        assert not missing, f"{what}: missing {len(missing)} positions clearly inside the top-k"
        assert not wrong, f"{what}: selected {len(wrong)} positions clearly outside the top-k"


def f32_bits_equal(a: np.ndarray, b: np.ndarray) -> bool:
    return np.array_equal(np.asarray(a, np.float32).view(np.uint32), np.asarray(b, np.float32).view(np.uint32))


def check_set(sel: np.ndarray, cand_pos: np.ndarray, cand_ref: np.ndarray, k: int, rtol: float,
              what: str = "") -> None:
    """Band rule on a selected set whose order is not checked (a shortlist or
    the picked buckets): size, no duplicates, members of the candidates, and
    every clear top-k member in / every clear outsider out."""
    sel = np.asarray(sel, dtype=np.int64)
    cand_pos = np.asarray(cand_pos, dtype=np.int64)
    cand_ref = np.asarray(cand_ref, dtype=np.float64)
    want = min(k, cand_pos.size)
    got = sel[sel >= 0]
    assert got.size == want, f"{what}: selected {got.size}, expected {want}"
    assert len(set(got.tolist())) == got.size, f"{what}: duplicates"
    cset = set(cand_pos.tolist())
    assert all(int(p) in cset for p in got), f"{what}: selected a non-candidate"
    if 0 < want < cand_pos.size:
        m = row_floor(cand_ref)
        tau = np.sort(cand_ref)[::-1][want - 1]
        delta = rtol * max(abs(tau), m)
        sset = set(got.tolist())
        assert all(int(p) in sset for p in cand_pos[cand_ref > tau + delta]), f"{what}: clear member missing"
        assert not any(int(p) in sset for p in cand_pos[cand_ref < tau - delta]), f"{what}: clear outsider in"
