"""Comparison rules between the CUDA path and the CPU oracle.

Selection parity: for a query whose oracle candidates (sorted by score desc,
index asc) are s_1 >= s_2 >= ..., the GPU's k-set must equal the oracle's
exactly when the relative gap at the boundary, (s_k - s_{k+1}) / |s_k|,
exceeds 1e-3; otherwise every index in the symmetric difference must have an
oracle score within 1e-3 * |s_k| of s_k.  Returned scores must match the
oracle's score of the same index within `rtol` (2e-2 for bf16 / E4M3, 1e-4
for fp32 inputs).
"""
from __future__ import annotations

import numpy as np

GAP = 1e-3
RTOL = {"f32": 1e-4, "bf16": 2e-2, "e4m3": 2e-2}


def check_selection(gpu_set, cand: np.ndarray, cand_scores: np.ndarray, k: int, what: str, gap: float = GAP):
    """gpu_set: the GPU's chosen indices (no -1); cand / cand_scores: the
    oracle's candidate indices and float64 scores."""
    gpu = np.asarray(sorted(int(x) for x in gpu_set), np.int64)
    assert len(set(gpu.tolist())) == len(gpu), f"{what}: duplicate indices {gpu}"
    cand = np.asarray(cand, np.int64)
    n = len(cand)
    if n <= k:
        assert gpu.tolist() == sorted(cand.tolist()), f"{what}: expected all {n} candidates, got {len(gpu)}"
        return 0
    assert len(gpu) == k, f"{what}: expected {k} indices, got {len(gpu)}"
    order = np.lexsort((cand, -cand_scores))
    top = set(cand[order[:k]].tolist())
    sk, sk1 = cand_scores[order[k - 1]], cand_scores[order[k]]
    diff = top.symmetric_difference(gpu.tolist())
    if not diff:
        return 0
    scale = max(abs(sk), 1e-30)
    rel_gap = (sk - sk1) / scale
    assert rel_gap <= gap, f"{what}: boundary gap {rel_gap:.3g} > {gap} but sets differ by {sorted(diff)[:8]}"
    pos = {int(c): i for i, c in enumerate(cand.tolist())}
    for x in diff:
        assert x in pos, f"{what}: index {x} is not a candidate"
        assert abs(cand_scores[pos[x]] - sk) <= gap * scale, \
            f"{what}: swapped index {x} has score {cand_scores[pos[x]]} outside the band around {sk}"
    return len(diff) // 2


def check_scores(gpu_idx, gpu_scores, oracle_score_of, rtol: float, what: str):
    gpu_idx = np.asarray(gpu_idx)
    keep = gpu_idx >= 0
    if not keep.any():
        return
    ref = oracle_score_of(gpu_idx[keep])
    got = np.asarray(gpu_scores)[keep].astype(np.float64)
    atol = 1e-6 * max(np.max(np.abs(ref)), 1e-30)
    bad = np.abs(got - ref) > rtol * np.abs(ref) + atol
    assert not bad.any(), f"{what}: scores off at {np.nonzero(bad)[0][:5]}: {got[bad][:5]} vs {ref[bad][:5]}"


def iou(a, b) -> float:
    a, b = set(int(x) for x in a if x >= 0), set(int(x) for x in b if x >= 0)
    if not a and not b:
        return 1.0
    return len(a & b) / len(a | b)


def recall(hisa, flat) -> float:
    """|HISA & flat| / |flat| of two index rows (-1 = none)."""
    a, b = set(int(x) for x in hisa if x >= 0), set(int(x) for x in flat if x >= 0)
    if not b:
        return 1.0
    return len(a & b) / len(b)
