"""Comparison rules shared by the GPU parity tests.

Index sets: bit-exact, except members whose oracle score lies within 1e-4 relative
of the boundary score (the B-th best key, or the Nq-th least similar query); such
near-ties are counted and returned.  Attention rows: max over rows of
|o - o_ref|_inf / |o_ref|_inf, evaluated with the oracle fed the GPU's own selection
so that selection near-ties do not leak into the output error.
"""
from __future__ import annotations

import numpy as np

from oracle import quoka_oracle as O

NEAR_TIE_REL = 1e-4
ATTN_TOL = {"f32": 1e-4, "bf16": 2e-2}


def check_index_row(row: np.ndarray, n: int, P: int) -> np.ndarray:
    """A GPU idx row: n ascending distinct entries in [0, P), then -1."""
    row = np.asarray(row, dtype=np.int64)
    head, tail = row[:n], row[n:]
    assert (tail == -1).all(), f"padding not -1: {tail[:8]}"
    assert ((head >= 0) & (head < P)).all(), f"index out of [0, {P})"
    assert (np.diff(head) > 0).all(), "indices not strictly ascending"
    return head


def compare_top_set(gpu: np.ndarray, score: np.ndarray, budget: int) -> int:
    """Compares a GPU top-B set to the oracle's; returns the number of near-tie keys
    in the symmetric difference (asserts every difference is a near-tie)."""
    ref = O.top_budget(score, budget)
    n = ref.shape[0]
    assert gpu.shape[0] == n, (gpu.shape, n)
    if n == score.shape[0]:
        assert np.array_equal(np.sort(gpu), ref)
        return 0
    diff = np.setxor1d(gpu, ref)
    if diff.size == 0:
        return 0
    sB = np.sort(score)[::-1][n - 1]
    band = NEAR_TIE_REL * abs(sB)
    bad = diff[np.abs(score[diff] - sB) > band]
    assert bad.size == 0, f"{bad.size} non-tie differences, e.g. {bad[:5]} scores " \
                          f"{score[bad[:5]]} vs boundary {sB}"
    return int(diff.size)


def compare_kept_set(gpu: np.ndarray, cos: np.ndarray, nq: int) -> int:
    """Compares a GPU kept-query set to the oracle's (smallest cosines)."""
    C = cos.shape[0]
    nk = min(nq, C)
    ref = np.sort(np.lexsort((np.arange(C), cos))[:nk])
    assert gpu.shape[0] == nk
    if nk == C:
        assert np.array_equal(np.sort(gpu), ref)
        return 0
    diff = np.setxor1d(gpu, ref)
    if diff.size == 0:
        return 0
    cb = np.sort(cos)[nk - 1]
    band = NEAR_TIE_REL * max(abs(cb), 1e-3)
    bad = diff[np.abs(cos[diff] - cb) > band]
    assert bad.size == 0, f"kept set differs beyond near-ties: {bad[:5]} {cos[bad[:5]]} vs {cb}"
    return int(diff.size)


def stratified_rows(h_q: int, h_kv: int, C: int, rng) -> list:
    """(head, position) rows that touch every query tile of the tensor-core attention.

    A tile packs the G = h_q / h_kv query heads of one KV head at TP = 128 // G
    consecutive positions (one CTA of an SM pair holds one tile).  Per KV head and per
    tile this takes one row at a random head of the group and a random position of the
    tile, and adds, for every head of the group, the first and the last position of the
    last tile (its ragged tail, when C is not a multiple of TP).
    """
    G = h_q // h_kv
    tp = max(1, 128 // G)
    rows = []
    for g in range(h_kv):
        heads = range(g * G, (g + 1) * G)
        for t0 in range(0, C, tp):
            rows.append((g * G + int(rng.integers(G)), t0 + int(rng.integers(min(tp, C - t0)))))
        last = (C - 1) // tp * tp
        for h in heads:
            rows += [(h, last), (h, C - 1)]
    return sorted(set(rows))


def row_rel_err(o: np.ndarray, ref: np.ndarray) -> float:
    """max over rows of |o - ref|_inf / |ref|_inf (rows along the last axis)."""
    o = np.asarray(o, dtype=np.float64).reshape(-1, o.shape[-1])
    ref = np.asarray(ref, dtype=np.float64).reshape(-1, ref.shape[-1])
    num = np.abs(o - ref).max(axis=1)
    den = np.maximum(np.abs(ref).max(axis=1), 1e-30)
    return float((num / den).max()) if num.size else 0.0
