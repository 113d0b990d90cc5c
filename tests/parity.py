"""Parity checks of GPU outputs against the CPU oracle.

Rules (scores in fp32 from bf16/fp8/fp32 inputs, oracle in float64):
  * every returned score:  |val - S[idx]| <= RTOL * |S[idx]| + ATOL_FRAC * max|S|
    (max|S| over the row: a floor for scores that cancel to ~0);
  * every row holds exactly min(k, visible) distinct indices, all visible,
    padded with -1 / -inf;
  * the index set equals the oracle's top-k except for keys whose oracle
    scores lie within the same tolerance of the oracle's k-th score
    (near-ties that fp32 accumulation may order either way).
"""
from __future__ import annotations

import numpy as np

from oracle import dsa_oracle as O

RTOL = 1e-3
ATOL_FRAC = 1e-6


def _tol(S, ref):
    scale = float(np.max(np.abs(S))) if S.size else 0.0
    return RTOL * np.abs(ref) + ATOL_FRAC * scale


def check_row(gi, gv, S, k, what="", idx_map=None):
    """One output row against the oracle's full score vector S over the row's
    candidate keys.  ``idx_map`` maps positions of S to key indices (default:
    position == key index)."""
    S = np.asarray(S, dtype=np.float64)
    keys = np.arange(S.shape[0]) if idx_map is None else np.asarray(idx_map, dtype=np.int64)
    n = S.shape[0]
    m = min(k, n)
    gi = np.asarray(gi).astype(np.int64)
    gv = np.asarray(gv).astype(np.float64)
    real = gi >= 0
    assert int(real.sum()) == m, f"{what}: {int(real.sum())} entries, expected {m}"
    assert np.all(gi[~real] == -1) and np.all(np.isneginf(gv[~real])), f"{what}: bad padding"
    sel = gi[real]
    sv = gv[real]
    assert np.unique(sel).shape[0] == m, f"{what}: duplicate indices"
    pos_of = {int(kk): i for i, kk in enumerate(keys)}
    try:
        p = np.array([pos_of[int(s)] for s in sel], dtype=np.int64)
    except KeyError as e:
        raise AssertionError(f"{what}: index {e} is not a visible candidate") from None
    ref = S[p]
    err = np.abs(sv - ref)
    tol = _tol(S, ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} score mismatches, e.g. key {sel[bad][0]} "
                           f"gpu {sv[bad][0]!r} oracle {ref[bad][0]!r}")
    oi, _ = O.select_topk(S, k, idx=keys)
    if m == n:
        assert set(sel.tolist()) == set(keys.tolist()), f"{what}: not all visible keys returned"
        return
    kth = S[pos_of[int(oi[-1])]]
    diff = set(sel.tolist()) ^ set(oi.tolist())
    if diff:
        dpos = np.array([pos_of[d] for d in diff])
        dev = np.abs(S[dpos] - kth)
        lim = RTOL * abs(kth) + ATOL_FRAC * float(np.max(np.abs(S)))
        assert np.all(dev <= lim), (f"{what}: {len(diff)} set differences beyond the k-th-score tolerance; "
                                    f"worst |S-kth| = {dev.max()!r} > {lim!r}")


def check_rows(gidx, gval, scores, k, what="", idx_maps=None):
    for r, S in enumerate(scores):
        check_row(gidx[r], gval[r], S, k, what=f"{what} row {r}",
                  idx_map=None if idx_maps is None else idx_maps[r])


def check_scores(S_gpu, S_ref, what=""):
    """Full score matrices: finite where the oracle is finite, -inf elsewhere."""
    S_gpu = np.asarray(S_gpu, dtype=np.float64)
    fin = np.isfinite(S_ref)
    assert np.all(np.isneginf(S_gpu[~fin])), f"{what}: entries beyond the prefix are not -inf"
    row_scale = np.max(np.where(fin, np.abs(S_ref), 0.0), axis=1, keepdims=True)
    tol = RTOL * np.abs(S_ref) + ATOL_FRAC * row_scale
    err = np.where(fin, np.abs(S_gpu - np.where(fin, S_ref, 0.0)), 0.0)
    bad = err > np.where(fin, tol, np.inf)
    assert not bad.any(), f"{what}: {int(bad.sum())} score mismatches (max err {err.max()!r})"
