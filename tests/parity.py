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


def _positions(keys, sel, what):
    """Positions in ``keys`` of each index in ``sel`` (keys unique); raises if
    one is not among them."""
    n = keys.shape[0]
    if n == 0:
        if sel.size:
            raise AssertionError(f"{what}: index {int(sel[0])} is not a visible candidate")
        return np.zeros(0, dtype=np.int64)
    order = np.argsort(keys, kind="stable")
    sk = keys[order]
    loc = np.searchsorted(sk, sel)
    ok = (loc < n) & (sk[np.minimum(loc, n - 1)] == sel)
    if not ok.all():
        raise AssertionError(f"{what}: index {int(sel[~ok][0])} is not a visible candidate")
    return order[loc]


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
    p = _positions(keys, sel, what)
    ref = S[p]
    err = np.abs(sv - ref)
    tol = _tol(S, ref)
    bad = err > tol
    assert not bad.any(), (f"{what}: {int(bad.sum())} score mismatches, e.g. key {sel[bad][0]} "
                           f"gpu {sv[bad][0]!r} oracle {ref[bad][0]!r}")
    oi, ov = O.select_topk(S, k, idx=keys)
    if m == n:
        assert set(sel.tolist()) == set(keys.tolist()), f"{what}: not all visible keys returned"
        return
    kth = ov[-1]
    diff = np.setxor1d(sel, oi)
    if diff.size:
        dev = np.abs(S[_positions(keys, diff, what)] - kth)
        lim = RTOL * abs(kth) + ATOL_FRAC * float(np.max(np.abs(S)))
        assert np.all(dev <= lim), (f"{what}: {len(diff)} set differences beyond the k-th-score tolerance; "
                                    f"worst |S-kth| = {dev.max()!r} > {lim!r}")


def sample_rows(T, k, n=512, seed=0, q_pos0=0, needles=None, group=None, extra=()):
    """A seeded sample of n distinct query rows of a T-row problem for the
    full-size parity checks: the first and last four rows (a whole first and
    last 4-row unit), rows whose position is below k (they see fewer than k
    keys) and around k, the 128-key tile edges near the start, rows at and just
    after planted keys (``needles``: key positions; a query at a needle's
    position is the first to see it), every group's first and last member for
    the groups the sample touches (``group``: size G), ``extra``, then
    uniform rows up to n."""
    rng = np.random.default_rng(seed)
    want = list(range(min(4, T))) + list(range(max(0, T - 4), T))
    lo = [p - q_pos0 for p in (0, 1, 126, 127, 128, 129, 255, 256, k // 2, k - 2, k - 1, k, k + 1)]
    want += [t for t in lo if 0 <= t < T]
    below = max(0, min(T, k - q_pos0))
    if below > 0:
        want += rng.integers(0, below, min(16, below)).tolist()
    if needles is not None:
        nd = np.asarray(needles, dtype=np.int64)
        nd = nd[(nd >= q_pos0) & (nd < q_pos0 + T)]
        if nd.size > 40:
            nd = np.sort(rng.choice(nd, 40, replace=False))
        for p in nd:
            want += [int(p - q_pos0), int(p - q_pos0 + 1)]
    want += [int(t) for t in extra]
    want = [t for t in want if 0 <= t < T]
    rows = []
    seen = set()
    for t in want:
        if t not in seen:
            seen.add(t)
            rows.append(t)
    while len(rows) < min(n, T):
        t = int(rng.integers(0, T))
        if t not in seen:
            seen.add(t)
            rows.append(t)
    rows = rows[:min(n, T)]
    if group:
        # both ends of every group the sample touches (the group boundaries)
        for g in sorted({t // group for t in rows}):
            for t in (g * group, min(T, (g + 1) * group) - 1):
                if t not in seen:
                    seen.add(t)
                    rows.append(t)
    return np.array(sorted(rows), dtype=np.int64)


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


def sample_groups(ng, G, q_pos0=0, needles=None, seed=0):
    """Eight groups of a full-size group-shared run, in adjacent pairs so that
    each pair's shared boundary lies in the sample: the first two, the last
    two, and two pairs in between (around groups that hold planted keys when
    ``needles`` is given, else at a third and two thirds of the groups).
    With G = 64 that is 512 member rows."""
    rng = np.random.default_rng(seed)
    mids = [ng // 3, (2 * ng) // 3]
    if needles is not None:
        g_of = (np.asarray(needles, dtype=np.int64) - q_pos0) // G
        g_of = np.unique(g_of[(g_of >= 2) & (g_of < ng - 3)])
        if g_of.size >= 2:
            mids = sorted(rng.choice(g_of, 2, replace=False).tolist())
    groups = [0, 1, mids[0], mids[0] + 1, mids[1], mids[1] + 1, ng - 2, ng - 1]
    return sorted({g for g in groups if 0 <= g < ng})


def check_group_sample(Q, W, Kd, gi, gv, bi, bv, groups, G, B, k, mode, q_pos0, q_dtype, what=""):
    """Full-size group-shared parity on whole groups.  The oracle forms each
    sampled group's proxy itself (member mean rounded to ``q_dtype``) and
    checks the GPU's bank against that proxy's top-B by the parity rule;
    every member is then checked on the GPU's bank (Refine: the member's own
    scores of the bank keys it sees, plus, for Refine with local additions,
    its own stretch of the group; Reuse: the proxy's ranking of those keys).
    Q, W: the torch query rows and weights (converted one group at a time);
    Kd: float64 keys [N, d]; gi/gv [T, k], bi/bv [ng, B] numpy outputs."""
    T = Q.shape[0]
    for g in groups:
        r0, r1 = g * G, min(T, (g + 1) * G)
        q = Q[r0:r1].detach().to("cpu").double().numpy()
        w = W[r0:r1].detach().to("cpu").double().numpy()
        qb, wb = O.proxy(q, w, G, q_dtype=q_dtype)
        L = q_pos0 + r1 - 1
        ps = O.score_rows(qb, wb, Kd[:L + 1])[0]
        check_row(bi[g], bv[g], ps, B, what=f"{what} bank g={g}")
        bank = bi[g][bi[g] >= 0].astype(np.int64)
        for t in range(r0, r1):
            p = q_pos0 + t
            cand = bank[bank <= p]
            if mode == O.REUSE:
                check_row(gi[t], gv[t], ps[cand], k, what=f"{what} reuse t={t}", idx_map=cand)
                continue
            if mode == O.REFINE_LOCAL:
                cand = np.union1d(cand, np.arange(q_pos0 + r0, p + 1))
            S = O.score_rows(q[t - r0:t - r0 + 1], w[t - r0:t - r0 + 1], Kd[cand])[0]
            check_row(gi[t], gv[t], S, k, what=f"{what} refine(mode {mode}) t={t}", idx_map=cand)
