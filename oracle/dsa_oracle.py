"""Plain CPU oracle for the DSA lightning indexer — TEST INFRASTRUCTURE ONLY.

Only ``tests/``, ``__graft_entry__.smoke()`` and the CPU-baseline and
reference legs of ``bench.py`` may import this module.  The product path (the CUDA library and
its Python binding) never calls it, and it shares no code with that path.

Everything here is slow and direct: float64 numpy, a full stable sort per
query row, no tiling and no fusion.  It follows the pages as follows.

* Score.  In the pages, the DeepSeek Sparse Attention (DSA) lightning
  indexer scores every key of the causal prefix for every query and keeps the
  top k = 2048 (MLI page, section Core Idea; PIVOT abstract; IndexCache page,
  section The Quadratic Tax), but none of them prints the score itself.  This
  library takes the standard DSA indexer form

      I[t, s] = sum_h w[t, h] * ReLU( q[t, h, :] . k[s, :] )

  with no extra scale factor.  For fp8 keys with a per-token scale, the key
  is k[s, :] = decode_e4m3(bytes[s, :]) * scale[s].
* Causality.  Query row t sits at key position p = q_pos0 + t and sees keys
  0..p (AttentionIndex page, Key findings: causality is enforced, a query
  never uses keys beyond its own prefix).
* Top-k.  Keys are ranked by (score descending, key index ascending) with one
  full stable sort; the first min(k, p + 1) are kept.  Rows that see fewer than
  k keys return all of them, padded with index -1 and score -inf.
* Group-shared form (PIVOT abstract): fixed-size groups of consecutive
  queries; the proxy is the mean of the members' q and w; one full-prefix scan
  by the proxy over the prefix of the group's last member gives a candidate
  bank of the best B keys; Refine re-scores the bank with each member's own
  q, w and takes its own top-k; Reuse gives each member the proxy's ranking
  over the bank, restricted to keys the member may see, cut to k.
* Decode (PIVOT abstract, MLI "Core Idea"): sequence b holds N_b cached keys
  and m_b new queries; new query j sits at position N_b - m_b + j.
* Group form in decode (PIVOT abstract: the queries of one multi-token
  prediction step are a natural group): a sequence's new queries are one
  group.  Refine may also take each member's own stretch of the group as
  query-specific candidates (ADIndex page, Inference).
* Two-stage routing comparators (AttentionIndex page, Architecture): blocks
  of 128 keys ranked by their mean key, and a plain k-means inverted file;
  each followed by the native score on the routed keys.
* Rounding.  The proxy query is stored in the queries' own dtype, so the
  group form rounds the float64 member mean to that dtype (``round_q``; a
  required ``q_dtype`` argument of ``proxy``, ``group`` and ``decode_group``).
  A block's mean key is stored in bf16; ``round_bf16`` rounds to nearest
  even, so that the oracle can run those steps from scratch.
* No query rows: nothing is selected; the group form has no groups.

Pins: every function here is checked in ``tests/test_oracle.py`` against
hand-worked values (``tests/golden/``), the fp8 format's published value
table, brute-force enumeration of subsets, closed forms and invariants.
"""
from __future__ import annotations

import numpy as np

__all__ = [
    "decode_e4m3", "key_values", "score_rows", "select_topk", "dense", "round_bf16", "round_q",
    "proxy", "group", "decode", "decode_group", "block_reps", "block_routed", "kmeans", "ivf_routed",
    "REFINE", "REUSE", "REFINE_LOCAL",
]

REFINE = 0
REUSE = 1
REFINE_LOCAL = 2  # Refine with query-specific additions (see ``group``)


# ----------------------------------------------------------------------------
# small steps (kept separate so that each can be checked on its own)
# ----------------------------------------------------------------------------
def _relu(x):
    """max(0, x) elementwise."""
    return np.maximum(x, 0.0)


def _n_visible(p):
    """A query at position p sees keys 0..p: p + 1 keys."""
    return p + 1


def _rank_order(scores, idx):
    """Order by score descending, then key index ascending (full stable sort)."""
    return np.lexsort((idx, -scores))


def decode_e4m3(b):
    """Decode OCP FP8 E4M3 bytes to float64.

    Layout: 1 sign bit, 4 exponent bits (bias 7), 3 mantissa bits.  Exponent
    field 0 encodes subnormals m * 2^-9; otherwise (1 + m/8) * 2^(e - 7).
    S.1111.111 is NaN; there are no infinities, so the largest finite value is
    S.1111.110 = 448.
    """
    b = np.asarray(b, dtype=np.uint8).astype(np.int64)
    sign = np.where(b & 0x80, -1.0, 1.0)
    e = (b >> 3) & 0xF
    m = b & 0x7
    sub = m.astype(np.float64) * 2.0 ** -9
    nrm = (1.0 + m / 8.0) * np.power(2.0, e - 7.0)
    v = sign * np.where(e == 0, sub, nrm)
    v = np.where((b & 0x7F) == 0x7F, np.nan, v)
    return v


def key_values(K, k_scale=None):
    """Keys as float64 [N, d]: fp8 bytes are decoded and times their token's scale."""
    K = np.asarray(K)
    if K.dtype == np.uint8:
        assert k_scale is not None, "fp8 keys need a per-token scale"
        s = np.asarray(k_scale, dtype=np.float64)
        return decode_e4m3(K) * s[:, None]
    assert k_scale is None
    return K.astype(np.float64)


def score_rows(q_rows, w_rows, Kd):
    """I[r, s] = sum_h w[r, h] * ReLU(q[r, h, :] . Kd[s, :]) for every row r, key s.

    q_rows [R, H, d], w_rows [R, H], Kd [S, d] (float64).  No causal cut here.
    """
    q_rows = np.asarray(q_rows, dtype=np.float64)
    w_rows = np.asarray(w_rows, dtype=np.float64)
    R, H, d = q_rows.shape
    dots = (q_rows.reshape(R * H, d) @ Kd.T).reshape(R, H, Kd.shape[0])
    return np.einsum("rh,rhs->rs", w_rows, _relu(dots))


def select_topk(scores, k, idx=None):
    """First min(k, n) entries of the (score desc, index asc) order.

    ``scores`` [n]; ``idx`` [n] key indices (default 0..n-1).  Returns
    (indices int64, scores float64) in rank order.
    """
    scores = np.asarray(scores, dtype=np.float64)
    idx = np.arange(scores.shape[0], dtype=np.int64) if idx is None else np.asarray(idx, np.int64)
    order = _rank_order(scores, idx)[:min(k, scores.shape[0])]
    return idx[order], scores[order]


def _pad(sel_idx, sel_val, k):
    oi = np.full(k, -1, dtype=np.int64)
    ov = np.full(k, -np.inf, dtype=np.float64)
    oi[:sel_idx.shape[0]] = sel_idx
    ov[:sel_val.shape[0]] = sel_val
    return oi, ov


def _row_chunks(rows, H, span, budget=1 << 27):
    step = max(1, budget // max(1, H * span * 8))
    for i in range(0, len(rows), step):
        yield rows[i:i + step]


def dense(q, w, K, k, q_pos0=0, k_scale=None, rows=None, return_scores=False):
    """Dense indexer: per query row its top-k over keys 0..q_pos0+t.

    Returns dict with ``idx`` [R, k] int64 (-1 padded), ``val`` [R, k] float64
    (-inf padded), ``count`` [R], ``rows``; with ``return_scores`` also
    ``scores``: list of the full prefix score vectors (for parity checks).
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Kd = key_values(K, k_scale)
    T, H, _ = q.shape
    rows = np.arange(T) if rows is None else np.asarray(rows, dtype=np.int64)
    R = rows.shape[0]
    out_i = np.full((R, k), -1, dtype=np.int64)
    out_v = np.full((R, k), -np.inf, dtype=np.float64)
    cnt = np.zeros(R, dtype=np.int64)
    full = [None] * R
    pos = {int(r): j for j, r in enumerate(rows)}
    order = np.argsort(rows)
    srows = rows[order]
    span = int(q_pos0 + srows.max() + 1) if R else 0
    for ch in _row_chunks(srows, H, span):
        nvis_max = _n_visible(int(q_pos0 + ch.max()))
        S = score_rows(q[ch], w[ch], Kd[:nvis_max])
        for j, r in enumerate(ch):
            nv = _n_visible(int(q_pos0 + r))
            row = S[j, :nv]
            si, sv = select_topk(row, k)
            o = pos[int(r)]
            out_i[o], out_v[o] = _pad(si, sv, k)
            cnt[o] = si.shape[0]
            if return_scores:
                full[o] = row.copy()
    res = {"idx": out_i, "val": out_v, "count": cnt, "rows": rows}
    if return_scores:
        res["scores"] = full
    return res


def round_bf16(x):
    """Round float64 values to the nearest bfloat16 (8 significant bits),
    ties to even.  The group form stores its proxy query in the query's own
    dtype, and block routing its representatives in bf16; this is that
    rounding, applied to the float64 means.  Zero stays zero; values are
    assumed in the normal bf16 range."""
    x = np.asarray(x, dtype=np.float64)
    out = np.zeros_like(x)
    nz = x != 0
    e = np.floor(np.log2(np.abs(x[nz])))
    ulp = np.exp2(e - 7)
    out[nz] = np.round(x[nz] / ulp) * ulp   # np.round: half to even
    return out


def round_q(x, q_dtype):
    """The proxy query as the library stores it: the float64 mean rounded to
    the query's own dtype ("bf16": nearest bfloat16, ties to even; "fp32":
    nearest float32; "f64": kept as is).  The PIVOT abstract says only that a
    group is aggregated into one proxy query; this library keeps that query
    in the dtype of the queries it aggregates, so the proxy scan runs on the
    same arithmetic as every other scan."""
    if q_dtype == "bf16":
        return round_bf16(x)
    if q_dtype == "fp32":
        return np.asarray(x, dtype=np.float64).astype(np.float32).astype(np.float64)
    if q_dtype == "f64":
        return np.asarray(x, dtype=np.float64)
    raise ValueError(f"q_dtype must be 'bf16', 'fp32' or 'f64', not {q_dtype!r}")


def proxy(q, w, G, *, q_dtype):
    """PIVOT proxy per group of G consecutive rows: the members' mean q and mean w.

    A last group with fewer than G rows averages over its actual members;
    no rows form no groups.  The mean q is rounded to ``q_dtype`` (see
    ``round_q``); the mean w stays float64.  Returns (qbar [ng, H, d],
    wbar [ng, H]).
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    T = q.shape[0]
    ng = (T + G - 1) // G
    if ng == 0:
        return np.zeros((0,) + q.shape[1:]), np.zeros((0,) + w.shape[1:])
    qb = np.stack([q[g * G:min(T, (g + 1) * G)].mean(axis=0) for g in range(ng)])
    wb = np.stack([w[g * G:min(T, (g + 1) * G)].mean(axis=0) for g in range(ng)])
    return round_q(qb, q_dtype), wb


def group(q, w, K, k, G, bank, mode, q_pos0=0, k_scale=None, qbar=None, wbar=None,
          groups=None, members=None, bank_override=None, *, q_dtype):
    """PIVOT group-shared indexer (Refine or Reuse).

    For group g (rows gG..min(T,(g+1)G)-1) with last member position L_g:
      1. proxy scores over keys 0..L_g with (qbar[g], wbar[g]);
      2. bank = first min(bank, L_g + 1) keys of the proxy's (score desc,
         index asc) order;
      3. Refine: member t scores bank keys <= p_t with its own q, w and keeps
         its top-k; Reuse: member t keeps the first k bank entries (in the
         proxy's order) with key <= p_t, valued by the proxy score.
         REFINE_LOCAL: Refine over the bank plus the query-specific keys the
         ADIndex page asks refinement to add (section Inference: tokens
         unique to one query are recovered).  The page does not say which;
         the reading taken here is the member's own stretch of the group,
         keys at positions p_first .. p_t (p_first = the group's first
         member), recent keys that the shared proxy may rank low.

    ``q_dtype`` is the dtype the queries came in ("bf16", "fp32"; "f64" for
    hand-worked float64 cases): the proxy query is the member mean rounded to
    it (``proxy``).  ``qbar``/``wbar`` replace ``proxy(q, w, G, q_dtype)``,
    e.g. with the proxy exactly as another implementation rounded it.  ``groups`` restricts
    the work to some groups; ``members`` (list of row indices) to some rows.
    ``bank_override`` {g: bank index array in proxy order} replaces step 1-2.
    Returns dict with ``bank_idx``/``bank_val`` {g: arrays in proxy order},
    ``bank_scores`` {g: full proxy score vector}, and ``idx``/``val``/``count``
    {row: padded arrays}, plus ``member_scores`` {row: full member score vector
    over keys 0..p_t} for Refine.
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Kd = key_values(K, k_scale)
    T = q.shape[0]
    ng = (T + G - 1) // G
    if qbar is None or wbar is None:
        qb, wb = proxy(q, w, G, q_dtype=q_dtype)
        qbar = qb if qbar is None else qbar
        wbar = wb if wbar is None else wbar
    qbar = np.asarray(qbar, dtype=np.float64)
    wbar = np.asarray(wbar, dtype=np.float64)
    if groups is None:
        groups = range(ng)
    mem_set = None if members is None else set(int(m) for m in members)
    res = {"bank_idx": {}, "bank_val": {}, "bank_scores": {}, "idx": {}, "val": {},
           "count": {}, "member_scores": {}}
    for g in groups:
        r0, r1 = g * G, min(T, (g + 1) * G)
        L = q_pos0 + r1 - 1
        nv = _n_visible(L)
        ps = score_rows(qbar[g:g + 1], wbar[g:g + 1], Kd[:nv])[0]
        res["bank_scores"][g] = ps
        if bank_override is not None and g in bank_override:
            b_idx = np.asarray(bank_override[g], dtype=np.int64)
            b_val = ps[b_idx]
        else:
            b_idx, b_val = select_topk(ps, bank)
        res["bank_idx"][g], res["bank_val"][g] = b_idx, b_val
        rows = [r for r in range(r0, r1) if mem_set is None or r in mem_set]
        for r in rows:
            p = q_pos0 + r
            keep = b_idx <= p
            if mode in (REFINE, REFINE_LOCAL):
                ms = score_rows(q[r:r + 1], w[r:r + 1], Kd[:_n_visible(p)])[0]
                res["member_scores"][r] = ms
                cand = b_idx[keep]
                if mode == REFINE_LOCAL:
                    cand = np.union1d(cand, np.arange(q_pos0 + r0, p + 1))
                si, sv = select_topk(ms[cand], k, idx=cand)
            elif mode == REUSE:
                si, sv = b_idx[keep][:k], b_val[keep][:k]
            else:
                raise ValueError(mode)
            res["idx"][r], res["val"][r] = _pad(si, sv, k)
            res["count"][r] = si.shape[0]
    return res


def decode(q, w, K, k_offsets, q_offsets, k, k_scale=None, return_scores=False):
    """Decode indexer over a batch of key caches.

    Sequence b owns keys K[k_offsets[b]:k_offsets[b+1]] (N_b of them, indexed
    0..N_b-1 within the sequence) and query rows q_offsets[b]..q_offsets[b+1]-1
    (m_b of them); new query j sits at position N_b - m_b + j and sees keys
    0..N_b - m_b + j.  Returns idx/val [sum m_b, k] with indices local to the
    sequence.
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    ko = np.asarray(k_offsets, dtype=np.int64)
    qo = np.asarray(q_offsets, dtype=np.int64)
    B = ko.shape[0] - 1
    M = int(qo[-1])
    out_i = np.full((M, k), -1, dtype=np.int64)
    out_v = np.full((M, k), -np.inf, dtype=np.float64)
    cnt = np.zeros(M, dtype=np.int64)
    scores = [None] * M
    Kall = np.asarray(K)
    sc = None if k_scale is None else np.asarray(k_scale)
    for b in range(B):
        k0, k1 = int(ko[b]), int(ko[b + 1])
        Nb = k1 - k0
        mb = int(qo[b + 1] - qo[b])
        Kd = key_values(Kall[k0:k1], None if sc is None else sc[k0:k1])
        for j in range(mb):
            r = int(qo[b]) + j
            p = Nb - mb + j
            S = score_rows(q[r:r + 1], w[r:r + 1], Kd[:_n_visible(p)])[0]
            si, sv = select_topk(S, k)
            out_i[r], out_v[r] = _pad(si, sv, k)
            cnt[r] = si.shape[0]
            if return_scores:
                scores[r] = S
    res = {"idx": out_i, "val": out_v, "count": cnt}
    if return_scores:
        res["scores"] = scores
    return res


def decode_group(q, w, K, k_offsets, q_offsets, k, bank, mode, k_scale=None, qbar=None, wbar=None,
                 bank_override=None, *, q_dtype):
    """PIVOT in decode: the new queries of one sequence form the group.

    The PIVOT abstract names the queries decoded together in one
    multi-token-prediction step as a natural group.  Sequence b (keys
    K[k_offsets[b]:k_offsets[b+1]], N_b of them; query rows
    q_offsets[b]..q_offsets[b+1]-1, m_b of them, query j at position
    N_b - m_b + j) is one group of G = m_b: its proxy is the members' mean,
    the proxy scans keys 0..N_b - 1 (the prefix of its last query), the bank is
    the proxy's top-`bank`, and every query refines or reuses exactly as in
    ``group``.  Indices are local to the sequence.

    ``q_dtype`` rounds the proxy query as in ``group``.  ``qbar`` [B, H, d] /
    ``wbar`` [B, H] replace the proxy (e.g. as another implementation rounded
    it); ``bank_override`` {b: bank indices}
    replaces the proxy's bank.  Returns idx/val/count over all query rows and
    bank_idx/bank_val/bank_scores {b: ...}.
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    ko = np.asarray(k_offsets, dtype=np.int64)
    qo = np.asarray(q_offsets, dtype=np.int64)
    B = ko.shape[0] - 1
    M = int(qo[-1])
    out_i = np.full((M, k), -1, dtype=np.int64)
    out_v = np.full((M, k), -np.inf, dtype=np.float64)
    cnt = np.zeros(M, dtype=np.int64)
    res = {"bank_idx": {}, "bank_val": {}, "bank_scores": {}}
    Kall = np.asarray(K)
    sc = None if k_scale is None else np.asarray(k_scale)
    for b in range(B):
        k0, k1 = int(ko[b]), int(ko[b + 1])
        r0, r1 = int(qo[b]), int(qo[b + 1])
        Nb, mb = k1 - k0, r1 - r0
        r = group(q[r0:r1], w[r0:r1], Kall[k0:k1], k, mb, bank, mode, q_pos0=Nb - mb,
                  k_scale=None if sc is None else sc[k0:k1],
                  qbar=None if qbar is None else np.asarray(qbar)[b:b + 1],
                  wbar=None if wbar is None else np.asarray(wbar)[b:b + 1],
                  bank_override=None if bank_override is None or b not in bank_override
                  else {0: bank_override[b]}, q_dtype=q_dtype)
        res["bank_idx"][b], res["bank_val"][b] = r["bank_idx"][0], r["bank_val"][0]
        res["bank_scores"][b] = r["bank_scores"][0]
        for j in range(mb):
            out_i[r0 + j], out_v[r0 + j], cnt[r0 + j] = r["idx"][j], r["val"][j], r["count"][j]
    res.update(idx=out_i, val=out_v, count=cnt)
    return res


def block_reps(K, block=128, k_scale=None):
    """Mean key of each contiguous block of `block` keys (the last block may
    be shorter): the block representatives of two-stage selection over
    contiguous blocks (AttentionIndex page, Why Positional Blocks Lose
    Recall: blocks ranked by mean-pooled representatives)."""
    Kd = key_values(K, k_scale)
    N = Kd.shape[0]
    nb = (N + block - 1) // block
    return np.stack([Kd[b * block:min(N, (b + 1) * block)].mean(axis=0) for b in range(nb)])


def block_routed(q, w, K, k, n_blocks, q_pos0=0, k_scale=None, block=128, reps=None, rows=None):
    """Two-stage selection over contiguous blocks, then the native score.

    Query row t at position p: (1) route: score the representatives of the
    complete blocks before it (blocks 0 .. (p+1)//block - 1, so routing sees
    no key beyond p) with the indexer formula and keep the best `n_blocks`
    (ties to the lower block); (2) refine: the candidates are the keys of
    those blocks plus the query's own partial block (keys (p+1)//block*block
    .. p), scored with the query's own q, w; keep the top-k.  ``reps`` may
    replace the float64 means (another implementation's rounding).  Returns
    idx/val/count per row plus the selected blocks.
    """
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Kd = key_values(K, k_scale)
    R = block_reps(K, block, k_scale) if reps is None else np.asarray(reps, dtype=np.float64)
    T = q.shape[0]
    rows = range(T) if rows is None else rows
    res = {"idx": {}, "val": {}, "count": {}, "blocks": {}}
    for t in rows:
        p = q_pos0 + t
        c = (p + 1) // block
        bs = score_rows(q[t:t + 1], w[t:t + 1], R[:c])[0] if c > 0 else np.zeros(0)
        sel, _ = select_topk(bs, n_blocks)
        cand = np.concatenate([np.arange(b * block, (b + 1) * block) for b in np.sort(sel)] +
                              [np.arange(c * block, p + 1)]).astype(np.int64)
        S = score_rows(q[t:t + 1], w[t:t + 1], Kd[cand])[0]
        si, sv = select_topk(S, k, idx=cand)
        res["idx"][t], res["val"][t] = _pad(si, sv, k)
        res["count"][t] = si.shape[0]
        res["blocks"][t] = sel
    return res


def kmeans(K, C, iters, k_scale=None):
    """Plain Lloyd's k-means over the keys (Euclidean), the index build of
    inverted-file routing (AttentionIndex page: keys grouped by similarity
    rather than position; its learned encoder and causal index versions are
    not part of this plain form).  Centroid i starts at key floor(i N / C);
    each iteration assigns every key to its nearest centroid (ties to the
    lower centroid), then moves each centroid to the mean of its members (a
    centroid without members stays).  Returns (assign [N] int64, centroids
    [C, d] float64)."""
    Kd = key_values(K, k_scale)
    N = Kd.shape[0]
    cen = Kd[(np.arange(C) * N) // C].copy()
    assign = np.zeros(N, dtype=np.int64)
    for _ in range(iters):
        d2 = (Kd * Kd).sum(1)[:, None] - 2.0 * Kd @ cen.T + (cen * cen).sum(1)[None, :]
        assign = np.argmin(d2, axis=1)  # first minimum = lower centroid on ties
        for c in range(C):
            m = assign == c
            if m.any():
                cen[c] = Kd[m].mean(axis=0)
    return assign, cen


def ivf_routed(q, w, K, k, n_probe, assign, centroids, q_pos0=0, k_scale=None, rows=None):
    """Inverted-file routing, then the native score (AttentionIndex page:
    route each query over the clusters, refine the candidates with the
    native indexer score).  Query row t at position p: score the centroids
    with the indexer formula, keep the best n_probe clusters (ties to the
    lower cluster); the candidates are their members with key <= p (the
    clusters span the whole key set: causality by masking, not versions);
    keep the top-k by the native score."""
    q = np.asarray(q, dtype=np.float64)
    w = np.asarray(w, dtype=np.float64)
    Kd = key_values(K, k_scale)
    assign = np.asarray(assign, dtype=np.int64)
    cen = np.asarray(centroids, dtype=np.float64)
    res = {"idx": {}, "val": {}, "count": {}, "clusters": {}}
    for t in (range(q.shape[0]) if rows is None else rows):
        p = q_pos0 + t
        cs = score_rows(q[t:t + 1], w[t:t + 1], cen)[0]
        sel, _ = select_topk(cs, n_probe)
        cand = np.nonzero(np.isin(assign[:p + 1], sel))[0].astype(np.int64)
        S = score_rows(q[t:t + 1], w[t:t + 1], Kd[cand])[0]
        si, sv = select_topk(S, k, idx=cand)
        res["idx"][t], res["val"][t] = _pad(si, sv, k)
        res["count"][t] = si.shape[0]
        res["clusters"][t] = sel
    return res
