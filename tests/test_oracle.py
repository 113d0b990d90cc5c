"""Pins for the CPU oracle (no GPU).

Each ``pin_*`` function checks the oracle against something other than
itself: values worked by hand (``tests/golden``), the fp8 format's published
value table, brute-force enumeration of subsets, library routines on special
cases, closed-form identities and invariants.  ``test_mutants_are_caught``
plants plausible mistakes in the oracle (on the CPU) and requires that some pin
fails for each.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
import torch

from oracle import dsa_oracle as O

GOLD = os.path.join(os.path.dirname(__file__), "golden")


def _load(name):
    with open(os.path.join(GOLD, name)) as f:
        return json.load(f)


def _nan_to_neginf(a):
    return np.array([[-np.inf if v is None else v for v in r] for r in a], dtype=np.float64)


# ---------------------------------------------------------------------------
# pins (each raises AssertionError on a mismatch)
# ---------------------------------------------------------------------------
def pin_e4m3_table(O):
    g = _load("e4m3_values.json")
    for hx, v in g["values"].items():
        got = O.decode_e4m3(np.array([int(hx, 16)], dtype=np.uint8))[0]
        assert got == v and math.copysign(1, got) == math.copysign(1, v), (hx, got, v)
    for hx in g["nan"]:
        assert np.isnan(O.decode_e4m3(np.array([int(hx, 16)], dtype=np.uint8))[0])


def pin_e4m3_library(O):
    allb = np.arange(256, dtype=np.uint8)
    lib = torch.from_numpy(allb).view(torch.float8_e4m3fn).to(torch.float64).numpy()
    got = O.decode_e4m3(allb)
    fin = ~np.isnan(lib)
    assert np.array_equal(np.isnan(got), ~fin)
    assert np.array_equal(got[fin], lib[fin])


def pin_dense_hand(O):
    g = _load("dense_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["k"], float)
    S = O.score_rows(q, w, K)
    for t, row in enumerate(g["scores"]):
        for s, v in enumerate(row):
            if v is not None:
                assert S[t, s] == v, (t, s, S[t, s], v)
    for kk, exp in g["topk"].items():
        r = O.dense(q, w, K, int(kk), q_pos0=g["q_pos0"])
        assert np.array_equal(r["idx"], np.array(exp["idx"])), (kk, r["idx"], exp["idx"])
        assert np.array_equal(r["val"], _nan_to_neginf(exp["val"])), (kk, r["val"])


def pin_ties_hand(O):
    g = _load("ties_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["k"], float)
    for kk, exp in g["topk"].items():
        r = O.dense(q, w, K, int(kk), q_pos0=g["q_pos0"])
        assert np.array_equal(r["idx"], np.array(exp["idx"])), (kk, r["idx"])


def pin_relu_zero_hand(O):
    g = _load("relu_zero_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["k"], float)
    S = O.score_rows(q, w, K)
    assert np.array_equal(S, np.array(g["scores"], float)), S
    assert not np.signbit(S[0]).any()   # exact +0, not a residue or -0


def pin_group_hand(O):
    g = _load("group_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["k"], float)
    qb, wb = O.proxy(q, w, g["G"], q_dtype="bf16")
    assert np.array_equal(qb, np.array(g["proxy_q"], float)) and np.array_equal(wb, np.array(g["proxy_w"], float))
    for c in g["cases"]:
        for mode, key in ((O.REFINE, "refine"), (O.REUSE, "reuse")):
            r = O.group(q, w, K, c["k"], g["G"], c["bank"], mode, q_pos0=g["q_pos0"], q_dtype="bf16")
            assert list(r["bank_idx"][0]) == c["bank_idx"], (c, r["bank_idx"])
            assert list(r["bank_val"][0]) == c["bank_val"]
            for m in range(2):
                assert list(r["idx"][m]) == c[key + "_idx"][m], (key, c, m, r["idx"][m])
                assert list(r["val"][m]) == c[key + "_val"][m], (key, c, m, r["val"][m])


def pin_proxy_rounding_hand(O):
    # the proxy query is rounded to the queries' dtype before its scan: with
    # bf16 queries the rounding turns a strict order into a tie, which moves
    # the bank and every member's result
    g = _load("proxy_round_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["k_rows"], float)
    for dt in ("bf16", "fp32"):
        e = g[dt]
        qb, wb = O.proxy(q, w, g["G"], q_dtype=dt)
        assert np.array_equal(qb, np.array(e["proxy_q"], float)), (dt, qb)
        assert np.array_equal(wb, np.array([[1.0]])), (dt, wb)
        for mode, key in ((O.REUSE, "reuse"), (O.REFINE, "refine")):
            r = O.group(q, w, K, g["k"], g["G"], g["bank"], mode, q_pos0=g["q_pos0"], q_dtype=dt)
            assert list(r["bank_idx"][0]) == e["bank_idx"] and list(r["bank_val"][0]) == e["bank_val"], (dt, r)
            for m in range(2):
                assert list(r["idx"][m]) == e[key + "_idx"][m], (dt, key, m, r["idx"][m])
                assert list(r["val"][m]) == e[key + "_val"][m], (dt, key, m, r["val"][m])
    # the same group as a decode step: one sequence of 3 cached keys whose 2 new
    # queries sit at positions 1 and 2
    for dt in ("bf16", "fp32"):
        e = g[dt]
        r = O.decode_group(q, w, K, [0, 3], [0, 2], g["k"], g["bank"], O.REUSE, q_dtype=dt)
        assert list(r["bank_idx"][0]) == e["bank_idx"], (dt, r["bank_idx"][0])
        assert [list(x) for x in r["idx"]] == e["reuse_idx"], (dt, r["idx"])
    # the fp32 rounding is float32's own
    x = np.array([1.0 + 2.0 ** -30, 3.0 + 2.0 ** -23, -0.1])
    assert np.array_equal(O.round_q(x, "fp32"), x.astype(np.float32).astype(np.float64))
    assert np.array_equal(O.round_q(x, "f64"), x)


def pin_decode_hand(O):
    g = _load("decode_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["keys"], float)
    r = O.decode(q, w, K, g["k_offsets"], g["q_offsets"], g["k"])
    assert np.array_equal(r["idx"], np.array(g["idx"])), r["idx"]
    assert np.array_equal(r["val"], _nan_to_neginf(g["val"])), r["val"]


def _rand_case(seed, T=6, N=9, H=3, d=5, q_pos0=3):
    rng = np.random.default_rng(seed)
    q = rng.standard_normal((T, H, d))
    w = rng.uniform(0, 1, (T, H))
    K = rng.standard_normal((N, d))
    return q, w, K, q_pos0


def pin_single_head_matmul(O):
    # one head, w = 1, non-negative q and k: every dot is >= 0 so the score is the
    # plain matrix product (library matmul)
    rng = np.random.default_rng(1)
    q = rng.uniform(0, 1, (7, 1, 6))
    K = rng.uniform(0, 1, (11, 6))
    S = O.score_rows(q, np.ones((7, 1)), K)
    assert np.allclose(S, np.matmul(q[:, 0, :], K.T), rtol=1e-14, atol=0)


def pin_relu_odd_identity(O):
    # ReLU(x) - ReLU(-x) = x, so for one head S(q) - S(-q) = w * (q . k)
    q, w, K, _ = _rand_case(2, H=1)
    d = O.score_rows(q, w, K) - O.score_rows(-q, w, K)
    assert np.allclose(d, w[:, :1] * np.matmul(q[:, 0, :], K.T), rtol=1e-12, atol=1e-14)


def pin_head_structure(O):
    # heads add up (split H into two parts), weights scale linearly, and a
    # permutation of heads (with their weights) changes nothing
    q, w, K, _ = _rand_case(3, H=4)
    S = O.score_rows(q, w, K)
    S_a = O.score_rows(q[:, :2], w[:, :2], K)
    S_b = O.score_rows(q[:, 2:], w[:, 2:], K)
    assert np.allclose(S, S_a + S_b, rtol=1e-13, atol=1e-15)
    assert np.allclose(O.score_rows(q, 2.5 * w, K), 2.5 * S, rtol=1e-13)
    perm = [2, 0, 3, 1]
    assert np.allclose(O.score_rows(q[:, perm], w[:, perm], K), S, rtol=1e-13)
    # positive scale of q passes through ReLU
    assert np.allclose(O.score_rows(3.0 * q, w, K), 3.0 * S, rtol=1e-13)
    # row / key correspondence: swapping two keys swaps two score columns
    K2 = K.copy()
    K2[[1, 4]] = K2[[4, 1]]
    S2 = O.score_rows(q, w, K2)
    assert np.allclose(S2[:, [4, 1]], S[:, [1, 4]], rtol=1e-13)


def pin_fp8_keys_scale(O):
    # per-token scale > 0 passes through ReLU: scores with scaled fp8 keys equal
    # scale[s] times the scores with the decoded bytes
    rng = np.random.default_rng(4)
    b = rng.integers(0, 256, (10, 4), dtype=np.uint8)
    b[(b & 0x7F) == 0x7F] = 0x38          # no NaN codes
    s = rng.uniform(0.5, 2.0, 10)
    q = rng.standard_normal((3, 2, 4))
    w = rng.uniform(0, 1, (3, 2))
    S = O.score_rows(q, w, O.key_values(b, s))
    S0 = O.score_rows(q, w, O.decode_e4m3(b))
    assert np.allclose(S, S0 * s[None, :], rtol=1e-13, atol=1e-300)


def _brute_topk(scores, k):
    """Max-sum k-subset; among equal sums the lexicographically smallest sorted index tuple."""
    n = len(scores)
    best = None
    for comb in itertools.combinations(range(n), min(k, n)):
        key = (-sum(scores[i] for i in comb), comb)
        if best is None or key < best:
            best = key
    return sorted(best[1])


def pin_topk_bruteforce(O):
    rng = np.random.default_rng(5)
    for trial in range(60):
        n = int(rng.integers(1, 12))
        k = int(rng.integers(1, 4))
        sc = rng.integers(-3, 4, n).astype(np.float64)   # many exact ties
        si, _ = O.select_topk(sc, k)
        assert sorted(si.tolist()) == _brute_topk(list(sc), k), (sc, k, si)
    # exhaustive: every row of a small causal problem, k <= 3, N <= 64
    q, w, K, q0 = _rand_case(6, T=8, N=64, H=2, d=3, q_pos0=56)
    K[10] = K[3]                                       # duplicate key -> exact tie
    for k in (1, 2, 3):
        r = O.dense(q, w, K, k, q_pos0=q0, return_scores=True)
        for t in range(8):
            row = r["scores"][t]
            assert len(row) == q0 + t + 1
            exp = _brute_topk(list(row), k)
            assert sorted(r["idx"][t][:r["count"][t]].tolist()) == exp


def pin_causality(O):
    q, w, K, _ = _rand_case(7, T=12, N=12, q_pos0=0)
    k = 5
    r = O.dense(q, w, K, k, q_pos0=0)
    for t in range(12):
        sel = r["idx"][t][r["idx"][t] >= 0]
        assert (sel <= t).all()
        if t + 1 < k:
            assert sorted(sel.tolist()) == list(range(t + 1))
            assert (r["idx"][t][t + 1:] == -1).all() and np.isneginf(r["val"][t][t + 1:]).all()
        else:
            assert len(sel) == k
    # a key beyond a query's position never changes that query's result
    K2 = K.copy()
    K2[11] = 100.0 * np.abs(K2[11])
    r2 = O.dense(q, w, K2, k, q_pos0=0)
    assert np.array_equal(r["idx"][:11], r2["idx"][:11])


def pin_group_invariants(O):
    q, w, K, _ = _rand_case(8, T=12, N=20, H=3, d=4, q_pos0=8)
    q0, k, G = 8, 4, 4
    dn = O.dense(q, w, K, k, q_pos0=q0)
    # Refine with a bank covering the whole prefix is dense selection
    rf = O.group(q, w, K, k, G, 64, O.REFINE, q_pos0=q0, q_dtype="f64")
    for t in range(12):
        assert np.array_equal(rf["idx"][t], dn["idx"][t])
    # G = 1: the proxy is the query itself, so Reuse == Refine == dense
    for mode in (O.REFINE, O.REUSE):
        r1 = O.group(q, w, K, k, 1, 6, mode, q_pos0=q0, q_dtype="f64")
        for t in range(12):
            assert np.array_equal(r1["idx"][t], dn["idx"][t]), (mode, t)
    # Reuse: the last member of a group gets exactly the proxy's top-k
    ru = O.group(q, w, K, k, G, 7, O.REUSE, q_pos0=q0, q_dtype="f64")
    for g in range(3):
        last = g * G + G - 1
        ps = ru["bank_scores"][g]
        pi, _ = O.select_topk(ps, k)
        assert sorted(ru["idx"][last].tolist()) == sorted(pi.tolist())
        # every member only receives keys it may see
        for t in range(g * G, g * G + G):
            sel = ru["idx"][t][ru["idx"][t] >= 0]
            assert (sel <= q0 + t).all()
    # the proxy of identical rows is the row; the proxy of two rows is their midpoint
    qq = np.repeat(q[:1], 4, axis=0)
    ww = np.repeat(w[:1], 4, axis=0)
    qb, wb = O.proxy(qq, ww, 4, q_dtype="f64")
    assert np.allclose(qb[0], q[0], rtol=1e-15) and np.allclose(wb[0], w[0], rtol=1e-15)
    qb, wb = O.proxy(q[:2], w[:2], 2, q_dtype="f64")
    assert np.allclose(qb[0], 0.5 * (q[0] + q[1]), rtol=1e-15)
    assert np.allclose(wb[0], 0.5 * (w[0] + w[1]), rtol=1e-15)
    # partial last group averages over its actual members
    qb, _ = O.proxy(q[:5], w[:5], 4, q_dtype="f64")
    assert qb.shape[0] == 2 and np.allclose(qb[1], q[4], rtol=1e-15)


def pin_decode_matches_dense(O):
    # a decode batch equals dense prefill on each sequence restricted to its
    # last m_b query positions
    rng = np.random.default_rng(9)
    lengths, ms = [7, 1, 12], [2, 1, 3]
    H, d, k = 2, 3, 4
    Ks = [rng.standard_normal((n, d)) for n in lengths]
    qs = [rng.standard_normal((m, H, d)) for m in ms]
    ws = [rng.uniform(0, 1, (m, H)) for m in ms]
    ko = np.concatenate([[0], np.cumsum(lengths)])
    qo = np.concatenate([[0], np.cumsum(ms)])
    r = O.decode(np.concatenate(qs), np.concatenate(ws), np.concatenate(Ks), ko, qo, k)
    for b in range(3):
        dn = O.dense(qs[b], ws[b], Ks[b], k, q_pos0=lengths[b] - ms[b])
        assert np.array_equal(r["idx"][qo[b]:qo[b + 1]], dn["idx"]), b


def pin_decode_group_hand(O):
    g = _load("decode_group_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["K"], float)
    for mode, key in ((O.REFINE, "refine"), (O.REUSE, "reuse")):
        r = O.decode_group(q, w, K, g["k_offsets"], g["q_offsets"], g["k"], g["bank"], mode, q_dtype="bf16")
        for b in range(2):
            assert np.array_equal(r["bank_idx"][b], g["bank_idx"][b]), (key, b, r["bank_idx"][b])
            assert np.array_equal(r["bank_val"][b], g["bank_val"][b]), (key, b, r["bank_val"][b])
        assert np.array_equal(r["idx"], np.array(g[key + "_idx"])), (key, r["idx"])
        assert np.array_equal(r["val"], np.array(g[key + "_val"])), (key, r["val"])
    d = O.decode(q, w, K, g["k_offsets"], g["q_offsets"], g["k"])
    assert np.array_equal(d["idx"], np.array(g["decode_idx"])) and np.array_equal(d["val"], g["decode_val"])


def pin_decode_group_invariants(O):
    rng = np.random.default_rng(11)
    lengths, ms = [9, 6, 14, 5], [2, 1, 3, 4]
    H, d, k = 2, 3, 3
    q = rng.standard_normal((sum(ms), H, d))
    w = rng.uniform(0, 1, (sum(ms), H))
    K = rng.standard_normal((sum(lengths), d))
    ko = np.concatenate([[0], np.cumsum(lengths)])
    qo = np.concatenate([[0], np.cumsum(ms)])
    dec = O.decode(q, w, K, ko, qo, k)
    # a bank as large as every cache makes Refine the decode indexer
    r = O.decode_group(q, w, K, ko, qo, k, max(lengths), O.REFINE, q_dtype="f64")
    assert np.array_equal(r["idx"], dec["idx"]) and np.array_equal(r["val"], dec["val"])
    rf = O.decode_group(q, w, K, ko, qo, k, 4, O.REFINE, q_dtype="f64")
    ru = O.decode_group(q, w, K, ko, qo, k, 4, O.REUSE, q_dtype="f64")
    for b in range(4):
        last = qo[b + 1] - 1
        # the last query may see the whole bank: Reuse gives it the proxy's top-k
        n = ru["count"][last]
        assert np.array_equal(ru["idx"][last][:n], ru["bank_idx"][b][:k]), b
        if ms[b] == 1:
            # one query: the proxy is the query, so all three agree
            assert np.array_equal(rf["idx"][last], dec["idx"][last]), b
            assert np.array_equal(ru["idx"][last], dec["idx"][last]), b
            assert np.allclose(ru["val"][last], dec["val"][last], rtol=1e-12), b
    # Refine with local additions: a bank as large as every cache gives the
    # decode indexer; with a small bank each query's candidates are the bank
    # plus its sequence's new keys up to its own position, so its selection is
    # causal, never worse than plain Refine, and the top-k of those candidates
    rl_full = O.decode_group(q, w, K, ko, qo, k, max(lengths), O.REFINE_LOCAL, q_dtype="f64")
    assert np.array_equal(rl_full["idx"], dec["idx"]) and np.array_equal(rl_full["val"], dec["val"])
    rl = O.decode_group(q, w, K, ko, qo, k, 4, O.REFINE_LOCAL, q_dtype="f64")
    for b in range(4):
        nb, mb = lengths[b], ms[b]
        Kb = K[ko[b]:ko[b + 1]]
        bank = rl["bank_idx"][b]
        for j in range(mb):
            r, p = qo[b] + j, nb - mb + j
            n = rl["count"][r]
            sel = rl["idx"][r][:n]
            assert np.all(sel <= p), (b, j)
            S = O.score_rows(q[r:r + 1], w[r:r + 1], Kb[:p + 1])[0]
            assert S[sel].min() >= S[rf["idx"][r][:rf["count"][r]]].min() - 1e-15, (b, j)
            cand = np.union1d(bank[bank <= p], np.arange(nb - mb, p + 1))
            oi, _ = O.select_topk(S[cand], k, idx=cand)
            assert np.array_equal(sel, oi), (b, j)


def pin_group_local_hand(O):
    g = _load("group_local_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["K"], float)
    for mode, key in ((O.REFINE, "refine"), (O.REFINE_LOCAL, "refine_local"), (O.REUSE, "reuse")):
        r = O.group(q, w, K, g["k"], g["G"], g["bank"], mode, q_pos0=g["q_pos0"], q_dtype="bf16")
        assert np.array_equal(r["bank_idx"][0], g["bank_idx"]), (key, r["bank_idx"][0])
        for t in range(2):
            assert np.array_equal(r["idx"][t], g[key + "_idx"][t]), (key, t, r["idx"][t])
            assert np.array_equal(r["val"][t], g[key + "_val"][t]), (key, t, r["val"][t])


def pin_group_local_invariants(O):
    q, w, K, _ = _rand_case(12, T=14, N=24, H=3, d=4, q_pos0=10)
    k, G = 4, 5
    dn = O.dense(q, w, K, k, q_pos0=10)
    full = O.group(q, w, K, k, G, 24, O.REFINE_LOCAL, q_pos0=10, q_dtype="f64")
    rf = O.group(q, w, K, k, G, 6, O.REFINE, q_pos0=10, q_dtype="f64")
    rl = O.group(q, w, K, k, G, 6, O.REFINE_LOCAL, q_pos0=10, q_dtype="f64")
    for t in range(14):
        p = 10 + t
        # a bank covering the prefix: the dense indexer
        assert np.array_equal(full["idx"][t], dn["idx"][t]), t
        n = rl["count"][t]
        sel = rl["idx"][t][:n]
        # causal, and never worse than plain Refine: its candidates are a superset
        assert np.all(sel <= p), t
        S = rl["member_scores"][t]
        assert S[sel].min() >= S[rf["idx"][t][:rf["count"][t]]].min() - 1e-15, t
        # the member's own key is always a candidate
        cand = np.union1d(rl["bank_idx"][t // G][rl["bank_idx"][t // G] <= p], np.arange(10 + (t // G) * G, p + 1))
        assert p in cand
        oi, _ = O.select_topk(S[cand], k, idx=cand)
        assert np.array_equal(sel, oi), t


def pin_block_routed_hand(O):
    g = _load("block_routed_hand.json")
    q, w, K = np.array(g["q"], float), np.array(g["w"], float), np.array(g["K"], float)
    r = O.block_routed(q, w, K, g["k"], g["n_blocks"], q_pos0=g["q_pos0"], block=g["block"])
    assert np.array_equal(r["blocks"][0], g["blocks"]), r["blocks"][0]
    assert np.array_equal(r["idx"][0], g["idx"]) and np.array_equal(r["val"][0], g["val"]), (r["idx"][0], r["val"][0])
    d = O.dense(q, w, K, g["k"], q_pos0=g["q_pos0"])
    assert np.array_equal(d["idx"][0], g["dense_idx"]) and np.array_equal(d["val"][0], g["dense_val"])


def pin_block_routed_invariants(O):
    q, w, K, _ = _rand_case(13, T=10, N=40, H=3, d=4, q_pos0=30)
    k = 5
    dn = O.dense(q, w, K, k, q_pos0=30)
    # every complete block routed: the candidates are the whole prefix
    allb = O.block_routed(q, w, K, k, 100, q_pos0=30, block=4)
    # blocks of one key: routing by the native score itself, so the k routed
    # keys are the dense top-k (the own partial block is then empty)
    one = O.block_routed(q, w, K, k, k, q_pos0=30, block=1)
    for t in range(10):
        assert np.array_equal(allb["idx"][t], dn["idx"][t]), t
        assert np.array_equal(one["idx"][t], dn["idx"][t]), t
    # the representative of a block is its mean key
    R = O.block_reps(K, 4)
    assert np.allclose(R[3], K[12:16].mean(axis=0)) and R.shape[0] == 10
    # routing sees complete blocks only: a query at p = 33 routes among blocks 0..7
    r = O.block_routed(q[3:4], w[3:4], K, k, 2, q_pos0=33, block=4)
    assert np.all(r["blocks"][0] < 8)


def pin_ivf_hand(O):
    g = _load("ivf_hand.json")
    K = np.array(g["K"], float)
    a, c = O.kmeans(K, g["C"], g["iters"])
    assert np.array_equal(a, g["assign"]), a
    assert np.allclose(c, g["centroids"]), c
    q, w = np.array(g["q"], float), np.array(g["w"], float)
    for pos, key in ((5, "at5"), (3, "at3")):
        r = O.ivf_routed(q, w, K, g["k"], g["n_probe"], a, c, q_pos0=pos)
        assert np.array_equal(r["idx"][0], g[key + "_idx"]), (pos, r["idx"][0])
        assert np.allclose(r["val"][0], g[key + "_val"]), (pos, r["val"][0])


def pin_ivf_invariants(O):
    rng = np.random.default_rng(14)
    K = np.concatenate([rng.standard_normal((15, 4)) * 0.1 + m for m in (rng.standard_normal((3, 4)) * 3)])
    K = K[rng.permutation(45)]
    a, c = O.kmeans(K, 3, 5)
    # a fixed point: every key sits with a nearest centroid, every centroid is its members' mean
    d2 = ((K[:, None, :] - c[None, :, :]) ** 2).sum(-1)
    assert np.all(d2[np.arange(45), a] <= d2.min(1) + 1e-12)
    for j in range(3):
        assert np.allclose(c[j], K[a == j].mean(0))
    q, w, _, _ = _rand_case(15, T=5, N=45, H=2, d=4, q_pos0=40)
    dn = O.dense(q, w, K, 4, q_pos0=40)
    # probing every cluster: the dense indexer
    r = O.ivf_routed(q, w, K, 4, 3, a, c, q_pos0=40)
    for t in range(5):
        assert np.array_equal(r["idx"][t], dn["idx"][t]), t
    # candidates stay causal and inside the routed clusters
    r1 = O.ivf_routed(q, w, K, 4, 1, a, c, q_pos0=40)
    for t in range(5):
        sel = r1["idx"][t][:r1["count"][t]]
        assert np.all(sel <= 40 + t) and np.all(np.isin(a[sel], r1["clusters"][t]))


def pin_round_bf16_library(O):
    # against torch's float32 -> bfloat16 conversion (round to nearest even)
    # on values exactly representable in float32, where both see the same number
    import torch
    rng = np.random.default_rng(16)
    x = np.concatenate([rng.standard_normal(20000) * 10.0 ** rng.integers(-6, 6, 20000),
                        [1.0, -1.0, 1.00390625, 1.01171875, 3.0, 255.5, -0.0078125]])
    x32 = x.astype(np.float32).astype(np.float64)
    ref = torch.tensor(x32, dtype=torch.float32).to(torch.bfloat16).double().numpy()
    assert np.array_equal(O.round_bf16(x32), ref)
    # ties: 1 + 2^-8 lies halfway between 1 and 1 + 2^-7 and goes to the even 1
    assert O.round_bf16(np.array([1.0 + 2.0 ** -8]))[0] == 1.0
    assert O.round_bf16(np.array([1.0 + 3 * 2.0 ** -8]))[0] == 1.0 + 2.0 ** -6


PINS = [pin_e4m3_table, pin_e4m3_library, pin_dense_hand, pin_ties_hand,
        pin_relu_zero_hand, pin_group_hand, pin_proxy_rounding_hand, pin_decode_hand, pin_single_head_matmul,
        pin_relu_odd_identity, pin_head_structure, pin_fp8_keys_scale,
        pin_topk_bruteforce, pin_causality, pin_group_invariants,
        pin_decode_matches_dense, pin_decode_group_hand, pin_decode_group_invariants,
        pin_group_local_hand, pin_group_local_invariants, pin_block_routed_hand, pin_block_routed_invariants,
        pin_ivf_hand, pin_ivf_invariants, pin_round_bf16_library]


@pytest.mark.parametrize("pin", PINS, ids=[p.__name__ for p in PINS])
def test_pin(pin):
    pin(O)


# ---------------------------------------------------------------------------
# planted mistakes: each must be caught by at least one pin
# ---------------------------------------------------------------------------
def _m_no_relu(mp):
    mp.setattr(O, "_relu", lambda x: x)


def _m_abs_relu(mp):
    mp.setattr(O, "_relu", lambda x: np.abs(x))


def _m_causal_exclusive(mp):
    mp.setattr(O, "_n_visible", lambda p: p)


def _m_causal_plus_one(mp):
    mp.setattr(O, "_n_visible", lambda p: p + 2)


def _m_tiebreak_high(mp):
    mp.setattr(O, "_rank_order", lambda s, i: np.lexsort((-i, -s)))


def _m_ascending(mp):
    mp.setattr(O, "_rank_order", lambda s, i: np.lexsort((i, s)))


def _m_e4m3_bias8(mp):
    real = O.decode_e4m3

    def bad(b):
        return real(b) * 0.5
    mp.setattr(O, "decode_e4m3", bad)


def _m_e4m3_no_subnormal(mp):
    real = O.decode_e4m3

    def bad(b):
        v = real(b)
        e = (np.asarray(b).astype(np.int64) >> 3) & 0xF
        return np.where(e == 0, 0.0, v)
    mp.setattr(O, "decode_e4m3", bad)


def _m_weight_outside(mp):
    def bad(qr, wr, Kd):
        R, H, d = qr.shape
        dots = (qr.reshape(R * H, d) @ Kd.T).reshape(R, H, -1)
        return O._relu(np.einsum("rh,rhs->rs", wr, dots))
    mp.setattr(O, "score_rows", bad)


def _m_transposed_weight(mp):
    def bad(qr, wr, Kd):
        R, H, d = qr.shape
        dots = (qr.reshape(R * H, d) @ Kd.T).reshape(R, H, -1)
        wt = wr[:, ::-1]
        return np.einsum("rh,rhs->rs", wt, O._relu(dots))
    mp.setattr(O, "score_rows", bad)


def _m_head_mean(mp):
    real = O.score_rows
    mp.setattr(O, "score_rows", lambda qr, wr, Kd: real(qr, wr, Kd) / qr.shape[1])


def _m_proxy_sum(mp):
    def bad(q, w, G, *, q_dtype):
        T = q.shape[0]
        ng = (T + G - 1) // G
        return (np.stack([q[g * G:(g + 1) * G].sum(0) for g in range(ng)]),
                np.stack([w[g * G:(g + 1) * G].sum(0) for g in range(ng)]))
    mp.setattr(O, "proxy", bad)


def _m_proxy_first_member(mp):
    def bad(q, w, G, *, q_dtype):
        T = q.shape[0]
        ng = (T + G - 1) // G
        return (np.stack([q[g * G] for g in range(ng)]), np.stack([w[g * G] for g in range(ng)]))
    mp.setattr(O, "proxy", bad)


def _m_decode_first_positions(mp):
    # decode queries placed at the first m positions instead of the last m
    real_dense = O.dense

    def bad(q, w, K, k_offsets, q_offsets, k, k_scale=None, return_scores=False):
        ko = np.asarray(k_offsets)
        qo = np.asarray(q_offsets)
        outs_i, outs_v = [], []
        for b in range(len(ko) - 1):
            r = real_dense(q[qo[b]:qo[b + 1]], w[qo[b]:qo[b + 1]], K[ko[b]:ko[b + 1]], k, q_pos0=0)
            outs_i.append(r["idx"])
            outs_v.append(r["val"])
        return {"idx": np.concatenate(outs_i), "val": np.concatenate(outs_v)}
    mp.setattr(O, "decode", bad)


def _m_decode_group_first_positions(mp):
    # the group's queries placed at the first m_b positions of their cache
    real_group = O.group

    def bad(q, w, K, k, G, bank, mode, q_pos0=0, **kw):
        return real_group(q, w, K, k, G, bank, mode, q_pos0=0, **kw)
    real = O.decode_group

    def dg(*a, **kw):
        with pytest.MonkeyPatch.context() as m2:
            m2.setattr(O, "group", bad)
            return real(*a, **kw)
    mp.setattr(O, "decode_group", dg)


def _m_proxy_unrounded(mp):
    # the proxy query kept at the float64 mean, whatever the queries' dtype
    mp.setattr(O, "round_q", lambda x, q_dtype: np.asarray(x, dtype=np.float64))


def _m_decode_group_scan_first_member(mp):
    # the proxy scans only its first member's prefix: the cache cut at N_b - m_b + 1
    real = O.decode_group

    def dg(q, w, K, k_offsets, q_offsets, k, bank, mode, **kw):
        ko, qo = np.asarray(k_offsets), np.asarray(q_offsets)
        out_i = np.full((int(qo[-1]), k), -1, dtype=np.int64)
        out_v = np.full((int(qo[-1]), k), -np.inf)
        res = {"bank_idx": {}, "bank_val": {}, "count": np.zeros(int(qo[-1]), dtype=np.int64)}
        for b in range(len(ko) - 1):
            Nb, mb = int(ko[b + 1] - ko[b]), int(qo[b + 1] - qo[b])
            r = real(q[qo[b]:qo[b + 1]], w[qo[b]:qo[b + 1]], K[ko[b]:ko[b] + Nb - mb + 1], [0, Nb - mb + 1],
                     [0, mb], k, bank, mode, **kw)
            out_i[qo[b]:qo[b + 1]], out_v[qo[b]:qo[b + 1]] = r["idx"], r["val"]
            res["bank_idx"][b], res["bank_val"][b] = r["bank_idx"][0], r["bank_val"][0]
            res["count"][qo[b]:qo[b + 1]] = r["count"]
        res.update(idx=out_i, val=out_v)
        return res
    mp.setattr(O, "decode_group", dg)


def _m_local_window_before_self(mp):
    # the query-specific keys stop before the member's own position
    real_union = np.union1d

    def bad(a, b):
        b = np.asarray(b)
        return real_union(a, b[:-1]) if b.size and b.dtype.kind == "i" else real_union(a, b)
    mp.setattr(O.np, "union1d", bad)


def _m_local_window_whole_group(mp):
    # every member adds the whole group's keys, its later members' included
    real = O.group

    def bad(q, w, K, k, G, bank, mode, q_pos0=0, **kw):
        if mode != O.REFINE_LOCAL:
            return real(q, w, K, k, G, bank, mode, q_pos0=q_pos0, **kw)
        res = real(q, w, K, k, G, bank, O.REFINE, q_pos0=q_pos0, **kw)
        Kd = O.key_values(K, kw.get("k_scale"))
        T = q.shape[0]
        for t in res["idx"]:
            g = t // G
            p = q_pos0 + t
            last = q_pos0 + min(T, (g + 1) * G) - 1
            b = res["bank_idx"][g]
            cand = np.union1d(b[b <= p], np.arange(q_pos0 + g * G, last + 1))
            S = O.score_rows(q[t:t + 1], w[t:t + 1], Kd[:last + 1])[0]
            si, sv = O.select_topk(S[cand], k, idx=cand)
            res["idx"][t], res["val"][t] = O._pad(si, sv, k)
            res["count"][t] = si.shape[0]
        return res
    mp.setattr(O, "group", bad)


def _m_block_own_block_dropped(mp):
    # the query's own partial block left out of the candidates
    real = O.block_routed

    def bad(q, w, K, k, n_blocks, q_pos0=0, k_scale=None, block=128, reps=None, rows=None):
        Kd = O.key_values(K, k_scale)
        R = O.block_reps(K, block, k_scale) if reps is None else reps
        res = {"idx": {}, "val": {}, "count": {}, "blocks": {}}
        for t in (range(q.shape[0]) if rows is None else rows):
            p = q_pos0 + t
            c = (p + 1) // block
            bs = O.score_rows(q[t:t + 1], w[t:t + 1], R[:c])[0]
            sel, _ = O.select_topk(bs, n_blocks)
            cand = np.concatenate([np.arange(b * block, (b + 1) * block) for b in np.sort(sel)]).astype(np.int64)
            S = O.score_rows(q[t:t + 1], w[t:t + 1], Kd[cand])[0]
            si, sv = O.select_topk(S, k, idx=cand)
            res["idx"][t], res["val"][t] = O._pad(si, sv, k)
            res["count"][t] = si.shape[0]
            res["blocks"][t] = sel
        return res
    mp.setattr(O, "block_routed", bad)


def _m_block_partial_blocks_routed(mp):
    # routing also ranks the block holding the query (its mean includes later keys)
    real = O.block_routed

    def bad(q, w, K, k, n_blocks, q_pos0=0, k_scale=None, block=128, reps=None, rows=None):
        return real(q, w, K, k, n_blocks, q_pos0=q_pos0 + block - 1, k_scale=k_scale, block=block, reps=reps,
                    rows=rows)
    mp.setattr(O, "block_routed", bad)


def _m_kmeans_one_iteration_short(mp):
    # the build stops one Lloyd iteration early
    real = O.kmeans

    def bad(K, C, iters, k_scale=None):
        return real(K, C, max(0, iters - 1), k_scale)
    mp.setattr(O, "kmeans", bad)


def _m_ivf_no_causal_mask(mp):
    # candidates taken from the whole cluster, later keys included
    real = O.ivf_routed

    def bad(q, w, K, k, n_probe, assign, centroids, q_pos0=0, k_scale=None, rows=None):
        return real(q, w, K, k, n_probe, assign, centroids, q_pos0=len(assign) - q.shape[0], k_scale=k_scale,
                    rows=rows)
    mp.setattr(O, "ivf_routed", bad)


def _m_round_bf16_truncate(mp):
    # bf16 rounding that truncates the mantissa instead of rounding to nearest
    def bad(x):
        x = np.asarray(x, dtype=np.float64)
        out = np.zeros_like(x)
        nz = x != 0
        ulp = np.exp2(np.floor(np.log2(np.abs(x[nz]))) - 7)
        out[nz] = np.trunc(x[nz] / ulp) * ulp
        return out
    mp.setattr(O, "round_bf16", bad)


MUTANTS = [_m_no_relu, _m_abs_relu, _m_causal_exclusive, _m_causal_plus_one,
           _m_tiebreak_high, _m_ascending, _m_e4m3_bias8, _m_e4m3_no_subnormal,
           _m_weight_outside, _m_transposed_weight, _m_head_mean, _m_proxy_sum,
           _m_proxy_first_member, _m_proxy_unrounded, _m_decode_first_positions, _m_decode_group_first_positions,
           _m_decode_group_scan_first_member, _m_local_window_before_self, _m_local_window_whole_group,
           _m_block_own_block_dropped, _m_block_partial_blocks_routed, _m_kmeans_one_iteration_short,
           _m_ivf_no_causal_mask, _m_round_bf16_truncate]


@pytest.mark.parametrize("mutant", MUTANTS, ids=[m.__name__ for m in MUTANTS])
def test_mutants_are_caught(mutant):
    caught = []
    for pin in PINS:
        with pytest.MonkeyPatch.context() as mp:
            mutant(mp)
            try:
                pin(O)
            except (AssertionError, ValueError, IndexError):
                caught.append(pin.__name__)
    assert caught, f"no pin catches {mutant.__name__}"
