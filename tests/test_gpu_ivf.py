"""Inverted-file routing (plain k-means index): CUDA path against the CPU oracle.

The index build is pinned by (1) one Lloyd iteration, which the oracle
reproduces from the same start (nearest initial centroid, then member
means), and (2) the fixed-point properties after several iterations: every
key sits with a nearest centroid and every centroid is its members' mean,
and the clustered key layout matches the assignment.  Routing and refine
are then checked against the oracle run on the GPU's own index (its bf16
routing centroids and its assignment), since k-means trajectories may part
at fp32 near-ties."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_row
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def _keys(inp):
    if inp.k_dtype == "fp8":
        return O.key_values(inp.k.cpu().numpy(), inp.k_scale.cpu().numpy())
    return _f64(inp.k)


def _check_layout(ix, Kraw, Kd, C):
    off = ix.part("off").cpu().numpy().astype(np.int64)
    perm = ix.part("perm").cpu().numpy().astype(np.int64)
    a = ix.part("assign").cpu().numpy().astype(np.int64)
    N = Kd.shape[0]
    assert off[0] == 0 and off[-1] == N and np.all(np.diff(off) == np.bincount(a, minlength=C))
    assert np.array_equal(np.sort(perm), np.arange(N))
    for c in range(C):
        assert np.all(a[perm[off[c]:off[c + 1]]] == c)
    ks = ix.part("keys").cpu()
    assert torch.equal(ks.view(torch.int16), Kraw[perm].view(torch.int16))   # the bf16 bytes, moved
    cen = ix.part("centroids").cpu().numpy().astype(np.float64)
    cb = ix.part("centroids_bf16").cpu().float().numpy().astype(np.float64)
    assert np.array_equal(cb, torch.tensor(cen, dtype=torch.float32).to(torch.bfloat16).float().numpy())
    return a, cen


def _nearest_ok(Kd, a, cen):
    d2 = (Kd * Kd).sum(1)[:, None] - 2.0 * Kd @ cen.T + (cen * cen).sum(1)[None, :]
    scale = (Kd * Kd).sum(1) + (cen * cen).sum(1).max()
    return np.all(d2[np.arange(Kd.shape[0]), a] <= d2.min(1) + 1e-5 * scale)


def test_ivf_build_one_iteration_matches_oracle():
    inp = make_dense_inputs("fp8_256k", device=DEV, T=64, N=3000, seed=61)
    Kd = _keys(inp)
    ix = dsa.dsa_ivf_build(inp.k, 24, iters=1, K_scale=inp.k_scale, check=True)
    Kw = inp.k.view(torch.float8_e4m3fn).to(torch.bfloat16).cpu()   # the widened bytes the index holds
    a, cen = _check_layout(ix, Kw, Kd, 24)
    oa, oc = O.kmeans(inp.k.cpu().numpy(), 24, 1, inp.k_scale.cpu().numpy())
    # same start, one assignment: identical up to fp32 near-ties
    init = Kd[(np.arange(24) * Kd.shape[0]) // 24]
    assert _nearest_ok(Kd, a, init)
    assert np.mean(a == oa) > 0.99
    for c in range(24):
        m = a == c
        if m.any():
            assert np.allclose(cen[c], Kd[m].mean(0), rtol=1e-5, atol=1e-5 * np.abs(Kd[m]).mean())


def test_ivf_build_fixed_point():
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=64, N=4096, seed=62)
    Kd = _f64(inp.k)
    ix = dsa.dsa_ivf_build(inp.k, 32, iters=6, check=True)
    a, cen = _check_layout(ix, inp.k.cpu(), Kd, 32)
    # the last assignment is nearest to the centroids it produced the means of
    # only after convergence; here: centroids are the members' means, and each
    # key was nearest to the previous centroids (checked via a 7th assignment)
    for c in range(32):
        m = a == c
        if m.any():
            assert np.allclose(cen[c], Kd[m].mean(0), rtol=1e-5, atol=1e-5 * np.abs(Kd[m]).mean())
    ix7 = dsa.dsa_ivf_build(inp.k, 32, iters=7, check=True)
    a7 = ix7.part("assign").cpu().numpy()
    assert _nearest_ok(Kd, a7.astype(np.int64), cen) or np.mean(a7 == a) > 0.99


def _check_routed(inp, C, iters, k, n_probe, what, rows=None):
    ix = dsa.dsa_ivf_build(inp.k, C, iters=iters, K_scale=inp.k_scale, check=True)
    idx, val, ci = dsa.dsa_index_ivf_routed(inp.q, inp.w, ix, k, n_probe, q_pos0=inp.q_pos0, K_scale=inp.k_scale,
                                            return_clusters=True, check=True)
    Kd = _keys(inp)
    a = ix.part("assign").cpu().numpy().astype(np.int64)
    cb = ix.part("centroids_bf16").cpu().double().numpy()
    q, w = _f64(inp.q), _f64(inp.w)
    gi, gv, gc = idx.cpu().numpy(), val.cpu().numpy(), ci.cpu().numpy()
    for t in (range(q.shape[0]) if rows is None else rows):
        p = inp.q_pos0 + t
        cs = O.score_rows(q[t:t + 1], w[t:t + 1], cb)[0]
        check_row(gc[t], cs[gc[t]].astype(np.float32), cs, n_probe, what=f"{what} route t={t}")
        cand = np.nonzero(np.isin(a[:p + 1], gc[t]))[0].astype(np.int64)
        S = O.score_rows(q[t:t + 1], w[t:t + 1], Kd[cand])[0]
        check_row(gi[t], gv[t], S, k, what=f"{what} refine t={t}", idx_map=cand)
    return ix, idx


def test_ivf_routed_small():
    inp = make_dense_inputs("fp8_256k", device=DEV, T=300, N=3000, seed=63)
    _check_routed(inp, 40, 4, 48, 5, "small")


def test_ivf_routed_bf16_from_zero():
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=500, N=500, q_pos0=0, seed=64)
    _check_routed(inp, 16, 3, 32, 3, "pos0")


def test_ivf_all_clusters_is_dense():
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=200, N=1500, seed=65)
    ix = dsa.dsa_ivf_build(inp.k, 12, iters=3, check=True)
    ri, _ = dsa.dsa_index_ivf_routed(inp.q, inp.w, ix, 40, 12, q_pos0=inp.q_pos0, check=True)
    di, _ = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 40, q_pos0=inp.q_pos0, check=True)
    a, b = ri.cpu().numpy(), di.cpu().numpy()
    for t in range(200):
        assert set(a[t].tolist()) == set(b[t].tolist()), t


def test_ivf_routed_full_size_sampled():
    # the fp8 256K keys (last 4096 queries), 2048 clusters, 64 probed (about 8K keys)
    inp = make_dense_inputs("fp8_256k", device=DEV, T=4096)
    _check_routed(inp, 2048, 4, 2048, 64, "full", rows=[0, 2047, 4095])
