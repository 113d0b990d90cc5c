"""Two-stage selection over 128-key blocks (block routing): CUDA path
against the CPU oracle.  The GPU's bf16 block representatives are checked
against the float64 block means (<= 1 bf16 ulp) and then used as the
oracle's representatives, so the routing check tests the routing; each
row's refine is checked on the GPU's routed blocks (whose own check passed)."""
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


def _bf16_ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-38)))
    return 2.0 ** (e - 7)


def _check(inp, k, n_blocks, what, rows=None):
    idx, val, bidx, reps = dsa.dsa_index_block_routed(inp.q, inp.w, inp.k, k, n_blocks, q_pos0=inp.q_pos0,
                                                      K_scale=inp.k_scale, return_blocks=True, return_reps=True,
                                                      check=True)
    if inp.k_dtype == "fp8":
        Kraw, ks = inp.k.cpu().numpy(), inp.k_scale.cpu().numpy()
    else:
        Kraw, ks = _f64(inp.k), None
    Kd = O.key_values(Kraw, ks)
    R64 = O.block_reps(Kraw, 128, ks)
    R = _f64(reps)
    # fp32 sums of 128 keys, then bf16: 1 bf16 ulp plus the sum's own
    # rounding, 128 * 2^-24 of the block's mean |key| (means that cancel)
    A = np.stack([np.abs(Kd[b * 128:(b + 1) * 128]).mean(axis=0) for b in range(R64.shape[0])])
    assert np.all(np.abs(R - R64) <= _bf16_ulp(R64) + 128 * 2.0 ** -24 * A + 1e-30), f"{what}: block representatives"
    q, w = _f64(inp.q), _f64(inp.w)
    T = q.shape[0]
    gi, gv, bi = idx.cpu().numpy(), val.cpu().numpy(), bidx.cpu().numpy()
    for t in (range(T) if rows is None else rows):
        p = inp.q_pos0 + t
        c = (p + 1) // 128
        # routing: the best n_blocks complete blocks by the representatives' score
        if c > 0:
            bs = O.score_rows(q[t:t + 1], w[t:t + 1], R[:c])[0]
            check_row(bi[t], np.where(bi[t] >= 0, bs[np.maximum(bi[t], 0)], -np.inf).astype(np.float32),
                      bs, n_blocks, what=f"{what} route t={t}")
        sel = bi[t][bi[t] >= 0].astype(np.int64)
        cand = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in np.sort(sel)] +
                              [np.arange(c * 128, p + 1)]).astype(np.int64)
        S = O.score_rows(q[t:t + 1], w[t:t + 1], Kd[cand])[0]
        check_row(gi[t], gv[t], S, k, what=f"{what} refine t={t}", idx_map=cand)
    return idx, val


def test_block_routed_small():
    # rows before, at and after block edges; queries with no complete block
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=700, N=1400, seed=51)
    _check(inp, 64, 3, "small")


def test_block_routed_from_position_zero():
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=400, N=400, q_pos0=0, seed=52)
    _check(inp, 32, 2, "pos0")


def test_block_routed_fp8():
    inp = make_dense_inputs("fp8_256k", device=DEV, T=300, N=2000, seed=53)
    _check(inp, 48, 4, "fp8")


def test_block_routed_all_blocks_is_dense():
    # routing every complete block: the candidates are the whole prefix
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=256, N=1024, seed=54)
    ri, _ = dsa.dsa_index_block_routed(inp.q, inp.w, inp.k, 50, 8, q_pos0=inp.q_pos0, check=True)
    di, _ = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 50, q_pos0=inp.q_pos0, check=True)
    a, b = ri.cpu().numpy(), di.cpu().numpy()
    for t in range(256):
        assert set(a[t].tolist()) == set(b[t].tolist()), t


def test_block_routed_full_size_sampled():
    # the fp8 256K workload with an 8K-key candidate budget (64 blocks), sampled rows
    inp = make_dense_inputs("fp8_256k", device=DEV, T=8192)
    _check(inp, 2048, 64, "full", rows=[0, 1, 4095, 8191])
