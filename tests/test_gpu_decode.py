"""Decode indexer over a batch of key caches: CUDA path against the CPU oracle."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_rows
from synthetic import make_decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def _check(inp, k, rows=None, what=""):
    idx, val = dsa.dsa_index_decode(inp.q, inp.w, inp.k, k, inp.k_offsets, inp.q_offsets, K_scale=inp.k_scale,
                                    check=True)
    if inp.k_dtype == "fp8":
        K, ks = inp.k.cpu().numpy(), inp.k_scale.cpu().numpy()
    else:
        K, ks = _f64(inp.k), None
    ko, qo = inp.k_offsets.numpy(), inp.q_offsets.numpy()
    q, w = _f64(inp.q), _f64(inp.w)
    B = len(ko) - 1
    rows = range(int(qo[-1])) if rows is None else rows
    scores, sel = [], []
    for r in rows:
        b = int(np.searchsorted(qo, r, side="right") - 1)
        nb, mb = int(ko[b + 1] - ko[b]), int(qo[b + 1] - qo[b])
        p = nb - mb + (r - int(qo[b]))
        Kd = O.key_values(K[ko[b]:ko[b] + p + 1], None if ks is None else ks[ko[b]:ko[b] + p + 1])
        scores.append(O.score_rows(q[r:r + 1], w[r:r + 1], Kd)[0])
        sel.append(r)
    gi, gv = idx.cpu().numpy()[sel], val.cpu().numpy()[sel]
    check_rows(gi, gv, scores, k, what=what)
    return idx, val


def test_decode_tensor_core_mixed_lengths():
    inp = make_decode_inputs(device=DEV, lengths=[300, 17, 1000, 129, 4096, 1], m=[2, 1, 3, 4, 2, 1], seed=31)
    _check(inp, 128, what="decode tc")


def test_decode_k_exceeds_cache():
    inp = make_decode_inputs(device=DEV, lengths=[50, 200, 7], m=[1, 2, 3], seed=32)
    idx, _ = _check(inp, 300, what="decode k>N")
    cnt = (idx >= 0).sum(dim=1).cpu().tolist()
    assert cnt == [50, 199, 200, 5, 6, 7]


def test_decode_cuda_core_fp32():
    inp = make_decode_inputs(device=DEV, lengths=[700, 33, 2000], m=[2, 1, 2], H=8, d=32, seed=33)
    inp.q = inp.q.float()
    inp.k = inp.k.float()
    inp.q_dtype = inp.k_dtype = "fp32"
    _check(inp, 64, what="decode fp32")


def test_decode_fp8_keys_cuda_core():
    inp = make_decode_inputs(device=DEV, lengths=[900, 64], m=[2, 1], H=16, d=64, seed=34, k_dtype="fp8")
    _check(inp, 100, what="decode fp8")


def test_decode_matches_dense_tail():
    # one sequence: decode of its last m positions equals dense prefill there
    inp = make_decode_inputs(device=DEV, lengths=[1500], m=[4], seed=35)
    di, dv = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 200, q_pos0=1500 - 4, check=True)
    ci, cv = dsa.dsa_index_decode(inp.q, inp.w, inp.k, 200, inp.k_offsets, inp.q_offsets, check=True)
    a, b = ci.cpu().numpy(), di.cpu().numpy()
    for t in range(4):
        assert set(a[t].tolist()) == set(b[t].tolist())


def test_decode_full_size_all_rows():
    # 32 caches x 131072 keys, 2 queries each, k = 2048: every one of the 64 rows
    inp = make_decode_inputs(device=DEV)
    assert int(inp.q_offsets[-1]) == 64
    _check(inp, 2048, rows=None, what="decode 32x128K")


def test_decode_fp8_keys_tensor_core():
    inp = make_decode_inputs(device=DEV, lengths=[1200, 300, 77], m=[2, 3, 1], seed=36, k_dtype="fp8")
    _check(inp, 96, what="decode fp8 tc")
