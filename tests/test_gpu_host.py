"""Host-buffer entry points: inputs and outputs in host memory, staged and
pipelined in row chunks by the library, against the CPU oracle."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_row, check_rows
from synthetic import make_dense_inputs, make_decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def _host(t, pinned=True):
    if t is None:
        return None
    h = t.detach().cpu().contiguous()
    return h.pin_memory() if pinned else h


def _keys(inp):
    if inp.k_dtype == "fp8":
        return inp.k.cpu().numpy(), inp.k_scale.cpu().numpy()
    return _f64(inp.k), None


@pytest.mark.parametrize("chunk_rows", [0, 256, 301], ids=["auto", "256", "ragged301"])
def test_dense_host_chunks(chunk_rows):
    # 1000 rows in chunks of 256 (last 232) or 304 (rounded up to 4; last 88),
    # queries at an offset into 1300 keys
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=1000, N=1300, seed=91)
    k = 128
    idx, val = dsa.dsa_index_dense_host(_host(inp.q), _host(inp.w), _host(inp.k), k, q_pos0=inp.q_pos0,
                                        chunk_rows=chunk_rows)
    assert not idx.is_cuda and idx.shape == (1000, k)
    K, _ = _keys(inp)
    q, w = _f64(inp.q), _f64(inp.w)
    rows = np.r_[0:8, 250:262, 300:310, 600:606, 990:1000]
    scores = [O.score_rows(q[t:t + 1], w[t:t + 1], K[:inp.q_pos0 + t + 1])[0] for t in rows]
    check_rows(idx.numpy()[rows], val.numpy()[rows], scores, k, what=f"dense host chunk={chunk_rows}")


def test_dense_host_fp8_and_pageable():
    # fp8 keys with their scales; pageable (not page-locked) host memory
    inp = make_dense_inputs("fp8_256k", device=DEV, T=300, N=800, seed=92)
    k = 64
    idx, val = dsa.dsa_index_dense_host(_host(inp.q, False), _host(inp.w, False), _host(inp.k, False), k,
                                        q_pos0=inp.q_pos0, K_scale=_host(inp.k_scale, False), chunk_rows=64,
                                        out=(torch.empty((300, k), dtype=torch.int32),
                                             torch.empty((300, k), dtype=torch.float32)))
    K, ks = _keys(inp)
    q, w = _f64(inp.q), _f64(inp.w)
    rows = np.r_[0:5, 60:70, 295:300]
    res = [O.dense(q[t:t + 1], w[t:t + 1], K, k, q_pos0=inp.q_pos0 + int(t), k_scale=ks, return_scores=True)
           for t in rows]
    check_rows(idx.numpy()[rows], val.numpy()[rows], [r["scores"][0] for r in res], k, what="dense host fp8")


def test_dense_host_fp32_simt():
    inp = make_dense_inputs("tiny_fp32_2k", device=DEV, T=200, N=200, seed=93)
    idx, val = dsa.dsa_index_dense_host(_host(inp.q), _host(inp.w), _host(inp.k), 16, q_pos0=0, chunk_rows=40)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    scores = [O.score_rows(q[t:t + 1], w[t:t + 1], K[:t + 1])[0] for t in range(200)]
    check_rows(idx.numpy(), val.numpy(), scores, 16, what="dense host fp32")


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_group_host_chunks(mode):
    # chunk_rows 100 rounds up to 128 = two groups of 64; 640 rows = 5 chunks
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=640, N=700, seed=94)
    G, B, k = 64, 256, 64
    idx, val = dsa.dsa_index_group_host(_host(inp.q), _host(inp.w), _host(inp.k), k, G, B, mode=mode,
                                        q_pos0=inp.q_pos0, chunk_rows=100)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    res = O.group(q, w, K, k, G, B, mode, q_pos0=inp.q_pos0, q_dtype="bf16")
    gi, gv = idx.numpy(), val.numpy()
    for g in range(640 // G):
        bank = res["bank_idx"][g].astype(np.int64)
        ps = res["bank_scores"][g]
        for t in (g * G, g * G + 31, g * G + G - 1):
            p = inp.q_pos0 + t
            cand = bank[bank <= p]
            if mode == dsa.DSA_GROUP_REUSE:
                check_row(gi[t], gv[t], ps[cand], k, what=f"reuse t={t}", idx_map=cand)
            else:
                S = O.score_rows(q[t:t + 1], w[t:t + 1], K[:p + 1])[0]
                check_row(gi[t], gv[t], S[cand], k, what=f"refine t={t}", idx_map=cand)


def test_decode_host():
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[900, 2100, 400], m=[2, 1, 3], seed=95)
    k = 256
    idx, val = dsa.dsa_index_decode_host(_host(inp.q), _host(inp.w), _host(inp.k), k, inp.k_offsets.cpu(),
                                         inp.q_offsets.cpu())
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    ko, qo = inp.k_offsets.cpu().numpy(), inp.q_offsets.cpu().numpy()
    gi, gv = idx.numpy(), val.numpy()
    for b in range(3):
        nb, mb = int(ko[b + 1] - ko[b]), int(qo[b + 1] - qo[b])
        for j in range(mb):
            r, p = int(qo[b]) + j, nb - mb + j
            S = O.score_rows(q[r:r + 1], w[r:r + 1], K[ko[b]:ko[b] + p + 1])[0]
            check_row(gi[r], gv[r], S, k, what=f"decode host b={b} j={j}")


def test_host_staging_too_small():
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=64, N=64, seed=96)
    small = torch.empty(1024, dtype=torch.uint8, device=DEV)
    with pytest.raises(ValueError):
        dsa.dsa_index_dense_host(_host(inp.q), _host(inp.w), _host(inp.k), 8, staging=small)
    need = dsa.dense_host_staging_bytes(64, 64, 64, 128, 8, dsa.DSA_DTYPE_BF16, dsa.DSA_DTYPE_BF16)
    st = torch.empty(need - 256, dtype=torch.uint8, device=DEV)
    q, w, K = _host(inp.q), _host(inp.w), _host(inp.k)
    idx = torch.empty((64, 8), dtype=torch.int32)
    val = torch.empty((64, 8), dtype=torch.float32)
    r = dsa.lib().dsa_index_dense_host(q.data_ptr(), w.data_ptr(), K.data_ptr(), None, 64, 64, 64, 128, 0, 8, 0, 0,
                                       0, idx.data_ptr(), val.data_ptr(), st.data_ptr(), st.numel(), None)
    assert r == -3   # DSA_ERR_WORKSPACE, nothing launched
