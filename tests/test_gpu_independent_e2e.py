"""End-to-end parity with the oracle run entirely on its own: it forms its
own proxies (float64 member means, rounded by the oracle to the queries'
bf16) and block representatives (float64 means rounded to bf16 by its own
round-to-nearest-even), its own banks and routed blocks, and the GPU's outputs are
compared with those.  No GPU intermediate enters the oracle here (the other
group tests also check each GPU stage on the GPU's previous stage, which
isolates a failing stage)."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_row
from synthetic import make_dense_inputs, make_decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["refine", "reuse", "refine_local"])
def test_group_end_to_end(mode):
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=640, N=700, seed=81)
    G, B, k = 64, 256, 64
    idx, val, bi, bv = dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=mode, q_pos0=inp.q_pos0,
                                           return_bank=True, check=True)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    res = O.group(q, w, K, k, G, B, mode, q_pos0=inp.q_pos0, q_dtype="bf16")
    bi, bv, gi, gv = bi.cpu().numpy(), bv.cpu().numpy(), idx.cpu().numpy(), val.cpu().numpy()
    for g in range(q.shape[0] // G):
        ps = res["bank_scores"][g]
        check_row(bi[g], bv[g], ps, B, what=f"bank g={g}")
        bank = res["bank_idx"][g].astype(np.int64)          # the oracle's own bank
        for t in range(g * G, (g + 1) * G):
            p = inp.q_pos0 + t
            cand = bank[bank <= p]
            if mode == dsa.DSA_GROUP_REUSE:
                check_row(gi[t], gv[t], ps[cand], k, what=f"reuse t={t}", idx_map=cand)
            else:
                if mode == dsa.DSA_GROUP_REFINE_LOCAL:
                    cand = np.union1d(cand, np.arange(inp.q_pos0 + g * G, p + 1))
                S = O.score_rows(q[t:t + 1], w[t:t + 1], K[:p + 1])[0]
                check_row(gi[t], gv[t], S[cand], k, what=f"refine t={t}", idx_map=cand)


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_decode_group_end_to_end(mode):
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[700, 1500, 300], m=[2, 3, 1], seed=82)
    k, B = 32, 128
    idx, val = dsa.dsa_index_decode_group(inp.q, inp.w, inp.k, k, inp.k_offsets, inp.q_offsets, B, mode=mode,
                                          check=True)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    ko, qo = inp.k_offsets.numpy(), inp.q_offsets.numpy()
    res = O.decode_group(q, w, K, ko, qo, k, B, mode, q_dtype="bf16")
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    for b in range(3):
        k0, k1, r0, r1 = int(ko[b]), int(ko[b + 1]), int(qo[b]), int(qo[b + 1])
        nb, mb = k1 - k0, r1 - r0
        bank = res["bank_idx"][b].astype(np.int64)
        ps = res["bank_scores"][b]
        for j in range(mb):
            r, p = r0 + j, nb - mb + j
            cand = bank[bank <= p]
            if mode == dsa.DSA_GROUP_REUSE:
                check_row(gi[r], gv[r], ps[cand], k, what=f"reuse b={b} j={j}", idx_map=cand)
            else:
                S = O.score_rows(q[r:r + 1], w[r:r + 1], K[k0:k0 + p + 1])[0]
                check_row(gi[r], gv[r], S[cand], k, what=f"refine b={b} j={j}", idx_map=cand)


def test_block_routed_end_to_end():
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=500, N=1500, seed=83)
    k, nbl = 48, 3
    idx, val, blocks = dsa.dsa_index_block_routed(inp.q, inp.w, inp.k, k, nbl, q_pos0=inp.q_pos0,
                                                  return_blocks=True, check=True)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    R = O.round_bf16(O.block_reps(K, 128))
    res = O.block_routed(q, w, K, k, nbl, q_pos0=inp.q_pos0, reps=R)
    gi, gv, gb = idx.cpu().numpy(), val.cpu().numpy(), blocks.cpu().numpy()
    for t in range(q.shape[0]):
        p = inp.q_pos0 + t
        c = (p + 1) // 128
        bs = O.score_rows(q[t:t + 1], w[t:t + 1], R[:c])[0]
        check_row(gb[t], np.where(gb[t] >= 0, bs[np.maximum(gb[t], 0)], -np.inf).astype(np.float32), bs, nbl,
                  what=f"route t={t}")
        sel = np.sort(res["blocks"][t])                          # the oracle's own routed blocks
        cand = np.concatenate([np.arange(b * 128, (b + 1) * 128) for b in sel] +
                              [np.arange(c * 128, p + 1)]).astype(np.int64)
        S = O.score_rows(q[t:t + 1], w[t:t + 1], K[cand])[0]
        check_row(gi[t], gv[t], S, k, what=f"refine t={t}", idx_map=cand)
