"""The 256K workload with fp8 keys (e4m3 bytes and a per-token scale) at its
full size, T = N = 262144, in the launch configuration the benchmark times:
dense and group-shared (Refine, Reuse) selection, checked against the CPU
oracle on sampled rows and groups.  The oracle decodes the fp8 keys itself
and forms its own proxies (float64 means rounded to bf16); member checks use
the GPU's bank once that bank has passed its own check, since at 256K keys
the proxy scores around the bank boundary lie far closer together than the
parity tolerance."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_row, check_rows
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
K_TOP, G, BANK = 2048, 64, 8192


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


@pytest.fixture(scope="module")
def inp():
    return make_dense_inputs("fp8_256k", device=DEV)


@pytest.fixture(scope="module")
def keys(inp):
    # the oracle's own decoding of the stored e4m3 bytes, times each token's scale
    return O.key_values(inp.k.cpu().numpy(), inp.k_scale.cpu().numpy())


def test_fp8_dense_full_size_sampled(inp, keys):
    T = inp.q.shape[0]
    assert T == 262144 and keys.shape[0] == 262144
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, K_TOP, q_pos0=inp.q_pos0, K_scale=inp.k_scale, check=True)
    rows = [0, 2047, 2048, 100003, T - 1]
    sel = torch.as_tensor(rows, device=DEV)
    q, w = _f64(inp.q[sel]), _f64(inp.w[sel])
    scores = [O.score_rows(q[j:j + 1], w[j:j + 1], keys[:inp.q_pos0 + r + 1])[0] for j, r in enumerate(rows)]
    check_rows(idx[sel].cpu().numpy(), val[sel].cpu().numpy(), scores, K_TOP, what="fp8 256K dense")


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_fp8_group_full_size_sampled(inp, keys, mode):
    T = inp.q.shape[0]
    idx, val, bidx, bval = dsa.dsa_index_group(inp.q, inp.w, inp.k, K_TOP, G, BANK, mode=mode, q_pos0=inp.q_pos0,
                                               K_scale=inp.k_scale, return_bank=True, check=True)
    for g in (0, 1000, T // G - 1):
        r0, r1 = g * G, min(T, (g + 1) * G)
        q, w = _f64(inp.q[r0:r1]), _f64(inp.w[r0:r1])
        qb, wb = O.proxy(q, w, G, q_dtype="bf16")
        L = inp.q_pos0 + r1 - 1
        ps = O.score_rows(qb, wb, keys[:L + 1])[0]
        bi, bv = bidx[g].cpu().numpy(), bval[g].cpu().numpy()
        check_row(bi, bv, ps, BANK, what=f"fp8 256K bank g={g}")
        bank = bi[bi >= 0].astype(np.int64)
        gi, gv = idx[r0:r1].cpu().numpy(), val[r0:r1].cpu().numpy()
        for j in (0, 37, r1 - r0 - 1):
            p = inp.q_pos0 + r0 + j
            cand = bank[bank <= p]
            if mode == dsa.DSA_GROUP_REFINE:
                S = O.score_rows(q[j:j + 1], w[j:j + 1], keys[:p + 1])[0]
                check_row(gi[j], gv[j], S[cand], K_TOP, what=f"fp8 256K refine t={r0 + j}", idx_map=cand)
            else:
                check_row(gi[j], gv[j], ps[cand], K_TOP, what=f"fp8 256K reuse t={r0 + j}", idx_map=cand)
