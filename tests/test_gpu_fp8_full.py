"""The 256K workload with fp8 keys (e4m3 bytes and a per-token scale) at its
full size, T = N = 262144, in the launch configuration the benchmark times:
dense and group-shared (Refine, Reuse) selection, checked against the CPU
oracle on 512 sampled rows (dense) and eight whole groups of 64 members
(group).  The oracle decodes the fp8 keys itself and forms its own proxies
(float64 means rounded to bf16); member checks use the GPU's bank once that
bank has passed its own check, since at 256K keys the proxy scores around
the bank boundary lie far closer together than the parity tolerance."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_group_sample, check_rows, sample_groups, sample_rows
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
    # 512 seeded rows: first and last units, rows below k, tile edges, rows at
    # and just after planted needle keys, uniform rows
    T = inp.q.shape[0]
    assert T == 262144 and keys.shape[0] == 262144
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, K_TOP, q_pos0=inp.q_pos0, K_scale=inp.k_scale, check=True)
    rows = sample_rows(T, K_TOP, n=512, seed=4, q_pos0=inp.q_pos0, needles=inp.needles)
    nd = inp.needles.numpy()
    assert len(rows) == 512 and np.isin(nd - inp.q_pos0, rows).sum() >= 20
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    for c0 in range(0, len(rows), 16):
        ch = rows[c0:c0 + 16]
        sel = torch.as_tensor(ch, device=DEV)
        q, w = _f64(inp.q[sel]), _f64(inp.w[sel])
        scores = [O.score_rows(q[j:j + 1], w[j:j + 1], keys[:inp.q_pos0 + r + 1])[0] for j, r in enumerate(ch)]
        check_rows(gi[ch], gv[ch], scores, K_TOP, what=f"fp8 256K dense rows {ch[0]}..")


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_fp8_group_full_size_sampled(inp, keys, mode):
    # eight whole groups in adjacent pairs (512 members), two pairs around
    # groups that hold needle keys
    T = inp.q.shape[0]
    idx, val, bidx, bval = dsa.dsa_index_group(inp.q, inp.w, inp.k, K_TOP, G, BANK, mode=mode, q_pos0=inp.q_pos0,
                                               K_scale=inp.k_scale, return_bank=True, check=True)
    groups = sample_groups(T // G, G, q_pos0=inp.q_pos0, needles=inp.needles, seed=5)
    check_group_sample(inp.q, inp.w, keys, idx.cpu().numpy(), val.cpu().numpy(), bidx.cpu().numpy(),
                       bval.cpu().numpy(), groups, G, BANK, K_TOP, mode, inp.q_pos0, "bf16",
                       what=f"fp8 256K mode {mode}")
