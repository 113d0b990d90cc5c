"""PIVOT in decode (each sequence's new queries form one group): CUDA path
against the CPU oracle.

As for the prefill group form, the GPU's bf16 proxy rows are first checked
against the float64 member means (<= 1 bf16 ulp) and then used as the
oracle's proxy input, so the bank check tests the scan; member checks use the
GPU's bank (whose own check passed)."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_row
from synthetic import make_decode_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def _bf16_ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-38)))
    return 2.0 ** (e - 7)


def _keys(inp):
    if inp.k_dtype == "fp8":
        return O.key_values(inp.k.cpu().numpy(), inp.k_scale.cpu().numpy())
    return _f64(inp.k)


def _check(inp, k, bank, mode, what, seqs=None):
    idx, val, bi, bv, pq, pw = dsa.dsa_index_decode_group(inp.q, inp.w, inp.k, k, inp.k_offsets, inp.q_offsets, bank,
                                                          mode=mode, K_scale=inp.k_scale, return_bank=True,
                                                          return_proxy=True, check=True)
    q, w, Kd = _f64(inp.q), _f64(inp.w), _keys(inp)
    ko, qo = inp.k_offsets.numpy(), inp.q_offsets.numpy()
    B = len(ko) - 1
    gq, gw = _f64(pq), _f64(pw)
    bi, bv, gi, gv = bi.cpu().numpy(), bv.cpu().numpy(), idx.cpu().numpy(), val.cpu().numpy()
    for b in (range(B) if seqs is None else seqs):
        k0, k1, r0, r1 = int(ko[b]), int(ko[b + 1]), int(qo[b]), int(qo[b + 1])
        nb, mb = k1 - k0, r1 - r0
        # proxy: the mean of this sequence's queries, bf16-rounded on the GPU
        qb = q[r0:r1].mean(axis=0)
        assert np.all(np.abs(gq[b] - qb) <= _bf16_ulp(qb) + 1e-30), f"{what}: proxy q of sequence {b}"
        assert np.allclose(gw[b], w[r0:r1].mean(axis=0), rtol=1e-6, atol=1e-7), f"{what}: proxy w of sequence {b}"
        # bank: the proxy's top-bank over the whole cache (it sits at N_b - 1)
        ps = O.score_rows(gq[b:b + 1], gw[b:b + 1], Kd[k0:k1])[0]
        check_row(bi[b], bv[b], ps, bank, what=f"{what} bank b={b}")
        m = bi[b] >= 0
        sv, si = bv[b][m].astype(np.float64), bi[b][m]
        assert np.all(np.diff(sv) <= 0) and np.all((np.diff(sv) < 0) | (np.diff(si) > 0)), f"{what}: bank order"
        bank_keys = si.astype(np.int64)
        for j in range(mb):
            r, p = r0 + j, nb - mb + j
            cand = bank_keys[bank_keys <= p]
            if mode in (dsa.DSA_GROUP_REFINE, dsa.DSA_GROUP_REFINE_LOCAL):
                S = O.score_rows(q[r:r + 1], w[r:r + 1], Kd[k0:k0 + p + 1])[0]
                if mode == dsa.DSA_GROUP_REFINE_LOCAL:
                    cand = np.union1d(cand, np.arange(nb - mb, p + 1))   # the sequence's new keys up to p
                check_row(gi[r], gv[r], S[cand], k, what=f"{what} refine(mode {mode}) b={b} j={j}", idx_map=cand)
            else:
                check_row(gi[r], gv[r], ps[cand], k, what=f"{what} reuse b={b} j={j}", idx_map=cand)
    return idx, val


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["refine", "reuse", "refine_local"])
def test_decode_group_mixed(mode):
    # mixed cache lengths (ragged tiles, one shorter than the bank) and 1..4 queries per sequence
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[300, 700, 1500, 129, 2050, 90],
                             m=[2, 1, 3, 4, 2, 3], seed=31)
    _check(inp, 32, 128, mode, "mixed")


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["refine", "reuse", "refine_local"])
def test_decode_group_fp8(mode):
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[640, 1100, 257], m=[2, 3, 1], seed=32,
                             k_dtype="fp8")
    _check(inp, 24, 96, mode, "fp8")


def test_decode_group_bank_covers_cache_is_decode():
    # a bank as large as every cache makes Refine the decode indexer
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[500, 300, 777], m=[2, 4, 1], seed=33)
    gi, _ = dsa.dsa_index_decode_group(inp.q, inp.w, inp.k, 40, inp.k_offsets, inp.q_offsets, 1024, mode=0,
                                       check=True)
    di, _ = dsa.dsa_index_decode(inp.q, inp.w, inp.k, 40, inp.k_offsets, inp.q_offsets, check=True)
    a, b = gi.cpu().numpy(), di.cpu().numpy()
    for r in range(a.shape[0]):
        assert set(a[r].tolist()) == set(b[r].tolist()), r


def test_decode_group_single_query_is_decode():
    # one query per sequence: the proxy is the query (bf16 mean of one row)
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[900, 2000, 450], m=1, seed=34)
    di, _ = dsa.dsa_index_decode(inp.q, inp.w, inp.k, 64, inp.k_offsets, inp.q_offsets, check=True)
    for mode in (0, 1):
        gi, _ = dsa.dsa_index_decode_group(inp.q, inp.w, inp.k, 64, inp.k_offsets, inp.q_offsets, 256, mode=mode,
                                           check=True)
        a, b = gi.cpu().numpy(), di.cpu().numpy()
        for r in range(a.shape[0]):
            assert set(a[r].tolist()) == set(b[r].tolist()), (mode, r)


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_decode_group_without_bank_output(mode):
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV, lengths=[300, 700, 1500, 129], m=[2, 1, 3, 4],
                             seed=35)
    fi, fv, _, _ = dsa.dsa_index_decode_group(inp.q, inp.w, inp.k, 32, inp.k_offsets, inp.q_offsets, 128, mode=mode,
                                              return_bank=True, check=True)
    pi, pv = dsa.dsa_index_decode_group(inp.q, inp.w, inp.k, 32, inp.k_offsets, inp.q_offsets, 128, mode=mode,
                                        check=True)
    ai, ap = torch.sort(fi, dim=1)
    bi, bp = torch.sort(pi, dim=1)
    assert torch.equal(ai, bi)
    assert torch.equal(torch.gather(fv, 1, ap), torch.gather(pv, 1, bp))


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_decode_group_full_size_sampled(mode):
    # the 32 x 128K decode batch, 2 queries per sequence, bank 8192, k 2048
    inp = make_decode_inputs("decode_bf16_32x128k", device=DEV)
    _check(inp, 2048, 8192, mode, "full", seqs=[0, 17, 31])
