"""Group-shared (PIVOT) indexer: CUDA path against the CPU oracle.

Following the oracle's reading of the proxy precision, the proxy rows the
GPU rounded to bf16 are first checked against the float64 member means
(<= 1 bf16 ulp), then used as the oracle's proxy input, so the bank check
tests the scan.  Member checks use the GPU's bank (whose own check passed)."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_group_sample, check_row, sample_groups
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def _bf16_ulp(x):
    e = np.floor(np.log2(np.maximum(np.abs(x), 1e-38)))
    return 2.0 ** (e - 7)


def _run_group(inp, k, G, B, mode):
    return dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=mode, q_pos0=inp.q_pos0, return_bank=True,
                               return_proxy=True, check=True)


def _check_group(inp, k, G, B, mode, what):
    idx, val, bidx, bval, pq, pw = _run_group(inp, k, G, B, mode)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    T = q.shape[0]
    ng = (T + G - 1) // G
    # proxy: GPU bf16 rounding of the fp32 mean within one ulp of the fp64 mean
    # the unrounded float64 means, to bound the GPU's fp32 mean + bf16 rounding
    qb, wb = O.proxy(q, w, G, q_dtype="f64")
    gq, gw = _f64(pq), _f64(pw)
    assert np.all(np.abs(gq - qb) <= _bf16_ulp(qb) + 1e-30), f"{what}: proxy q off by more than 1 bf16 ulp"
    assert np.allclose(gw, wb, rtol=1e-6, atol=1e-7), f"{what}: proxy w"
    res = O.group(q, w, K, k, G, B, O.REFINE, q_pos0=inp.q_pos0, qbar=gq, wbar=gw, q_dtype="bf16")
    bi, bv = bidx.cpu().numpy(), bval.cpu().numpy()
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    for g in range(ng):
        ps = res["bank_scores"][g]
        # bank = the proxy's top-B over its prefix
        check_row(bi[g], bv[g], ps, B, what=f"{what} bank g={g}")
        # ranked: scores non-increasing, equal scores by ascending key
        m = bi[g] >= 0
        sv, si = bv[g][m].astype(np.float64), bi[g][m]
        assert np.all(np.diff(sv) <= 0) and np.all((np.diff(sv) < 0) | (np.diff(si) > 0)), f"{what}: bank order"
        bank = bi[g][m].astype(np.int64)
        for t in range(g * G, min(T, (g + 1) * G)):
            p = inp.q_pos0 + t
            cand = bank[bank <= p]
            if mode in (dsa.DSA_GROUP_REFINE, dsa.DSA_GROUP_REFINE_LOCAL):
                S = O.score_rows(q[t:t + 1], w[t:t + 1], K[:p + 1])[0]
                if mode == dsa.DSA_GROUP_REFINE_LOCAL:
                    # plus the member's own stretch of the group
                    cand = np.union1d(cand, np.arange(inp.q_pos0 + g * G, p + 1))
                check_row(gi[t], gv[t], S[cand], k, what=f"{what} refine(mode {mode}) t={t}", idx_map=cand)
            else:
                # Reuse: the first k bank keys it may see, in the proxy's ranking,
                # valued by the proxy score
                check_row(gi[t], gv[t], ps[cand], k, what=f"{what} reuse t={t}", idx_map=cand)
    return idx, val


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["refine", "reuse", "refine_local"])
def test_group_small(mode):
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=640, N=640, seed=21)
    _check_group(inp, 64, 64, 256, mode, "G64 B256")


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["refine", "reuse", "refine_local"])
def test_group_ragged(mode):
    # group size not a multiple of the 4-query unit, partial last group, offset queries
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=100, N=700, seed=22)
    _check_group(inp, 16, 6, 48, mode, "G6 B48")


def test_refine_full_bank_equals_dense():
    # a bank covering the whole prefix makes Refine the dense indexer (same
    # kernel arithmetic on the same keys: identical sets)
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=300, N=300, seed=23)
    gi, _ = dsa.dsa_index_group(inp.q, inp.w, inp.k, 50, 16, 512, mode=0, q_pos0=0, check=True)
    di, _ = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 50, q_pos0=0, check=True)
    a, b = gi.cpu().numpy(), di.cpu().numpy()
    for t in range(300):
        assert set(a[t].tolist()) == set(b[t].tolist()), t


def test_group_size_one_matches_dense():
    # G = 1: the proxy is the query itself (bf16 mean of one row = the row)
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=120, N=400, seed=24)
    di, dv = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 32, q_pos0=inp.q_pos0, check=True)
    for mode in (0, 1):
        gi, gv = dsa.dsa_index_group(inp.q, inp.w, inp.k, 32, 1, 64, mode=mode, q_pos0=inp.q_pos0, check=True)
        a, b = gi.cpu().numpy(), di.cpu().numpy()
        for t in range(120):
            assert set(a[t].tolist()) == set(b[t].tolist()), (mode, t)


def _same_rows(a_idx, a_val, b_idx, b_val):
    # equal row sets (outputs are sets): sort each row by index on the device
    ai, ap = torch.sort(a_idx, dim=1)
    bi, bp = torch.sort(b_idx, dim=1)
    assert torch.equal(ai, bi)
    assert torch.equal(torch.gather(a_val, 1, ap), torch.gather(b_val, 1, bp))


@pytest.mark.parametrize("mode", [0, 1, 2], ids=["refine", "reuse", "refine_local"])
@pytest.mark.parametrize("shape", [(640, 640, 64, 256, 64), (100, 700, 6, 48, 16), (300, 300, 64, 2048, 100)],
                         ids=["G64", "G6", "bank-ge-prefix"])
def test_group_without_bank_output(mode, shape):
    # without a bank output Refine skips the ranking and Reuse ranks only the
    # top k + G - 1 bank entries: member outputs equal the fully ranked path's
    T, N, G, B, k = shape
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=T, N=N, seed=25)
    fi, fv, _, _, _, _ = _run_group(inp, k, G, B, mode)
    pi, pv = dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=mode, q_pos0=inp.q_pos0, check=True)
    _same_rows(fi, fv, pi, pv)


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_group_full_size_sampled(mode):
    # the 128K group workload (G = 64, B = 8192, k = 2048) at full size: eight
    # whole groups in adjacent pairs (512 members, group boundaries included)
    inp = make_dense_inputs("group_bf16_128k", device=DEV)
    G, B, k = 64, 8192, 2048
    T = inp.q.shape[0]
    idx, val, bidx, bval = dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=mode, q_pos0=inp.q_pos0,
                                               return_bank=True, check=True)
    # the bench's call (no bank output) gives the same member sets
    pi, pv = dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=mode, q_pos0=inp.q_pos0, check=True)
    _same_rows(idx, val, pi, pv)
    del pi, pv
    groups = sample_groups(T // G, G, q_pos0=inp.q_pos0, seed=3)
    assert len(groups) == 8 and groups[0] == 0 and groups[-1] == T // G - 1
    check_group_sample(inp.q, inp.w, _f64(inp.k), idx.cpu().numpy(), val.cpu().numpy(), bidx.cpu().numpy(),
                       bval.cpu().numpy(), groups, G, B, k, mode, inp.q_pos0, "bf16", what=f"128K mode {mode}")


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_group_fp8_keys(mode):
    inp = make_dense_inputs("fp8_256k", device=DEV, T=256, N=512)
    idx, val, bidx, bval, pq, pw = dsa.dsa_index_group(inp.q, inp.w, inp.k, 32, 64, 128, mode=mode,
                                                       q_pos0=inp.q_pos0, K_scale=inp.k_scale, return_bank=True,
                                                       return_proxy=True, check=True)
    Kd = O.key_values(inp.k.cpu().numpy(), inp.k_scale.cpu().numpy())
    gq, gw = _f64(pq), _f64(pw)
    bi, bv = bidx.cpu().numpy(), bval.cpu().numpy()
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    q, w = _f64(inp.q), _f64(inp.w)
    for g in range(4):
        L = inp.q_pos0 + (g + 1) * 64 - 1
        ps = O.score_rows(gq[g:g + 1], gw[g:g + 1], Kd[:L + 1])[0]
        check_row(bi[g], bv[g], ps, 128, what=f"fp8 bank g={g}")
        bank = bi[g][bi[g] >= 0].astype(np.int64)
        for t in range(g * 64, (g + 1) * 64, 9):
            p = inp.q_pos0 + t
            cand = bank[bank <= p]
            S = (O.score_rows(q[t:t + 1], w[t:t + 1], Kd[:p + 1])[0] if mode == 0 else ps)
            check_row(gi[t], gv[t], S[cand], 32, what=f"fp8 member t={t}", idx_map=cand)


def test_refine_local_full_size_sampled():
    # the 128K group workload with query-specific additions: eight whole groups
    inp = make_dense_inputs("group_bf16_128k", device=DEV)
    G, B, k = 64, 8192, 2048
    T = inp.q.shape[0]
    idx, val, bidx, bval = dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=dsa.DSA_GROUP_REFINE_LOCAL,
                                               q_pos0=inp.q_pos0, return_bank=True, check=True)
    groups = sample_groups(T // G, G, q_pos0=inp.q_pos0, seed=4)
    check_group_sample(inp.q, inp.w, _f64(inp.k), idx.cpu().numpy(), val.cpu().numpy(), bidx.cpu().numpy(),
                       bval.cpu().numpy(), groups, G, B, k, O.REFINE_LOCAL, inp.q_pos0, "bf16",
                       what="128K refine_local")


@pytest.mark.parametrize("mode", [0, 1], ids=["refine", "reuse"])
def test_group_maximum_bank(mode):
    # the largest bank the ABI takes (16384) with k = 4096
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=192, N=20000, seed=72)
    _check_group(inp, 4096, 64, 16384, mode, "bank 16384")
