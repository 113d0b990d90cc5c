"""The dense entry point that allocates nothing (dsa_index_dense_static).

Some callers cannot give the library a workspace (a host application that
has reserved all device memory for itself, a loop where a late cudaMalloc
may fail or stall).  This entry point keeps its scratch in a fixed array the
library reserves on load.  Its results must equal those of dsa_index_dense on
the same inputs, call after call: the shared array keeps the previous call's
contents, which must not leak into the next call.

This file is collected last so that a run stopping at the first failure has
run every other test first; it also passes alone in a fresh process.
"""
import ctypes

import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import RTOL, check_rows
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _static_call(q, w, K, k, q_pos0):
    """Through the C ABI directly: nothing but the caller's tensors."""
    T, H, d = q.shape
    N = K.shape[0]
    idx = torch.full((T, k), -7, dtype=torch.int32, device=DEV)
    val = torch.zeros((T, k), dtype=torch.float32, device=DEV)
    st = torch.cuda.current_stream().cuda_stream
    rc = dsa.lib().dsa_index_dense_static(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                          ctypes.c_void_p(K.data_ptr()), T, N, H, d, q_pos0, k,
                                          ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(val.data_ptr()),
                                          ctypes.c_void_p(st))
    assert rc == 0, dsa.lib().dsa_status_string(rc)
    return idx, val


def _same(a_idx, a_val, b_idx, b_val):
    ai, av = a_idx.cpu().numpy(), a_val.cpu().numpy()
    bi, bv = b_idx.cpu().numpy(), b_val.cpu().numpy()
    for t in range(ai.shape[0]):
        oa, ob = np.argsort(ai[t]), np.argsort(bi[t])
        assert np.array_equal(ai[t][oa], bi[t][ob]), f"row {t}: index sets differ"
        va, vb = av[t][oa].astype(np.float64), bv[t][ob].astype(np.float64)
        fin = np.isfinite(vb)
        assert np.array_equal(np.isfinite(va), fin)
        assert np.all(np.abs(va[fin] - vb[fin]) <= RTOL * np.abs(vb[fin])), f"row {t}: scores differ"


def test_static_scratch_matches_workspace_entry_point_twice():
    # two calls in a row with different problems: the second must not see the
    # first one's leftovers in the shared scratch
    cases = [dict(T=333, N=1500, seed=51, k=200), dict(T=260, N=700, seed=52, k=64)]
    for c in cases:
        inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=c["T"], N=c["N"], seed=c["seed"])
        si, sv = _static_call(inp.q, inp.w, inp.k, c["k"], inp.q_pos0)
        ri, rv = dsa.dsa_index_dense(inp.q, inp.w, inp.k, c["k"], q_pos0=inp.q_pos0, check=True)
        _same(si, sv, ri, rv)
        # and against the CPU oracle itself, every row
        r = O.dense(inp.q.double().cpu().numpy(), inp.w.double().cpu().numpy(), inp.k.double().cpu().numpy(),
                    c["k"], q_pos0=inp.q_pos0, return_scores=True)
        check_rows(si.cpu().numpy(), sv.cpu().numpy(), r["scores"], c["k"], what="static entry")


def test_static_scratch_rejects_oversize():
    # more keys than the fixed scratch holds even for a single CTA
    q = torch.zeros((1, 64, 128), dtype=torch.bfloat16, device=DEV)
    w = torch.zeros((1, 64), dtype=torch.float32, device=DEV)
    N = 1 << 21
    K = torch.zeros((N, 128), dtype=torch.bfloat16, device=DEV)
    idx = torch.empty((1, 4), dtype=torch.int32, device=DEV)
    val = torch.empty((1, 4), dtype=torch.float32, device=DEV)
    rc = dsa.lib().dsa_index_dense_static(ctypes.c_void_p(q.data_ptr()), ctypes.c_void_p(w.data_ptr()),
                                          ctypes.c_void_p(K.data_ptr()), 1, N, 64, 128, N - 1, 4,
                                          ctypes.c_void_p(idx.data_ptr()), ctypes.c_void_p(val.data_ptr()), None)
    assert rc == -3  # DSA_ERR_WORKSPACE
