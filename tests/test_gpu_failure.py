"""The bounded waits' failure path, exercised on the GPU without a fault.

Every wait of the tensor-core kernel has a poll budget.  Here a wait is made
to run out on purpose: the first CTA of a dense launch never loads its first
key tile (dsa_debug_set_wait), so the MMA issuer's wait for that tile gives
up after a short budget.  The launch must record DSA_ERR_TIMEOUT in the
status word, let the copies it already issued land, free its tensor memory
and return; the same device and workspace must then serve a normal call
whose results match the oracle (ADIndex — Deployment Guidance: a fallback
path is only trusted once it is exercised)."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_rows
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"
DSA_ERR_TIMEOUT = -5


def _oracle_check(inp, idx, val, k, what):
    r = O.dense(inp.q.double().cpu().numpy(), inp.w.double().cpu().numpy(), inp.k.double().cpu().numpy(), k,
                q_pos0=inp.q_pos0, return_scores=True)
    check_rows(idx.cpu().numpy(), val.cpu().numpy(), r["scores"], k, what=what)


def test_wait_runs_out_then_device_serves_a_normal_call():
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=64, N=4096, seed=61)
    k = 64
    ws = torch.zeros(dsa.dense_workspace_bytes(64, 4096, 64, 128, k, 0, 0), dtype=torch.uint8, device=DEV)
    dsa.dsa_debug_set_wait(1000, hold_first_tile=True)   # a millisecond
    try:
        dsa.dsa_index_dense(inp.q, inp.w, inp.k, k, q_pos0=inp.q_pos0, workspace=ws)
        with pytest.raises(dsa.DsaError) as e:
            dsa.dsa_check_status(ws)
        assert e.value.status == DSA_ERR_TIMEOUT
    finally:
        dsa.dsa_debug_set_wait(0, hold_first_tile=False)
    torch.cuda.synchronize()
    # the status read cleared the word; the same workspace serves a normal call
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, k, q_pos0=inp.q_pos0, workspace=ws, check=True)
    _oracle_check(inp, idx, val, k, "after a timed-out launch")


def test_short_budget_alone_keeps_results():
    # a budget of 20 ms is far above any wait of a working launch
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=130, N=2000, seed=62)
    dsa.dsa_debug_set_wait(20000)
    try:
        idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 100, q_pos0=inp.q_pos0, check=True)
    finally:
        dsa.dsa_debug_set_wait(0)
    _oracle_check(inp, idx, val, 100, "short wait budget")
    assert np.all(idx.cpu().numpy()[:, 0] >= 0)
