"""The library's scoring-kernel timer: it counts and times exactly the
scoring-kernel launches made while armed, up to the armed number."""
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu


def test_timer_counts_scoring_launches():
    inp = make_dense_inputs("dense_bf16_32k", device="cuda", T=512, N=1024, seed=5)
    ws = torch.zeros(dsa.dense_workspace_bytes(512, 1024, 64, 128, 64, 0, 0), dtype=torch.uint8, device="cuda")

    def run():
        dsa.dsa_index_dense(inp.q, inp.w, inp.k, 64, q_pos0=inp.q_pos0, workspace=ws)

    run()
    dsa.dsa_kernel_timer_start(4)
    for _ in range(3):
        run()
    ms, n = dsa.dsa_kernel_timer_stop()
    assert n == 3 and ms > 0.0
    # launches past the armed number are not timed
    dsa.dsa_kernel_timer_start(1)
    run()
    run()
    ms1, n1 = dsa.dsa_kernel_timer_stop()
    assert n1 == 1 and 0.0 < ms1
    # a second start while armed is refused; the timer still stops cleanly
    dsa.dsa_kernel_timer_start(2)
    with pytest.raises(dsa.DsaError):
        dsa.dsa_kernel_timer_start(2)
    _, n2 = dsa.dsa_kernel_timer_stop()
    assert n2 == 0
    dsa.dsa_check_status(ws)


def test_timer_group_and_decode_launch_counts():
    # Refine launches the scoring kernel twice (proxy scan, bank re-scoring),
    # Reuse once; decode once (the merge kernel is not timed)
    inp = make_dense_inputs("group_bf16_128k", device="cuda", T=256, N=512, seed=6)
    for mode, want in ((0, 2), (1, 1)):
        dsa.dsa_kernel_timer_start(8)
        dsa.dsa_index_group(inp.q, inp.w, inp.k, 32, 64, 128, mode=mode, q_pos0=inp.q_pos0, check=True)
        _, n = dsa.dsa_kernel_timer_stop()
        assert n == want, (mode, n)
    from synthetic import make_decode_inputs
    d = make_decode_inputs("decode_bf16_32x128k", device="cuda", lengths=[300, 700], m=2, seed=7)
    dsa.dsa_kernel_timer_start(8)
    dsa.dsa_index_decode(d.q, d.w, d.k, 32, d.k_offsets, d.q_offsets, check=True)
    _, n = dsa.dsa_kernel_timer_stop()
    assert n == 1
