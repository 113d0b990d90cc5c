"""Empty calls (no query rows): every entry point accepts them, launches
nothing and returns rows of shape [0, k]; the oracle's answer for the same
empty input is also empty."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O

pytestmark = pytest.mark.gpu
DEV = "cuda"
H, D = 64, 128


def _keys(N, dtype=torch.bfloat16):
    g = torch.Generator(device="cpu").manual_seed(7)
    return (torch.randn(N, D, generator=g) / D ** 0.5).to(dtype).to(DEV)


def _empty_q(dtype=torch.bfloat16, h=H, d=D):
    return torch.empty((0, h, d), dtype=dtype, device=DEV), torch.empty((0, h), dtype=torch.float32, device=DEV)


def test_dense_empty():
    K = _keys(300)
    q, w = _empty_q()
    idx, val = dsa.dsa_index_dense(q, w, K, 16, q_pos0=300, check=True)
    ref = O.dense(np.zeros((0, H, D)), np.zeros((0, H)), K.cpu().double().numpy(), 16, q_pos0=300)
    assert idx.shape == val.shape == ref["idx"].shape == (0, 16)
    # the exact fp32 kernel's shape
    q32, w32 = _empty_q(torch.float32, 4, 64)
    idx, _ = dsa.dsa_index_dense(q32, w32, torch.zeros((10, 64), device=DEV), 4, q_pos0=10, check=True)
    assert idx.shape == (0, 4)
    # no keys either
    idx, _ = dsa.dsa_index_dense(q, w, torch.empty((0, D), dtype=torch.bfloat16, device=DEV), 8, q_pos0=0)
    assert idx.shape == (0, 8)
    idx, _ = dsa.dsa_index_dense_static(q, w, K, 16, q_pos0=300)
    assert idx.shape == (0, 16)


@pytest.mark.parametrize("mode", [0, 1, 2])
def test_group_empty(mode):
    K = _keys(300)
    q, w = _empty_q()
    idx, val = dsa.dsa_index_group(q, w, K, 16, 8, 64, mode=mode, q_pos0=300, check=True)
    assert idx.shape == (0, 16)
    ref = O.group(np.zeros((0, H, D)), np.zeros((0, H)), K.cpu().double().numpy(), 16, 8, 64, mode, q_pos0=300,
                  q_dtype="bf16")
    assert len(ref["idx"]) == 0 and len(ref["bank_idx"]) == 0


def test_decode_empty():
    q, w = _empty_q()
    K = torch.empty((0, D), dtype=torch.bfloat16, device=DEV)
    ko = torch.zeros(1, dtype=torch.int64)
    qo = torch.zeros(1, dtype=torch.int32)
    idx, _ = dsa.dsa_index_decode(q, w, K, 32, ko, qo, check=True)
    assert idx.shape == (0, 32)
    idx, _ = dsa.dsa_index_decode_group(q, w, K, 32, ko, qo, 64, check=True)
    assert idx.shape == (0, 32)
    ref = O.decode(np.zeros((0, H, D)), np.zeros((0, H)), np.zeros((0, D)), np.array([0]), np.array([0]), 32)
    assert ref["idx"].shape == (0, 32)


def test_routed_empty():
    K = _keys(1024)
    q, w = _empty_q()
    idx, _ = dsa.dsa_index_block_routed(q, w, K, 16, 2, q_pos0=1024, check=True)
    assert idx.shape == (0, 16)
    index = dsa.dsa_ivf_build(K, 8, iters=2, check=True)
    idx, _ = dsa.dsa_index_ivf_routed(q, w, index, 16, 2, q_pos0=1024, check=True)
    assert idx.shape == (0, 16)


def test_host_entries_empty():
    K = _keys(300).cpu()
    q = torch.empty((0, H, D), dtype=torch.bfloat16)
    w = torch.empty((0, H), dtype=torch.float32)
    idx, _ = dsa.dsa_index_dense_host(q, w, K, 16, q_pos0=300)
    assert idx.shape == (0, 16) and not idx.is_cuda
    idx, _ = dsa.dsa_index_group_host(q, w, K, 16, 8, 64, q_pos0=300)
    assert idx.shape == (0, 16)
    idx, _ = dsa.dsa_index_decode_host(q, w, torch.empty((0, D), dtype=torch.bfloat16), 16,
                                       torch.zeros(1, dtype=torch.int64), torch.zeros(1, dtype=torch.int32))
    assert idx.shape == (0, 16)
    assert dsa.dense_host_staging_bytes(0, 300, H, D, 16, 0, 0) == 256


def test_empty_checks_shape_arguments():
    # an empty call still rejects bad shape arguments
    q, w = _empty_q()
    with pytest.raises(dsa.DsaError):
        dsa.dsa_index_dense(q, w, _keys(10), 0, q_pos0=10)          # k < 1
    with pytest.raises(dsa.DsaError):
        dsa.dsa_index_dense(q, w, _keys(10), 4, q_pos0=11)          # q_pos0 beyond the keys
    with pytest.raises(dsa.DsaError):
        dsa.dsa_index_group(q, w, _keys(10), 16, 8, 8, q_pos0=10)   # bank < k
