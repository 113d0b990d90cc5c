"""Dense prefill indexer: CUDA path (through the C ABI) against the CPU oracle."""
import numpy as np
import pytest
import torch

import sparse_attention_token_index_b200 as dsa
from oracle import dsa_oracle as O
from parity import check_rows, check_scores, sample_rows
from synthetic import make_dense_inputs

pytestmark = pytest.mark.gpu
DEV = "cuda"


def _f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def _keys(inp):
    if inp.k_dtype == "fp8":
        return inp.k.cpu().numpy(), inp.k_scale.cpu().numpy()
    return _f64(inp.k), None


def _run_and_check(inp, k, rows=None, what=""):
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, k, q_pos0=inp.q_pos0, K_scale=inp.k_scale, check=True)
    K, ks = _keys(inp)
    T = inp.q.shape[0]
    rows = np.arange(T) if rows is None else np.asarray(rows)
    q = _f64(inp.q[torch.as_tensor(rows, device=inp.q.device)])
    w = _f64(inp.w[torch.as_tensor(rows, device=inp.w.device)])
    # oracle on the sampled rows: re-index so row j of q is original row rows[j]
    res = [O.dense(q[j:j + 1], w[j:j + 1], K, k, q_pos0=inp.q_pos0 + int(r), k_scale=ks, return_scores=True)
           for j, r in enumerate(rows)]
    scores = [r["scores"][0] for r in res]
    gi = idx.cpu().numpy()[rows]
    gv = val.cpu().numpy()[rows]
    check_rows(gi, gv, scores, k, what=what)
    return idx, val


def test_tiny_fp32_full():
    # fp32 throughout (exact CUDA-core path), every row of the 2048 x 2048 problem
    inp = make_dense_inputs("tiny_fp32_2k", device=DEV)
    _run_and_check(inp, 64, what="tiny fp32")


@pytest.mark.parametrize("k", [1, 100, 1000])
def test_bf16_tensor_core_ragged(k):
    # 700 keys = 5 full tiles of 128 + a ragged tail of 60; 175 query units
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=700, N=700, seed=5)
    _run_and_check(inp, k, what=f"bf16 tc k={k}")


def test_bf16_tensor_core_offset_queries():
    # queries at the end of a longer prefix (q_pos0 > 0), T not a multiple of 4
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=130, N=900, seed=6)
    assert inp.q_pos0 == 770
    _run_and_check(inp, 300, what="bf16 tc offset")


def test_bf16_k_exceeds_prefix():
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=300, N=300, seed=7)
    idx, val = _run_and_check(inp, 2048, what="k > N")
    cnt = (idx >= 0).sum(dim=1).cpu().numpy()
    assert np.array_equal(cnt, np.arange(1, 301))


def test_single_query_single_key():
    g = torch.Generator(device=DEV).manual_seed(0)
    q = torch.randn(1, 64, 128, generator=g, device=DEV).to(torch.bfloat16)
    w = torch.rand(1, 64, generator=g, device=DEV)
    K = torch.randn(1, 128, generator=g, device=DEV).to(torch.bfloat16)
    idx, val = dsa.dsa_index_dense(q, w, K, 4, check=True)
    assert idx.cpu().tolist() == [[0, -1, -1, -1]]
    S = O.score_rows(_f64(q), _f64(w), _f64(K))[0, 0]
    assert abs(val[0, 0].item() - S) <= 1e-3 * abs(S) + 1e-6


def _exact_inputs(T, N, H, d, seed):
    # small integers in q and k and dyadic weights: every product and sum is
    # exact in fp32, so GPU scores equal the oracle's and selection (ties
    # included) must match bit for bit
    g = torch.Generator(device=DEV).manual_seed(seed)
    q = torch.randint(-2, 3, (T, H, d), generator=g, device=DEV).to(torch.bfloat16)
    base = torch.randint(-2, 3, (37, d), generator=g, device=DEV)
    K = base[torch.randint(0, 37, (N,), generator=g, device=DEV)].to(torch.bfloat16)  # many duplicate keys
    w = torch.randint(0, 3, (T, H), generator=g, device=DEV).float() * 0.5
    return q, w, K


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_exact_scores_ties_bit_exact(path):
    H, d = (64, 128) if path == "tc" else (8, 32)
    T, N, k = 200, 600, 50
    q, w, K = _exact_inputs(T, N, H, d, 11)
    if path == "simt":
        q, K = q.float(), K.float()
    idx, val = dsa.dsa_index_dense(q, w, K, k, check=True)
    r = O.dense(_f64(q), _f64(w), _f64(K), k, q_pos0=N - T)
    gi, gv = idx.cpu().numpy(), val.cpu().numpy()
    for t in range(T):
        order = np.argsort(gi[t])
        ro = np.argsort(r["idx"][t])
        assert np.array_equal(gi[t][order], r["idx"][t][ro]), f"row {t}"
        assert np.array_equal(gv[t][order].astype(np.float64), r["val"][t][ro]), f"row {t}"


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_debug_scores_match_oracle(path):
    if path == "tc":
        inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=260, N=260, seed=8)
    else:
        inp = make_dense_inputs("tiny_fp32_2k", device=DEV, T=200, N=333)
    S = dsa.dsa_debug_scores(inp.q, inp.w, inp.k, q_pos0=inp.q_pos0, check=True)
    K, ks = _keys(inp)
    ref = O.score_rows(_f64(inp.q), _f64(inp.w), O.key_values(K, ks))
    T, N = ref.shape
    pos = inp.q_pos0 + np.arange(T)
    ref = np.where(np.arange(N)[None, :] <= pos[:, None], ref, -np.inf)
    check_scores(S.cpu().numpy(), ref, what=path)


def test_bf16_other_shape_cuda_core():
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=150, N=400, H=8, d=64, seed=9)
    _run_and_check(inp, 64, what="bf16 H=8 d=64")


def test_fp8_keys_cuda_core_small():
    inp = make_dense_inputs("fp8_256k", device=DEV, T=120, N=500, H=16, d=64)
    _run_and_check(inp, 80, what="fp8 keys")


def test_dense_full_size_sampled():
    # the 32K x 32K bf16 workload at full size, k = 2048, in the benchmark's
    # launch configuration: 512 seeded rows (first and last units, rows that
    # see fewer than k keys, tile edges, uniform rows)
    inp = make_dense_inputs("dense_bf16_32k", device=DEV)
    T = inp.q.shape[0]
    rows = sample_rows(T, 2048, n=512, seed=1, q_pos0=inp.q_pos0, needles=inp.needles)
    assert len(rows) == 512 and rows[0] == 0 and rows[-1] == T - 1 and (rows < 2048).sum() >= 16
    _run_and_check(inp, 2048, rows=rows, what="dense 32K")


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_all_keys_identical(path):
    # every score of a row is equal: the selection must be the k lowest key
    # indices (more ties than the staging buffer holds)
    T, N, k = 8, 3000, 100
    H, d = (64, 128) if path == "tc" else (4, 16)
    g = torch.Generator(device=DEV).manual_seed(41)
    q = torch.randn(T, H, d, generator=g, device=DEV)
    K = torch.randn(1, d, generator=g, device=DEV).expand(N, d).contiguous()
    w = torch.rand(T, H, generator=g, device=DEV)
    if path == "tc":
        q, K = q.to(torch.bfloat16), K.to(torch.bfloat16)
    idx, val = dsa.dsa_index_dense(q, w, K, k, check=True)
    for t in range(T):
        assert sorted(idx[t].tolist()) == list(range(k)), t
        assert len(set(val[t].tolist())) == 1


def test_fp8_keys_tensor_core():
    # e4m3 keys with a per-key scale at H = 64, d = 128: keys widened exactly
    # to bf16, the scale applied to the score
    inp = make_dense_inputs("fp8_256k", device=DEV, T=400, N=900)
    assert inp.k.dtype == torch.uint8
    _run_and_check(inp, 128, what="fp8 tc")


def test_fp8_debug_scores_tensor_core():
    inp = make_dense_inputs("fp8_256k", device=DEV, T=200, N=300)
    S = dsa.dsa_debug_scores(inp.q, inp.w, inp.k, q_pos0=inp.q_pos0, K_scale=inp.k_scale, check=True)
    K, ks = _keys(inp)
    ref = O.score_rows(_f64(inp.q), _f64(inp.w), O.key_values(K, ks))
    pos = inp.q_pos0 + np.arange(200)
    ref = np.where(np.arange(300)[None, :] <= pos[:, None], ref, -np.inf)
    check_scores(S.cpu().numpy(), ref, what="fp8 tc")


@pytest.mark.parametrize("path", ["tc", "simt"])
def test_maximum_k(path):
    # k at its maximum (65536) over a prefix a little longer: the threshold bin
    # holds thousands of entries, so the select's sub-bin and radix paths run
    N, T, k = 70000, 6, 65536
    if path == "tc":
        inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=T, N=N, seed=71)
    else:
        inp = make_dense_inputs("tiny_fp32_2k", device=DEV, T=T, N=N, seed=71)
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, k, q_pos0=inp.q_pos0, check=True)
    q, w, K = _f64(inp.q), _f64(inp.w), _f64(inp.k)
    S = O.score_rows(q, w, K)
    rows = list(range(T))
    check_rows(idx.cpu().numpy(), val.cpu().numpy(), [S[t, :inp.q_pos0 + t + 1] for t in rows], k,
               what=f"max k {path}")
