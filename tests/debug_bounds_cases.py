"""Calls run by test_gpu_debug_bounds.py in a child process whose DSA_LIB is
the bounds-checking debug build of the library: every entry point on shapes
that reach the kernels' edges (ragged tiles, k above the prefix, the largest
k, partial groups, mixed decode lengths, fp8 keys, both kernels).  Every
call is checked through the status word (a failed bounds check reads as an
invalid internal state) and a few rows against the CPU oracle."""
import os
import sys

import numpy as np
import torch

HERE = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, os.path.dirname(HERE))
sys.path.insert(0, HERE)

import sparse_attention_token_index_b200 as dsa  # noqa: E402
from oracle import dsa_oracle as O  # noqa: E402
from parity import check_row  # noqa: E402
from synthetic import make_dense_inputs, make_decode_inputs  # noqa: E402

DEV = "cuda"


def f64(x):
    return x.detach().to("cpu").to(torch.float64).numpy()


def dense_rows(inp, idx, val, k, rows, what):
    K = O.key_values(inp.k.cpu().numpy(), inp.k_scale.cpu().numpy()) if inp.k_scale is not None else f64(inp.k)
    for t in rows:
        p = inp.q_pos0 + t
        S = O.score_rows(f64(inp.q[t:t + 1]), f64(inp.w[t:t + 1]), K[:p + 1])[0]
        check_row(idx[t].cpu().numpy(), val[t].cpu().numpy(), S, k, what=f"{what} t={t}")


def main():
    assert os.path.basename(dsa.lib_path) == "libdsa_index_debug.so", dsa.lib_path
    for k in (1, 100, 1000, 2048):
        inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=700, N=700, seed=5)
        idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, k, q_pos0=inp.q_pos0, check=True)
        dense_rows(inp, idx, val, k, [0, 1, 350, 698, 699], f"dense k={k}")
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=6, N=70000, seed=71)
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 65536, q_pos0=inp.q_pos0, check=True)
    dense_rows(inp, idx, val, 65536, [0, 5], "max k")
    inp = make_dense_inputs("fp8_256k", device=DEV, T=300, N=900)
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 128, q_pos0=inp.q_pos0, K_scale=inp.k_scale, check=True)
    dense_rows(inp, idx, val, 128, [0, 299], "fp8 dense")
    inp = make_dense_inputs("tiny_fp32_2k", device=DEV, T=200, N=333)
    idx, val = dsa.dsa_index_dense(inp.q, inp.w, inp.k, 64, q_pos0=inp.q_pos0, check=True)
    dense_rows(inp, idx, val, 64, [0, 199], "fp32 kernel")
    for mode in (0, 1, 2):
        for (T, N, G, B, k) in ((100, 700, 6, 48, 16), (640, 640, 64, 256, 64)):
            inp = make_dense_inputs("group_bf16_128k", device=DEV, T=T, N=N, seed=22)
            dsa.dsa_index_group(inp.q, inp.w, inp.k, k, G, B, mode=mode, q_pos0=inp.q_pos0, return_bank=True,
                                check=True)
    d = make_decode_inputs(device=DEV, lengths=[300, 17, 1000, 129, 4096, 1], m=[2, 1, 3, 4, 2, 1], seed=31)
    idx, val = dsa.dsa_index_decode(d.q, d.w, d.k, 128, d.k_offsets, d.q_offsets, check=True)
    d = make_decode_inputs(device=DEV, lengths=[50, 200, 7], m=[1, 2, 3], seed=32)
    dsa.dsa_index_decode(d.q, d.w, d.k, 300, d.k_offsets, d.q_offsets, check=True)
    d = make_decode_inputs(device=DEV, lengths=[700, 1500, 300], m=[2, 3, 1], seed=82)
    for mode in (0, 1, 2):
        dsa.dsa_index_decode_group(d.q, d.w, d.k, 32, d.k_offsets, d.q_offsets, 128, mode=mode, check=True)
    inp = make_dense_inputs("group_bf16_128k", device=DEV, T=500, N=1500, seed=83)
    dsa.dsa_index_block_routed(inp.q, inp.w, inp.k, 48, 3, q_pos0=inp.q_pos0, check=True)
    index = dsa.dsa_ivf_build(inp.k, 16, iters=3, check=True)
    dsa.dsa_index_ivf_routed(inp.q, inp.w, index, 48, 4, q_pos0=inp.q_pos0, check=True)
    inp = make_dense_inputs("dense_bf16_32k", device=DEV, T=260, N=700, seed=52)
    dsa.dsa_index_dense_static(inp.q, inp.w, inp.k, 64, q_pos0=inp.q_pos0)
    torch.cuda.synchronize()
    print("debug-bounds cases ok")


if __name__ == "__main__":
    main()
