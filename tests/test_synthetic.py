"""Seeded input generators (no GPU): shapes, determinism, recipe properties."""
import numpy as np
import torch

from oracle import dsa_oracle as O
from synthetic import make_dense_inputs, make_decode_inputs, encode_e4m3


def test_dense_shapes_and_determinism():
    a = make_dense_inputs("dense_bf16_32k", T=300, N=500, seed=11)
    b = make_dense_inputs("dense_bf16_32k", T=300, N=500, seed=11)
    assert a.q.shape == (300, 64, 128) and a.q.dtype == torch.bfloat16
    assert a.k.shape == (500, 128) and a.w.shape == (300, 64) and a.w.dtype == torch.float32
    assert a.q_pos0 == 200
    assert torch.equal(a.q, b.q) and torch.equal(a.k, b.k) and torch.equal(a.w, b.w)
    c = make_dense_inputs("dense_bf16_32k", T=300, N=500, seed=12)
    assert not torch.equal(a.k, c.k)


def test_tiny_recipe():
    x = make_dense_inputs("tiny_fp32_2k", T=512, N=512)
    assert x.q.dtype == torch.float32 and x.q.shape == (512, 4, 64)
    assert float(x.w.min()) >= 0 and float(x.w.max()) <= 1


def test_lowrank_neighbour_overlap():
    # neighbouring queries share most of their top-k (the recipe's purpose)
    x = make_dense_inputs("dense_bf16_32k", T=64, N=2048, H=16, seed=3)
    r = O.dense(x.q.float().numpy(), x.w.numpy(), x.k.float().numpy(), 128, q_pos0=x.q_pos0)
    ov = [len(set(r["idx"][t]) & set(r["idx"][t + 1])) / 128 for t in range(63)]
    # rows of an unrelated draw share about k/N = 6% by chance
    y = make_dense_inputs("dense_bf16_32k", T=64, N=2048, H=16, seed=4)
    r2 = O.dense(y.q.float().numpy(), y.w.numpy(), x.k.float().numpy(), 128, q_pos0=x.q_pos0)
    chance = [len(set(r["idx"][t]) & set(r2["idx"][t])) / 128 for t in range(64)]
    assert np.mean(ov) > 0.3 and np.mean(ov) > 2 * np.mean(chance)


def test_fp8_roundtrip():
    g = torch.Generator().manual_seed(0)
    x = torch.randn(256, 128, generator=g) * 0.1
    b, s = encode_e4m3(x)
    assert b.dtype == torch.uint8 and (s > 0).all()
    dec = O.decode_e4m3(b.numpy()) * s.numpy()[:, None].astype(np.float64)
    err = np.abs(dec - x.numpy())
    # e4m3 keeps 3 mantissa bits: relative error <= 2^-4 for normal values;
    # values under the smallest normal (2^-6 * scale) are off by <= half a subnormal step
    tol = np.maximum(2.0 ** -4 * np.abs(x.numpy()), 2.0 ** -10 * s.numpy()[:, None])
    assert (err <= tol + 1e-12).all()


def test_fp8_mixture_recipe():
    x = make_dense_inputs("fp8_256k", T=128, N=1024)
    assert x.k.dtype == torch.uint8 and x.k_scale.shape == (1024,)
    assert x.q.dtype == torch.bfloat16


def test_decode_recipe():
    x = make_decode_inputs(lengths=[300, 17, 1000], m=[2, 1, 3], H=8, d=64)
    assert x.k.shape == (1317, 64) and x.q.shape == (6, 8, 64)
    assert x.k_offsets.tolist() == [0, 300, 317, 1317]
    assert x.q_offsets.tolist() == [0, 2, 3, 6]


def test_needle_positions_reported():
    # the recipes report where they planted keys (data for choosing parity rows)
    x = make_dense_inputs("fp8_256k", T=512, N=4000)
    n = x.needles.numpy()
    assert n.shape == (20,) and np.all(np.diff(n) > 0) and n[0] >= 0 and n[-1] < 4000
    y = make_decode_inputs(lengths=[300, 17, 1000], m=[2, 1, 3], H=8, d=64)
    ny = y.needles.numpy()
    assert ny.shape == (3 + 1 + 10,)
    assert np.all((ny[:3] < 300)) and ny[3] in range(300, 317) and np.all((ny[4:] >= 317) & (ny[4:] < 1317))
    z = make_dense_inputs("tiny_fp32_2k", T=512, N=512)
    assert z.needles.shape == (32,)                     # 16 keys per 256-position block
    assert make_dense_inputs("dense_bf16_32k", T=64, N=256).needles is None
    # the planted decode keys lean along the sequence's query direction
    u = y.q[:2].float().sum(dim=(0, 1))
    proj = (y.k[:300].float() @ (u / u.norm())).numpy()
    assert proj[ny[:3]].min() > np.median(proj)
