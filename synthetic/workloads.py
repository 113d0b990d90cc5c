"""Seeded synthetic workloads shaped like the long-context indexer benchmarks.

The pages evaluate on long-context suites with real models; neither is
available here, so these generators stand in for their *shape*: long causal
prefixes, k = 2048, long-tailed score rows (planted high-score keys) and
neighbouring queries whose top-k overlap (a shared low-rank latent that
drifts slowly with position).  The PIVOT abstract observes both properties
(neighbouring queries pick largely the same keys; along the keys, indexer
scores have a long tail), and the AttentionIndex worked example scatters
similar keys over positions, which the fp8 recipe's key clusters follow.

Every draw comes from ``torch.Generator(device).manual_seed(seed)``; the same
call on the same device type always returns the same tensors.  Nothing here
scores keys or selects them.
"""
from __future__ import annotations

import math
from dataclasses import dataclass
from typing import Optional

import torch

# Workload recipes.  Sizes are those of the benchmark configurations; the
# ``make_*`` functions accept smaller sizes with the same recipe for tests.
CONFIGS = {
    # Tiny dense prefill, fp32 throughout.
    "tiny_fp32_2k": dict(kind="planted", T=2048, N=2048, H=4, d=64, k=64,
                         q_dtype="fp32", k_dtype="fp32", seed=0),
    # Dense prefill, bf16 q/k, fp32 w.
    "dense_bf16_32k": dict(kind="lowrank", T=32768, N=32768, H=64, d=128, k=2048,
                           q_dtype="bf16", k_dtype="bf16", seed=1),
    # Decode: 32 sequences x 131072 cached keys, 2 new queries each.
    "decode_bf16_32x128k": dict(kind="decode", B=32, Nb=131072, m=2, H=64, d=128,
                                k=2048, q_dtype="bf16", k_dtype="bf16", seed=2),
    # Group-shared prefill at 128K (Refine and Reuse).
    "group_bf16_128k": dict(kind="lowrank", T=131072, N=131072, H=64, d=128, k=2048,
                            G=64, bank=8192, q_dtype="bf16", k_dtype="bf16", seed=3),
    # Long-context prefill with fp8 e4m3 keys + per-token fp32 scale.
    "fp8_256k": dict(kind="mixture", T=262144, N=262144, H=64, d=128, k=2048,
                     G=64, bank=8192, q_dtype="bf16", k_dtype="fp8", seed=4),
}

_TORCH_DTYPE = {"fp32": torch.float32, "bf16": torch.bfloat16}

E4M3_MAX = 448.0


@dataclass
class DenseInputs:
    q: torch.Tensor            # [T, H, d] fp32 or bf16
    w: torch.Tensor            # [T, H] fp32
    k: torch.Tensor            # [N, d] fp32 / bf16, or uint8 e4m3 bytes
    k_scale: Optional[torch.Tensor]  # [N] fp32 (fp8 keys only)
    q_pos0: int                # query row t sits at key position q_pos0 + t
    q_dtype: str
    k_dtype: str
    needles: Optional[torch.Tensor] = None  # [n] int64 (host): positions of planted keys, ascending


@dataclass
class DecodeInputs:
    q: torch.Tensor            # [sum m_b, H, d]
    w: torch.Tensor            # [sum m_b, H] fp32
    k: torch.Tensor            # [sum N_b, d]
    k_scale: Optional[torch.Tensor]
    k_offsets: torch.Tensor    # [B+1] int64 (host)
    q_offsets: torch.Tensor    # [B+1] int32 (host)
    q_dtype: str
    k_dtype: str
    needles: Optional[torch.Tensor] = None  # [n] int64 (host): planted key rows of K, ascending


def _gen(device, seed: int) -> torch.Generator:
    g = torch.Generator(device=device)
    g.manual_seed(int(seed))
    return g


def _randn(g, shape, device):
    return torch.randn(shape, generator=g, device=device, dtype=torch.float32)


def _unit(v: torch.Tensor) -> torch.Tensor:
    return v / v.norm()


def encode_e4m3(x: torch.Tensor):
    """Per-row fp8 e4m3 encoding of keys: scale = amax(|row|)/448, bytes = RNE(row/scale).

    Returns (uint8 bytes [N, d], fp32 scale [N]); scale > 0 for every row.
    Input preparation only: the indexer reads the stored bytes and scales.
    """
    amax = x.abs().amax(dim=1).clamp_min(1e-30)
    scale = (amax / E4M3_MAX).to(torch.float32)
    y = (x / scale[:, None]).clamp(-E4M3_MAX, E4M3_MAX)
    b = y.to(torch.float8_e4m3fn).view(torch.uint8)
    assert bool((scale > 0).all())
    return b.contiguous(), scale.contiguous()


def _ar1_latent(g, L: int, r: int, rho: float, device) -> torch.Tensor:
    """Stationary AR(1) latent over positions: c[t] = rho c[t-1] + sqrt(1-rho^2) e[t]."""
    blk = 256
    nb = (L + blk - 1) // blk
    eps = _randn(g, (nb * blk, r), device) * math.sqrt(1.0 - rho * rho)
    i = torch.arange(blk, device=device, dtype=torch.float32)
    expo = (i[:, None] - i[None, :])
    P = torch.where(expo >= 0, torch.pow(torch.tensor(rho, device=device), expo.clamp_min(0)),
                    torch.zeros((), device=device))
    decay = torch.pow(torch.tensor(rho, device=device), i + 1.0)  # rho^(i+1)
    within = torch.matmul(P, eps.view(nb, blk, r))                # [nb, blk, r]
    out = torch.empty(nb, blk, r, device=device, dtype=torch.float32)
    prev = _randn(g, (r,), device)                                 # c[-1] ~ N(0, 1)
    for b in range(nb):
        out[b] = within[b] + decay[:, None] * prev[None, :]
        prev = out[b, -1]
    return out.view(nb * blk, r)[:L].contiguous()


def _cast(x: torch.Tensor, dtype: str) -> torch.Tensor:
    return x.to(_TORCH_DTYPE[dtype]).contiguous()


def _lowrank_queries(g, T, H, d, lat, q_pos0, q_dtype, device, chunk=4096):
    r = lat.shape[1]
    Bq = _randn(g, (H, d, r), device) / math.sqrt(r)
    out = torch.empty((T, H, d), dtype=_TORCH_DTYPE[q_dtype], device=device)
    # per-row noise carries 1/5 of a query's variance, the slowly drifting shared
    # latent 4/5, so that neighbouring queries rank keys alike
    a = 0.5
    s = 1.0 / math.sqrt((1.0 + a * a) * d)
    for t0 in range(0, T, chunk):
        t1 = min(T, t0 + chunk)
        z = _randn(g, (t1 - t0, H, d), device)
        c = lat[q_pos0 + t0:q_pos0 + t1]                          # [n, r]
        shared = torch.einsum("hdr,nr->nhd", Bq, c)
        out[t0:t1] = ((a * z + shared) * s).to(out.dtype)
    return out


def make_dense_inputs(cfg: str | dict, device="cpu", T: Optional[int] = None,
                      N: Optional[int] = None, H: Optional[int] = None,
                      d: Optional[int] = None, q_pos0: Optional[int] = None,
                      seed: Optional[int] = None) -> DenseInputs:
    """Inputs for the prefill (dense / group) indexer following a named recipe.

    ``T``, ``N``, ``H``, ``d`` override the recipe's sizes (tests use small
    ones); by default queries occupy the last T positions: q_pos0 = N - T.
    """
    c = dict(CONFIGS[cfg]) if isinstance(cfg, str) else dict(cfg)
    T = c["T"] if T is None else T
    N = c["N"] if N is None else N
    H = c["H"] if H is None else H
    d = c["d"] if d is None else d
    seed = c["seed"] if seed is None else seed
    q_pos0 = N - T if q_pos0 is None else q_pos0
    assert 0 <= q_pos0 and q_pos0 + T <= N
    qd, kd = c["q_dtype"], c["k_dtype"]
    g = _gen(device, seed)
    kind = c["kind"]
    k_scale = None
    needles = None
    if kind == "planted":
        sig = 1.0 / math.sqrt(d)
        u = _unit(_randn(g, (d,), device))
        kf = _randn(g, (N, d), device) * sig
        qf = _randn(g, (T, H, d), device) * sig
        # 16 planted keys (and query rows) per 256-position block, +3 sigma along u.
        planted = []
        for arr, n in ((kf, N), (qf, T)):
            for b0 in range(0, n, 256):
                nb = min(256, n - b0)
                pick = torch.randperm(nb, generator=g, device=device)[:min(16, nb)] + b0
                if arr.dim() == 2:
                    arr[pick] += 3.0 * sig * u
                    planted.append(pick)
                else:
                    arr[pick] += 3.0 * sig * u[None, :]
        needles = torch.sort(torch.cat(planted)).values
        w = torch.rand((T, H), generator=g, device=device, dtype=torch.float32)
        q = _cast(qf, qd)
        k = _cast(kf, kd)
    elif kind == "lowrank":
        rho = math.exp(-1.0 / 64.0)
        lat = _ar1_latent(g, N, 8, rho, device)
        q = _lowrank_queries(g, T, H, d, lat, q_pos0, qd, device)
        Bk = _randn(g, (d, 8), device) / math.sqrt(8)
        kf = (_randn(g, (N, d), device) + lat @ Bk.T) / math.sqrt(2 * d)
        k = _cast(kf, kd)
        w = torch.rand((T, H), generator=g, device=device, dtype=torch.float32)
    elif kind == "mixture":
        rho = math.exp(-1.0 / 64.0)
        lat = _ar1_latent(g, N, 8, rho, device)
        q = _lowrank_queries(g, T, H, d, lat, q_pos0, qd, device)
        sig = 1.0 / math.sqrt(d)
        ncl = 64
        mu = _randn(g, (ncl, d), device) * sig * 2.0
        assign = torch.randint(0, ncl, (N,), generator=g, device=device)
        kf = mu[assign] + _randn(g, (N, d), device) * (0.5 * sig)
        nneedle = max(1, int(round(0.005 * N)))
        rows = torch.randint(0, T, (16,), generator=g, device=device)
        u = _unit(q[rows].float().sum(dim=(0, 1)))
        pos = torch.randperm(N, generator=g, device=device)[:nneedle]
        kf[pos] += 4.0 * sig * u
        needles = torch.sort(pos).values
        w = torch.rand((T, H), generator=g, device=device, dtype=torch.float32)
        if kd == "fp8":
            k, k_scale = encode_e4m3(kf)
        else:
            k = _cast(kf, kd)
    else:
        raise ValueError(f"not a prefill recipe: {kind}")
    return DenseInputs(q=q.contiguous(), w=w.contiguous(), k=k, k_scale=k_scale,
                       q_pos0=int(q_pos0), q_dtype=qd, k_dtype=kd,
                       needles=None if needles is None else needles.to("cpu", torch.int64))


def make_decode_inputs(cfg: str | dict = "decode_bf16_32x128k", device="cpu",
                       lengths=None, m=None, H=None, d=None, seed=None,
                       k_dtype: Optional[str] = None) -> DecodeInputs:
    """Decode batch: per sequence b a cache K_b[N_b, d] and m_b new queries.

    ``lengths`` (list of N_b) and ``m`` (int or list of m_b) override the
    recipe.  1% of each sequence's keys are planted +4 sigma along the
    normalised sum of that sequence's query heads, so they score high.
    """
    c = dict(CONFIGS[cfg]) if isinstance(cfg, str) else dict(cfg)
    H = c["H"] if H is None else H
    d = c["d"] if d is None else d
    seed = c["seed"] if seed is None else seed
    if lengths is None:
        lengths = [c["Nb"]] * c["B"]
    B = len(lengths)
    if m is None:
        m = c["m"]
    ms = [m] * B if isinstance(m, int) else list(m)
    assert len(ms) == B and all(1 <= mb <= nb for mb, nb in zip(ms, lengths))
    qd = c["q_dtype"]
    kd = c["k_dtype"] if k_dtype is None else k_dtype
    g = _gen(device, seed)
    sig = 1.0 / math.sqrt(d)
    Ntot, Mtot = int(sum(lengths)), int(sum(ms))
    qf = _randn(g, (Mtot, H, d), device) * sig
    kf = torch.empty((Ntot, d), device=device, dtype=torch.float32)
    ko, qo = 0, 0
    planted = []
    for nb, mb in zip(lengths, ms):
        kb = _randn(g, (nb, d), device) * sig
        u = _unit(qf[qo:qo + mb].sum(dim=(0, 1)))
        npl = max(1, int(round(0.01 * nb)))
        pos = torch.randperm(nb, generator=g, device=device)[:npl]
        kb[pos] += 4.0 * sig * u
        planted.append(torch.sort(pos).values + ko)
        kf[ko:ko + nb] = kb
        ko += nb
        qo += mb
    w = torch.rand((Mtot, H), generator=g, device=device, dtype=torch.float32)
    k_scale = None
    if kd == "fp8":
        k, k_scale = encode_e4m3(kf)
    else:
        k = _cast(kf, kd)
    k_off = torch.zeros(B + 1, dtype=torch.int64)
    k_off[1:] = torch.cumsum(torch.tensor(lengths, dtype=torch.int64), 0)
    q_off = torch.zeros(B + 1, dtype=torch.int32)
    q_off[1:] = torch.cumsum(torch.tensor(ms, dtype=torch.int64), 0).to(torch.int32)
    return DecodeInputs(q=_cast(qf, qd), w=w.contiguous(), k=k, k_scale=k_scale,
                        k_offsets=k_off, q_offsets=q_off, q_dtype=qd, k_dtype=kd,
                        needles=torch.cat(planted).to("cpu", torch.int64))
