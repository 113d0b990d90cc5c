"""Benchmark of the lightning indexer on B200.

    python bench.py [--gpus N] [--steps K] [--warmup W] [--config NAME] [--impl reference]

One step = one full indexer pass (scores + per-query top-k) over the
workload's synthetic inputs, already resident in HBM.  Default workload:
dense prefill, T = N = 32768 causal, H = 64, d = 128, k = 2048, bf16 q/k,
fp32 w.  Timing: W untimed steps, then K steps between barrier +
synchronize on both sides, CUDA events on the launching stream, max over
ranks.  Under torchrun each rank runs its own copy of the workload (the
path shards by independent query rows / sequences with no exchange step),
so per-GPU work is fixed as N grows.

Prints one JSON line (rank 0).  ``--impl reference`` times the CPU oracle
on a bounded sample of the same workload instead.
"""
from __future__ import annotations

import argparse
import json
import os
import statistics
import sys
import time

import numpy as np
import torch

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "indexer G score-pairs/s + top-k rows/s at 1 B200; % tensor/HBM roofline"


def _oracle_threads():
    """(threads the oracle computes on, host cores): numpy's BLAS pool (its
    matrix products; the sorts run on one thread) and the box's core count."""
    host = len(os.sched_getaffinity(0)) if hasattr(os, "sched_getaffinity") else (os.cpu_count() or 1)
    try:
        from threadpoolctl import threadpool_info
        blas = [i.get("num_threads", 1) for i in threadpool_info() if i.get("user_api") == "blas"]
        return (max(blas) if blas else 1), host
    except Exception:
        return host, host


def _dtype_label(cfg):
    """The arithmetic types the path computes in: bf16 q and k, or bf16 q with
    e4m3 keys (widened exactly to bf16 for the MMA, scale in fp32)."""
    q, k = cfg.get("q_dtype", "bf16"), cfg.get("k_dtype", "bf16")
    if q == k:
        return q
    return f"{q} q / {'e4m3' if k == 'fp8' else k} k"


def _parallelism(world):
    return (f"dp{world}: rank r indexes its own batch (seed + r), no collective on the data path"
            if world > 1 else "single GPU")


# A scoring kernel timed inside a timed region shorter than this ran as a
# burst (the measured burst cuBLAS figure applies); a longer region is
# sustained operation under the power cap.
SUSTAINED_AFTER_S = 2.0


def _peaks():
    p = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(p):
        with open(p) as f:
            j = json.load(f)
        return dict(hbm=float(j["hbm_gbs"]), bf16=float(j["bf16_tflops"]),
                    bf16_sus=float(j.get("bf16_tflops_sustained", j["bf16_tflops"])), src="measured")
    return dict(hbm=6650.0, bf16=1590.0, bf16_sus=1400.0, src="fallback")


# ---------------------------------------------------------------------------
# workloads
# ---------------------------------------------------------------------------
def _f64(t):
    return t.detach().to("cpu").to(torch.float64).numpy()


GROUP_OVERRIDE = None   # --group: group size of the group workloads
SHARD = 0               # this rank's batch of the workload: seed = the workload's seed + SHARD
BANK_OVERRIDE = None    # --bank: candidate bank of the group workloads
M_OVERRIDE = None       # --m: new queries per sequence of the decode workloads


def _row_recall(got_idx, ref_idx):
    """Per row |got ∩ ref| / |ref| (ignoring -1 padding), on the host."""
    g, r = got_idx.cpu().numpy(), ref_idx.cpu().numpy()
    out = np.empty(r.shape[0])
    for t in range(r.shape[0]):
        ref = r[t][r[t] >= 0]
        out[t] = np.intersect1d(g[t][g[t] >= 0], ref).size / max(1, ref.size)
    return out


class Workload:
    """One step = one full call of the indexer on resident inputs.

    pairs: score pairs the metric counts per step (group modes: the
    dense-equivalent causal pairs); alg_pairs: pairs actually scored;
    bound / alg_flops / alg_bytes: the roofline of the dominant kernel (the
    scoring kernel), summed over its launches in one step."""
    launches_per_step = 1
    kernel_launches_per_step = 1   # launches of the scoring kernel (the dominant one)
    bound = "tensor"
    alg_bytes = 0

    def e2e_buffers(self):
        dev = [torch.empty_like(t) for t in self.host_src]
        hout = [torch.empty(self.out[0].shape, dtype=torch.int32).pin_memory(),
                torch.empty(self.out[1].shape, dtype=torch.float32).pin_memory()]
        h2d = sum(t.numel() * t.element_size() for t in dev)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        return dev, hout, h2d, d2h

    def host_inputs(self):
        return [t.cpu().pin_memory() for t in self.host_src]

    def e2e_step(self, host, dev_bufs, host_out):
        for d_, h_ in zip(dev_bufs, host):
            d_.copy_(h_, non_blocking=True)
        self.call(*dev_bufs)
        host_out[0].copy_(self.out[0], non_blocking=True)
        host_out[1].copy_(self.out[1], non_blocking=True)

    e2e_note = ("pinned host inputs copied in (torch copies on the stream), the device entry point, idx/val "
                "copied out, every step")

    def _host_e2e_buffers(self, staging_bytes):
        """Buffers of the host-buffer entry point: a device staging buffer
        and page-locked outputs; the byte counts are the step's copies."""
        self.staging = torch.empty(staging_bytes, dtype=torch.uint8, device=self.out[0].device)
        hout = [torch.empty(self.out[0].shape, dtype=torch.int32).pin_memory(),
                torch.empty(self.out[1].shape, dtype=torch.float32).pin_memory()]
        h2d = sum(t.numel() * t.element_size() for t in self.host_src)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        return None, hout, h2d, d2h

    def step(self):
        self.call(*self.host_src)

    def check(self):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_check_status(self.ws)

    def _oracle_loop(self, budget_s, one):
        t0 = time.perf_counter()
        pairs = nrows = 0
        i = 0
        while time.perf_counter() - t0 < budget_s:
            pairs += one(i)
            nrows += 1
            i += 1
        return pairs, nrows, time.perf_counter() - t0


class Dense(Workload):
    name = "dense_bf16_32k"

    def __init__(self, device, size=None, name=None):
        from synthetic import CONFIGS, make_dense_inputs
        self.name = name or self.name
        self.cfg = dict(CONFIGS[self.name])
        if size:
            self.cfg["T"] = self.cfg["N"] = int(size)
        self.inp = make_dense_inputs(self.name, device=device, T=self.cfg["T"], N=self.cfg["N"],
                                     seed=self.cfg["seed"] + SHARD)
        self.T, self.N, self.k = self.cfg["T"], self.cfg["N"], self.cfg["k"]
        q0 = self.inp.q_pos0
        self.pairs = self.alg_pairs = self.T * q0 + self.T * (self.T + 1) // 2
        self.alg_flops = self.alg_pairs * 2 * self.cfg["H"] * self.cfg["d"]
        self.rows = self.T
        i = self.inp
        self.host_src = [i.q, i.w, i.k] + ([i.k_scale] if i.k_scale is not None else [])

    def describe(self):
        c = self.cfg
        kd = "fp8 e4m3 k + fp32 per-key scale" if c["k_dtype"] == "fp8" else "bf16 k"
        return {"workload": f"{self.name}: dense prefill T=N={c['T']} causal, H={c['H']}, d={c['d']}, "
                            f"k={c['k']}, bf16 q, {kd}, fp32 w, {c['kind']} recipe, seed {c['seed']}",
                "T": c["T"], "N": c["N"], "H": c["H"], "d": c["d"], "k": c["k"],
                "l2": f"inputs larger than L2 (Q is {c['T'] * c['H'] * c['d'] * 2 >> 20} MiB), no flush"}

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        T, H, d = i.q.shape
        kd = 2 if self.cfg["k_dtype"] == "fp8" else 0
        self.ws = torch.zeros(dsa.dense_workspace_bytes(T, self.N, H, d, self.k, 0, kd), dtype=torch.uint8,
                              device=i.q.device)
        self.out = (torch.empty((T, self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((T, self.k), dtype=torch.float32, device=i.q.device))
        self.launches_per_step = 2 if kd == 2 else 1

    def call(self, q, w, k, ks=None):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_dense(q, w, k, self.k, q_pos0=self.inp.q_pos0, K_scale=ks, out=self.out, workspace=self.ws)

    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        K = i.k.cpu().numpy() if self.cfg["k_dtype"] == "fp8" else _f64(i.k)
        ks = i.k_scale.cpu().numpy() if i.k_scale is not None else None
        rng = np.random.default_rng(seed)

        def one(_):
            t = int(rng.integers(0, self.T))
            O.dense(_f64(i.q[t:t + 1]), _f64(i.w[t:t + 1]), K, self.k, q_pos0=i.q_pos0 + t, k_scale=ks)
            return i.q_pos0 + t + 1
        return self._oracle_loop(budget_s, one)


    e2e_note = ("dsa_index_dense_host: page-locked host inputs and outputs, copy-in / indexer / copy-out "
                "pipelined in row chunks by the library, every step")

    def e2e_buffers(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        T, H, d = i.q.shape
        kd = dsa.DSA_DTYPE_FP8_E4M3 if i.k_scale is not None else dsa.DSA_DTYPE_BF16
        return self._host_e2e_buffers(dsa.dense_host_staging_bytes(T, self.N, H, d, self.k, dsa.DSA_DTYPE_BF16, kd))

    def e2e_step(self, host, dev_bufs, host_out):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_dense_host(host[0], host[1], host[2], self.k, q_pos0=self.inp.q_pos0,
                                 K_scale=host[3] if len(host) > 3 else None, out=host_out, staging=self.staging)


class BlockRouted(Dense):
    """Two-stage selection over 128-key blocks (comparator): route each query
    to its best n_blocks complete blocks by their mean key, refine on them."""
    n_blocks = 64   # an 8K-key candidate budget
    e2e_buffers = Workload.e2e_buffers
    e2e_step = Workload.e2e_step
    e2e_note = Workload.e2e_note

    def __init__(self, device, size=None, name="fp8_256k"):
        super().__init__(device, size, name=name)
        T, q0, nb = self.T, self.inp.q_pos0, self.n_blocks
        H, d = self.cfg["H"], self.cfg["d"]
        # routing scores each complete block before the query; the refine
        # scores the routed blocks plus the own partial block
        route = sum((q0 + t + 1) // 128 for t in range(0, T, 64)) * 64
        refine = sum(min(nb, (q0 + t + 1) // 128) * 128 + (q0 + t + 1) % 128 for t in range(0, T, 64)) * 64
        self.alg_pairs = route + refine
        self.alg_flops = self.alg_pairs * 2 * H * d
        kd = self.cfg["k_dtype"] == "fp8"
        # (fp8 widening,) block means, routing, refine; routing and refine
        # both run the scoring kernel
        self.launches_per_step = 4 if kd else 3
        self.kernel_launches_per_step = 2

    def describe(self):
        d = super().describe()
        d["workload"] = d["workload"].replace("dense prefill", f"block-routed prefill ({self.n_blocks} blocks of 128 "
                                                               f"keys routed by their mean, then refined)")
        d["n_blocks"] = self.n_blocks
        d["metric_pairs"] = "dense-equivalent causal pairs (alg_pairs = routing + refine)"
        return d

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        T, H, d = i.q.shape
        kd = 2 if self.cfg["k_dtype"] == "fp8" else 0
        self.ws = torch.zeros(dsa.block_routed_workspace_bytes(T, self.N, H, d, self.k, self.n_blocks, 0, kd),
                              dtype=torch.uint8, device=i.q.device)
        self.out = (torch.empty((T, self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((T, self.k), dtype=torch.float32, device=i.q.device))

    def call(self, q, w, k, ks=None):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_block_routed(q, w, k, self.k, self.n_blocks, q_pos0=self.inp.q_pos0, K_scale=ks, out=self.out,
                                   workspace=self.ws)

    def recall(self, blocks=4, rows=512):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        got = []
        for t0 in np.linspace(0, self.T - rows, blocks).astype(int):
            t0 = int(t0)
            di, _ = dsa.dsa_index_dense(i.q[t0:t0 + rows], i.w[t0:t0 + rows], i.k, self.k,
                                        q_pos0=i.q_pos0 + t0, K_scale=i.k_scale)
            got.append(_row_recall(self.out[0][t0:t0 + rows], di))
        r = np.concatenate(got)
        return {"mean": float(r.mean()), "min": float(r.min()), "rows": int(r.size),
                "note": f"|routed top-k ∩ dense top-k| / |dense top-k| over {blocks} blocks of {rows} rows"}

    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        K = i.k.cpu().numpy() if self.cfg["k_dtype"] == "fp8" else _f64(i.k)
        ks = i.k_scale.cpu().numpy() if i.k_scale is not None else None
        R = O.block_reps(K, 128, ks)
        rng = np.random.default_rng(seed)

        def one(_):
            t = int(rng.integers(0, self.T))
            O.block_routed(_f64(i.q[t:t + 1]), _f64(i.w[t:t + 1]), K, self.k, self.n_blocks, q_pos0=i.q_pos0 + t,
                           k_scale=ks, reps=R)
            return i.q_pos0 + t + 1
        return self._oracle_loop(budget_s, one)


class IvfRouted(BlockRouted):
    """Inverted-file routing (comparator): a plain k-means index of the keys,
    each query probing its best n_probe clusters, refined on their members."""
    iters = 10
    # the oracle routes on this library's index: no CPU-only reference arm
    reference_unavailable = ("the plain k-means index of 256K keys takes minutes of CPU time; the oracle times "
                             "routing + refine as the cpu_baseline of the GPU arm, on the GPU-built index")

    def __init__(self, device, size=None, name="fp8_256k"):
        super().__init__(device, size, name=name)
        self.C = max(1, self.N // 128)          # about 128 keys per cluster
        self.n_probe = self.n_blocks            # the same 8K-key budget as block routing
        T, q0 = self.T, self.inp.q_pos0
        # routing scores every centroid; the refine about n_probe * 128 keys
        self.alg_pairs = T * self.C + T * self.n_probe * 128
        self.alg_flops = self.alg_pairs * 2 * self.cfg["H"] * self.cfg["d"]
        self.launches_per_step = 3              # routing, tiles per query, refine
        self.kernel_launches_per_step = 2
        self.build_ms = None
        i = self.inp
        # the keys enter through the index, built once outside the timed steps
        self.host_src = [i.q, i.w] + ([i.k_scale] if i.k_scale is not None else [])

    def describe(self):
        d = Dense.describe(self)
        d["workload"] = d["workload"].replace("dense prefill", f"IVF-routed prefill (k-means index of {self.C} "
                                                               f"clusters, {self.iters} iterations, {self.n_probe} "
                                                               f"probed per query, then refined)")
        d.update(clusters=self.C, n_probe=self.n_probe, build_ms=self.build_ms,
                 metric_pairs="dense-equivalent causal pairs (alg_pairs = centroid routing + refine)")
        return d

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        e0.record()
        self.index = dsa.dsa_ivf_build(i.k, self.C, iters=self.iters, K_scale=i.k_scale)
        e1.record()
        torch.cuda.synchronize()
        self.build_ms = e0.elapsed_time(e1)
        self.max_tiles = self.index.probe_tile_bound(self.n_probe)
        T, H, d = i.q.shape
        self.out = (torch.empty((T, self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((T, self.k), dtype=torch.float32, device=i.q.device))
        kd = 2 if self.cfg["k_dtype"] == "fp8" else 0
        self.ws = torch.zeros(dsa.ivf_routed_workspace_bytes(T, self.N, H, d, self.k, self.C, self.n_probe,
                                                             self.max_tiles, 0, kd),
                              dtype=torch.uint8, device=i.q.device)

    def call(self, q, w, ks=None):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_ivf_routed(q, w, self.index, self.k, self.n_probe, q_pos0=self.inp.q_pos0, K_scale=ks,
                                 max_tiles=self.max_tiles, out=self.out, workspace=self.ws)

    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        K = i.k.cpu().numpy() if self.cfg["k_dtype"] == "fp8" else _f64(i.k)
        ks = i.k_scale.cpu().numpy() if i.k_scale is not None else None
        a = self.index.part("assign").cpu().numpy().astype(np.int64)
        cen = self.index.part("centroids_bf16").cpu().double().numpy()
        rng = np.random.default_rng(seed)

        def one(_):
            t = int(rng.integers(0, self.T))
            O.ivf_routed(_f64(i.q[t:t + 1]), _f64(i.w[t:t + 1]), K, self.k, self.n_probe, a, cen,
                         q_pos0=i.q_pos0 + t, k_scale=ks)
            return i.q_pos0 + t + 1
        return self._oracle_loop(budget_s, one)


class Group(Workload):
    def __init__(self, device, size=None, name="group_bf16_128k", mode=0):
        from synthetic import CONFIGS, make_dense_inputs
        self.name = name
        self.mode = mode
        self.cfg = dict(CONFIGS[name])
        if size:
            self.cfg["T"] = self.cfg["N"] = int(size)
        self.inp = make_dense_inputs(name, device=device, T=self.cfg["T"], N=self.cfg["N"],
                                     seed=self.cfg["seed"] + SHARD)
        c = self.cfg
        c["G"] = GROUP_OVERRIDE or c["G"]
        c["bank"] = BANK_OVERRIDE or c["bank"]
        self.T, self.N, self.k, self.G, self.B = c["T"], c["N"], c["k"], c["G"], c["bank"]
        q0 = self.inp.q_pos0
        self.pairs = self.T * q0 + self.T * (self.T + 1) // 2      # dense-equivalent
        ng = (self.T + self.G - 1) // self.G
        scan = sum(min(self.T, (g + 1) * self.G) + q0 for g in range(ng))
        refine = 0
        if mode in (0, 2):
            for g in range(ng):
                nb = min(self.B, q0 + min(self.T, (g + 1) * self.G))
                nm = min(self.T, (g + 1) * self.G) - g * self.G
                # Refine with local additions streams G more key slots per group
                refine += (nb + (self.G if mode == 2 else 0)) * nm
        self.alg_pairs = scan + refine
        self.alg_flops = self.alg_pairs * 2 * c["H"] * c["d"]
        self.rows = self.T
        i = self.inp
        self.host_src = [i.q, i.w, i.k] + ([i.k_scale] if i.k_scale is not None else [])
        # proxy mean, proxy scan, then Refine: (local key map +) bank gather + re-scoring; Reuse: bank ranking
        self.launches_per_step = {0: 4, 1: 3, 2: 5}[mode] + (1 if c["k_dtype"] == "fp8" else 0)
        self.kernel_launches_per_step = 1 if mode == 1 else 2

    def describe(self):
        c = self.cfg
        m = {0: "Refine", 1: "Reuse", 2: "Refine with local additions"}[self.mode]
        kd = "fp8 e4m3 k + scale" if c["k_dtype"] == "fp8" else "bf16 k"
        return {"workload": f"{self.name}: group-shared prefill ({m}) T=N={c['T']} causal, H={c['H']}, d={c['d']}, "
                            f"G={c['G']}, bank={c['bank']}, k={c['k']}, bf16 q, {kd}, fp32 w, seed {c['seed']}",
                "T": c["T"], "N": c["N"], "G": c["G"], "bank": c["bank"], "k": c["k"], "mode": m,
                "metric_pairs": "dense-equivalent causal pairs (alg_pairs = proxy scan + bank re-scoring)",
                "l2": "inputs larger than L2, no flush"}

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        T, H, d = i.q.shape
        kd = 2 if self.cfg["k_dtype"] == "fp8" else 0
        self.ws = torch.zeros(dsa.group_workspace_bytes(T, self.N, H, d, self.k, self.G, self.B, 0, kd),
                              dtype=torch.uint8, device=i.q.device)
        self.out = (torch.empty((T, self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((T, self.k), dtype=torch.float32, device=i.q.device))

    def call(self, q, w, k, ks=None):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_group(q, w, k, self.k, self.G, self.B, mode=self.mode, q_pos0=self.inp.q_pos0, K_scale=ks,
                            out=self.out, workspace=self.ws)

    e2e_note = ("dsa_index_group_host: page-locked host inputs and outputs, copy-in / indexer / copy-out "
                "pipelined in chunks of whole groups by the library, every step")

    def e2e_buffers(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        T, H, d = i.q.shape
        kd = dsa.DSA_DTYPE_FP8_E4M3 if i.k_scale is not None else dsa.DSA_DTYPE_BF16
        return self._host_e2e_buffers(dsa.group_host_staging_bytes(T, self.N, H, d, self.k, self.G, self.B,
                                                                   dsa.DSA_DTYPE_BF16, kd))

    def e2e_step(self, host, dev_bufs, host_out):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_group_host(host[0], host[1], host[2], self.k, self.G, self.B, mode=self.mode,
                                 q_pos0=self.inp.q_pos0, K_scale=host[3] if len(host) > 3 else None, out=host_out,
                                 staging=self.staging)

    def recall(self, blocks=4, rows=512):
        """Mean recall of the exact dense top-k (this library's dense kernel)
        by the group output, over `blocks` row blocks spread over the
        workload, outside the timed region."""
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        got = []
        for t0 in np.linspace(0, self.T - rows, blocks).astype(int):
            t0 = int(t0) // self.G * self.G
            di, _ = dsa.dsa_index_dense(i.q[t0:t0 + rows], i.w[t0:t0 + rows], i.k, self.k,
                                        q_pos0=i.q_pos0 + t0, K_scale=i.k_scale)
            got.append(_row_recall(self.out[0][t0:t0 + rows], di))
        r = np.concatenate(got)
        return {"mean": float(r.mean()), "min": float(r.min()), "rows": int(r.size),
                "note": f"|group top-k ∩ dense top-k| / |dense top-k| over {blocks} blocks of {rows} rows"}

    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        K = i.k.cpu().numpy() if self.cfg["k_dtype"] == "fp8" else _f64(i.k)
        ks = i.k_scale.cpu().numpy() if i.k_scale is not None else None
        rng = np.random.default_rng(seed)
        ng = (self.T + self.G - 1) // self.G

        def one(_):
            # one whole group (proxy scan + every member); counted like the
            # GPU arm: the members' dense-equivalent causal pairs
            g = int(rng.integers(0, ng))
            r0, r1 = g * self.G, min(self.T, (g + 1) * self.G)
            O.group(_f64(i.q[r0:r1]), _f64(i.w[r0:r1]), K[:i.q_pos0 + r1], self.k, self.G, self.B, self.mode,
                    q_pos0=i.q_pos0 + r0, k_scale=None if ks is None else ks[:i.q_pos0 + r1],
                    q_dtype=self.cfg["q_dtype"])
            return sum(i.q_pos0 + t + 1 for t in range(r0, r1))
        return self._oracle_loop(budget_s, one)


class Decode(Workload):
    name = "decode_bf16_32x128k"
    bound = "hbm"
    alg_bytes_note = "cached keys once + queries + weights"

    def __init__(self, device, size=None):
        from synthetic import CONFIGS, make_decode_inputs
        self.cfg = dict(CONFIGS[self.name])
        if size:
            self.cfg["Nb"] = int(size)
        if M_OVERRIDE:
            self.cfg["m"] = int(M_OVERRIDE)
        c = self.cfg
        self.inp = make_decode_inputs(self.name, device=device, lengths=[c["Nb"]] * c["B"], m=c["m"],
                                      seed=c["seed"] + SHARD)
        self.k = c["k"]
        m = c["m"]
        self.pairs = self.alg_pairs = c["B"] * sum(c["Nb"] - m + j + 1 for j in range(m))
        self.alg_flops = self.alg_pairs * 2 * c["H"] * c["d"]
        i = self.inp
        # compulsory HBM bytes of the scoring kernel: every cached key once,
        # the queries and weights (the merge kernel writes the outputs)
        self.alg_bytes = (i.k.numel() * i.k.element_size() + i.q.numel() * i.q.element_size()
                          + i.w.numel() * 4)
        self.rows = i.q.shape[0]
        self.ko = i.k_offsets.to(device, torch.int64)
        self.qo = i.q_offsets.to(device, torch.int32)
        self.total_keys = int(i.k_offsets[-1])
        self.host_src = [i.q, i.w, i.k]
        self.launches_per_step = 2

    def describe(self):
        c = self.cfg
        return {"workload": f"{self.name}: decode, {c['B']} caches x {c['Nb']} keys bf16, {c['m']} new queries "
                            f"each, H={c['H']}, d={c['d']}, k={c['k']}, 1% planted keys, seed {c['seed']}",
                "B": c["B"], "Nb": c["Nb"], "m": c["m"], "H": c["H"], "d": c["d"], "k": c["k"],
                "l2": f"keys larger than L2 ({self.inp.k.numel() * 2 >> 20} MiB), no flush"}

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        c = self.cfg
        self.ws = torch.zeros(dsa.decode_workspace_bytes(c["B"], i.q.shape[0], c["Nb"], c["H"], c["d"], self.k,
                                                         0, 0), dtype=torch.uint8, device=i.q.device)
        self.out = (torch.empty((i.q.shape[0], self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((i.q.shape[0], self.k), dtype=torch.float32, device=i.q.device))

    def call(self, q, w, k):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_decode(q, w, k, self.k, self.ko, self.qo, max_keys=self.cfg["Nb"], total_keys=self.total_keys,
                             out=self.out, workspace=self.ws)

    e2e_note = ("dsa_index_decode_host: page-locked host caches, queries and outputs, one copy-in / indexer / "
                "copy-out per step")

    def e2e_buffers(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        c = self.cfg
        self.ko_h, self.qo_h = i.k_offsets.cpu().to(torch.int64), i.q_offsets.cpu().to(torch.int32)
        return self._host_e2e_buffers(dsa.decode_host_staging_bytes(c["B"], i.q.shape[0], self.total_keys, c["Nb"],
                                                                    c["H"], c["d"], self.k, dsa.DSA_DTYPE_BF16,
                                                                    dsa.DSA_DTYPE_BF16))

    def e2e_step(self, host, dev_bufs, host_out):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_decode_host(host[0], host[1], host[2], self.k, self.ko_h, self.qo_h, max_keys=self.cfg["Nb"],
                                  out=host_out, staging=self.staging)

    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        c = self.cfg
        rng = np.random.default_rng(seed)
        cache = {}

        def one(_):
            r = int(rng.integers(0, i.q.shape[0]))
            b, j = r // c["m"], r % c["m"]
            if b not in cache:
                cache.clear()
                cache[b] = _f64(i.k[b * c["Nb"]:(b + 1) * c["Nb"]])
            p = c["Nb"] - c["m"] + j
            S = O.score_rows(_f64(i.q[r:r + 1]), _f64(i.w[r:r + 1]), cache[b][:p + 1])[0]
            O.select_topk(S, self.k)
            return p + 1
        return self._oracle_loop(budget_s, one)


class DecodeGroup(Decode):
    """PIVOT in decode: each sequence's new queries form one group (bank 8192)."""
    bank = 8192
    e2e_buffers = Workload.e2e_buffers
    e2e_step = Workload.e2e_step
    e2e_note = Workload.e2e_note
    alg_bytes_note = "cached keys once + proxies (+ Refine: gathered bank keys, queries, weights)"

    def __init__(self, device, size=None, mode=0):
        super().__init__(device, size)
        c = self.cfg
        self.mode = mode
        m, nb = c["m"], c["Nb"]
        # proxy scan over every cache, then (Refine) each query over the bank
        self.alg_pairs = c["B"] * nb + (c["B"] * m * min(self.bank, nb) if mode == 0 else 0)
        self.alg_flops = self.alg_pairs * 2 * c["H"] * c["d"]
        i = self.inp
        # compulsory HBM bytes of the scoring kernels: every cached key once and
        # the proxies; Refine adds its gathered bank keys and its queries
        self.alg_bytes = i.k.numel() * i.k.element_size() + c["B"] * c["H"] * (c["d"] * 2 + 4)
        if mode == 0:
            self.alg_bytes += c["B"] * min(self.bank, nb) * c["d"] * 2 + i.q.numel() * 2 + i.w.numel() * 4
        self.kernel_launches_per_step = 2 if mode == 0 else 1
        # proxy mean, scan, merge, then Refine: gather + re-scoring; Reuse: ranking
        self.launches_per_step = 5 if mode == 0 else 4

    def describe(self):
        d = super().describe()
        m = "Refine" if self.mode == 0 else "Reuse"
        d["workload"] = d["workload"].replace("decode,", f"decode group ({m}, bank {self.bank}, group = a sequence's "
                                                           f"new queries),")
        d["bank"], d["mode"] = self.bank, m
        d["metric_pairs"] = "dense-equivalent decode pairs (alg_pairs = proxy scan + bank re-scoring)"
        return d

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        c = self.cfg
        self.ws = torch.zeros(dsa.decode_group_workspace_bytes(c["B"], i.q.shape[0], c["Nb"], c["H"], c["d"],
                                                               self.k, self.bank, 0, 0),
                              dtype=torch.uint8, device=i.q.device)
        self.out = (torch.empty((i.q.shape[0], self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((i.q.shape[0], self.k), dtype=torch.float32, device=i.q.device))

    def call(self, q, w, k):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_index_decode_group(q, w, k, self.k, self.ko, self.qo, self.bank, mode=self.mode,
                                   max_keys=self.cfg["Nb"], total_keys=self.total_keys, out=self.out,
                                   workspace=self.ws)

    def recall(self):
        """Mean recall of the decode indexer's exact top-k by the group output."""
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        di, _ = dsa.dsa_index_decode(i.q, i.w, i.k, self.k, self.ko, self.qo, max_keys=self.cfg["Nb"],
                                     total_keys=self.total_keys)
        r = _row_recall(self.out[0], di)
        return {"mean": float(r.mean()), "min": float(r.min()), "rows": int(r.size),
                "note": "|group top-k ∩ decode top-k| / |decode top-k| over every query row"}

    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        c = self.cfg
        rng = np.random.default_rng(seed)
        m, nb = c["m"], c["Nb"]

        def one(_):
            # one whole sequence: proxy scan + its queries; counted like the
            # GPU arm (the queries' dense-equivalent pairs)
            b = int(rng.integers(0, c["B"]))
            K = _f64(i.k[b * nb:(b + 1) * nb])
            O.decode_group(_f64(i.q[b * m:(b + 1) * m]), _f64(i.w[b * m:(b + 1) * m]), K, [0, nb], [0, m],
                           self.k, self.bank, self.mode, q_dtype=c["q_dtype"])
            return sum(nb - m + j + 1 for j in range(m))
        return self._oracle_loop(budget_s, one)


WORKLOADS = {
    "dense_bf16_32k": lambda dev, size: Dense(dev, size),
    "decode_bf16_32x128k": lambda dev, size: Decode(dev, size),
    "decode_bf16_32x128k_group_refine": lambda dev, size: DecodeGroup(dev, size, 0),
    "decode_bf16_32x128k_group_reuse": lambda dev, size: DecodeGroup(dev, size, 1),
    "group_bf16_128k_refine": lambda dev, size: Group(dev, size, "group_bf16_128k", 0),
    "group_bf16_128k_reuse": lambda dev, size: Group(dev, size, "group_bf16_128k", 1),
    "group_bf16_128k_refine_local": lambda dev, size: Group(dev, size, "group_bf16_128k", 2),
    "dense_bf16_128k": lambda dev, size: Dense(dev, size or 131072, name="group_bf16_128k"),
    "fp8_256k_dense": lambda dev, size: Dense(dev, size, name="fp8_256k"),
    "fp8_256k_block_routed": lambda dev, size: BlockRouted(dev, size, name="fp8_256k"),
    "group_bf16_128k_block_routed": lambda dev, size: BlockRouted(dev, size, name="group_bf16_128k"),
    "fp8_256k_ivf_routed": lambda dev, size: IvfRouted(dev, size, name="fp8_256k"),
    "group_bf16_128k_ivf_routed": lambda dev, size: IvfRouted(dev, size, name="group_bf16_128k"),
    "fp8_256k_group_refine": lambda dev, size: Group(dev, size, "fp8_256k", 0),
    "fp8_256k_group_reuse": lambda dev, size: Group(dev, size, "fp8_256k", 1),
}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons sampled every 50 ms by NVML (reads only).

    NVML is opened before the timed region and sampled once more when it
    ends, so that a short timed region still has a clock record."""
    REASONS = {"hw_slowdown": 0x8, "sw_thermal_slowdown": 0x20, "hw_thermal_slowdown": 0x40,
               "hw_power_brake_slowdown": 0x80, "sw_power_cap": 0x4}

    def __init__(self, gpu_index):
        import threading
        self.gpu = gpu_index
        self.samples = []
        self.reasons = set()
        self.max_mhz = None
        self._stop = threading.Event()
        self._thr = None
        self._nvml = None
        self._h = None
        self.err = None

    def _sample(self):
        N, h = self._nvml, self._h
        self.samples.append(float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)))
        r = int(N.nvmlDeviceGetCurrentClocksEventReasons(h))
        for nm, bit in self.REASONS.items():
            if r & bit:
                self.reasons.add(nm)

    def _run(self):
        try:
            while True:
                self._sample()
                if self._stop.wait(0.05):
                    break
        except Exception as e:  # pragma: no cover - reported in the JSON line
            self.err = repr(e)

    def start(self):
        import threading
        vis = os.environ.get("CUDA_VISIBLE_DEVICES")
        if vis:
            try:
                self.gpu = int(vis.split(",")[self.gpu])
            except (ValueError, IndexError):
                pass
        try:
            import pynvml as N
            N.nvmlInit()
            self._nvml = N
            self._h = N.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(self._h, N.NVML_CLOCK_SM))
        except Exception as e:  # no NVML: the JSON line says why
            self.err = repr(e)
            self._nvml = None
            return
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()

    def stop(self):
        self._stop.set()
        if self._thr is not None:
            self._thr.join(timeout=5)
        if self._nvml is not None:
            try:
                self._sample()  # the end of the timed region
                self._nvml.nvmlShutdown()
            except Exception as e:  # pragma: no cover
                self.err = self.err or repr(e)
        out = {"sm_mhz": statistics.median(self.samples) if self.samples else None, "sm_max_mhz": self.max_mhz,
               "samples": len(self.samples), "reasons": sorted(self.reasons), "source": "NVML, 50 ms"}
        if self.err:
            out["error"] = self.err
        return out


# ---------------------------------------------------------------------------
def _dist():
    ws = int(os.environ.get("WORLD_SIZE", "1"))
    if ws > 1:
        import datetime
        import torch.distributed as dist
        lr = int(os.environ.get("LOCAL_RANK", "0"))
        torch.cuda.set_device(lr)
        dist.init_process_group("nccl", timeout=datetime.timedelta(seconds=120),
                                device_id=torch.device("cuda", lr))
        return dist, dist.get_rank(), ws, lr
    return None, 0, 1, 0


def _barrier(dist):
    if dist is not None:
        dist.barrier()


def kernel_source_hash(read):
    """sha256 (16 hex digits) of the scoring kernel's device code: dsa_tc.cu
    up to its host launchers, dsa_topk.cuh and dsa_common.cuh, without
    comments, #include lines and whitespace.  `read(name)` returns a file's
    text.  Only a change of device code makes a traffic capture stale."""
    import hashlib
    import re
    h = hashlib.sha256()
    for f in ("dsa_tc.cu", "dsa_topk.cuh", "dsa_common.cuh"):
        src = read(f)
        if f == "dsa_tc.cu":
            src = src[:src.index("static int launch_tc(")]
        src = re.sub(r"/\*.*?\*/", "", src, flags=re.S)
        src = re.sub(r"//[^\n]*", "", src)
        src = re.sub(r"#include[^\n]*", "", src)
        h.update(re.sub(r"\s+", "", src).encode())
    return h.hexdigest()[:16]


def _kernel_source_hash():
    def read(name):
        with open(os.path.join(ROOT, "sparse_attention_token_index_b200", "csrc", name)) as fh:
            return fh.read()
    return kernel_source_hash(read)


def _traffic(config, resized=False):
    """ncu DRAM bytes per scoring-kernel launch from profiles/, or None when
    there is no capture for this workload, the kernel changed since, or the
    run is resized (--T): the captures are of the workloads' own sizes."""
    if resized:
        return None
    p = os.path.join(ROOT, "profiles", f"{config}_traffic.txt")
    if not os.path.exists(p):
        return None
    kv = {}
    with open(p) as f:
        for line in f:
            if "=" in line and not line.startswith("#"):
                a, b = line.split("=", 1)
                kv[a.strip()] = b.strip()
    if kv.get("kernel_source") != _kernel_source_hash():
        return None
    return int(kv["bytes_per_launch"])


def _max_over_ranks(dist, x, device="cuda"):
    """The slowest rank's time: every rank takes part, every rank gets it."""
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device=device)
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def whole_job_rate(units_per_rank_step, world, steps, slowest_ms):
    """Whole-job throughput of N replicas: the units all ranks processed in
    the timed steps over the slowest rank's time (units per second)."""
    return units_per_rank_step * world * steps / (slowest_ms / 1e3)


def run_reference(args):
    """The CPU oracle, as it stands, on a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = WORKLOADS[args.config](dev, args.T)
    if getattr(wl, "reference_unavailable", None):
        print(json.dumps({"impl": "reference", "unavailable": wl.reference_unavailable}))
        return
    cores, host_cores = _oracle_threads()
    per_step = max(1.0, 20.0 / max(1, args.steps + args.warmup))
    for _ in range(args.warmup):
        wl.oracle_sample(budget_s=per_step)
    pairs = 0
    el = 0.0
    rows = 0
    for s in range(args.steps):
        p, r, e = wl.oracle_sample(budget_s=per_step, seed=s + 1)
        pairs += p
        rows += r
        el += e
    v = pairs / el / 1e9
    line = {"metric": METRIC, "value": v, "unit": "Gpairs/s", "impl": "reference", "n_gpus": args.gpus,
            "steps": args.steps, "warmup": args.warmup, "ms_per_step": 1e3 * el / args.steps,
            "higher_is_better": True, "scaling": "weak", "vs_baseline": None, "dtype": "f64",
            "data": "synthetic", "config": dict(wl.describe(), parallelism=_parallelism(
                int(os.environ.get("WORLD_SIZE", args.gpus)))),
            "cpu_baseline": {"value": v, "unit": "Gpairs/s", "cores": cores, "host_cores": host_cores,
                             "kind": "oracle",
                             "sample": f"{rows} random query rows of the workload, full causal prefix each, "
                                       f"numpy float64 scores + full stable sort"},
            "e2e": {"value": v, "unit": "Gpairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="dense_bf16_32k", choices=sorted(WORKLOADS),
                    help="dense_bf16_32k is the headline workload; the others measure the remaining paths")
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--T", type=int, default=None,
                    help="other T = N (prefill) or cache length (decode), e.g. for profiling captures")
    ap.add_argument("--group", type=int, default=None, help="group size G of the group workloads")
    ap.add_argument("--bank", type=int, default=None, help="candidate bank B of the group workloads")
    ap.add_argument("--m", type=int, default=None, help="new queries per sequence (1..4) of the decode workloads")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    global GROUP_OVERRIDE, BANK_OVERRIDE, M_OVERRIDE
    GROUP_OVERRIDE, BANK_OVERRIDE, M_OVERRIDE = args.group, args.bank, args.m
    if args.bank:
        DecodeGroup.bank = args.bank
    if args.impl == "reference":
        run_reference(args)
        return

    dist, rank, world, local = _dist()
    torch.cuda.set_device(local)
    # weak scaling: every rank indexes its own batch of the workload's shape
    global SHARD
    SHARD = rank
    import sparse_attention_token_index_b200 as dsa
    dsa.lib()
    wl = WORKLOADS[args.config]("cuda", args.T)
    wl.setup()
    stream = torch.cuda.current_stream()

    for _ in range(args.warmup):
        wl.step()
    wl.check()

    clk = ClockSampler(local)
    ev = [(torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)) for _ in range(args.steps)]
    # the library records an event pair around each scoring-kernel launch
    # on this stream (events created here, before the timed region)
    n_kernel = wl.kernel_launches_per_step * args.steps
    dsa.dsa_kernel_timer_start(n_kernel)
    _barrier(dist)
    torch.cuda.synchronize()
    clk.start()
    for e0, e1 in ev:
        e0.record(stream)
        wl.step()
        e1.record(stream)
    torch.cuda.synchronize()
    _barrier(dist)
    clocks = clk.stop()
    kernel_ms, kernel_n = dsa.dsa_kernel_timer_stop()
    if kernel_n != n_kernel:
        raise RuntimeError(f"timed {kernel_n} scoring-kernel launches, expected {n_kernel}")
    wl.check()
    per = [e0.elapsed_time(e1) for e0, e1 in ev]  # ms per launch
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    total_ms = _max_over_ranks(dist, total_ms)
    kernel_ms = _max_over_ranks(dist, kernel_ms)
    ms_step = total_ms / args.steps
    value = whole_job_rate(wl.pairs, world, args.steps, total_ms) / 1e9
    alg_value = whole_job_rate(wl.alg_pairs, world, args.steps, total_ms) / 1e9
    rows_s = whole_job_rate(wl.rows, world, args.steps, total_ms)

    pk = _peaks()
    avg_launch = kernel_ms / kernel_n                     # ms per scoring-kernel launch
    scope = (f"kernel time from CUDA events around each of the {kernel_n} scoring-kernel launches in the timed "
             f"region ({wl.kernel_launches_per_step} per step, {kernel_ms / args.steps:.4f} ms of the "
             f"{ms_step:.4f} ms step)")
    per_launch_flops = wl.alg_flops / wl.kernel_launches_per_step
    per_launch_bytes = wl.alg_bytes / wl.kernel_launches_per_step
    if wl.bound == "tensor":
        achieved = per_launch_flops / (avg_launch / 1e3) / 1e12
        sustained = total_ms / 1e3 > SUSTAINED_AFTER_S
        peak = pk["bf16_sus"] if sustained else pk["bf16"]
        rule = (f"the timed region ran {total_ms / 1e3:.2f} s: "
                + ("longer than" if sustained else "shorter than")
                + f" {SUSTAINED_AFTER_S:.0f} s, so the {'sustained' if sustained else 'burst'} figure applies")
        roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                "traffic": None, "alg_per_launch": per_launch_flops, "kernel_ms": avg_launch,
                "frac_burst": achieved / pk["bf16"], "frac_sustained": achieved / pk["bf16_sus"],
                "note": f"algorithmic 2*H*d flop per scored pair; peak = {pk['src']} "
                        f"{'sustained' if sustained else 'burst'} cuBLAS bf16 ({rule}); {scope}"}
    else:
        achieved = per_launch_bytes / (avg_launch / 1e3) / 1e9
        peak = pk["hbm"]
        roof = {"bound": "hbm", "achieved": achieved, "peak": peak, "unit": "GB/s", "frac": achieved / peak,
                "traffic": None, "alg_per_launch": per_launch_bytes, "kernel_ms": avg_launch,
                "note": f"algorithmic bytes = {wl.alg_bytes_note}; peak = {pk['src']} "
                        f"copy bandwidth; {scope}"}
    roof["traffic"] = _traffic(args.config, resized=args.T is not None)

    e2e = None
    if not args.no_e2e:
        host = wl.host_inputs()
        dev, hout, h2d, d2h = wl.e2e_buffers()
        for _ in range(2):
            wl.e2e_step(host, dev, hout)
        torch.cuda.synchronize()
        _barrier(dist)
        e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
        n_e2e = max(3, min(args.steps, 10))
        e0.record(stream)
        for _ in range(n_e2e):
            wl.e2e_step(host, dev, hout)
        e1.record(stream)
        torch.cuda.synchronize()
        e2e_ms = _max_over_ranks(dist, e0.elapsed_time(e1))
        e2e = {"value": whole_job_rate(wl.pairs, world, n_e2e, e2e_ms) / 1e9, "unit": "Gpairs/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "note": wl.e2e_note}

    recall = wl.recall() if hasattr(wl, "recall") else None   # after timing; the last step's output
    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        p, r, el = wl.oracle_sample(budget_s=15.0)
        thr, host_cores = _oracle_threads()
        cpu = {"value": p / el / 1e9, "unit": "Gpairs/s", "cores": thr, "host_cores": host_cores, "kind": "oracle",
               "sample": f"{r} random query rows of the workload ({p} causal pairs), full prefix each, "
                         f"numpy float64 + full stable sort, {el:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gpairs/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": _dtype_label(wl.cfg), "data": "synthetic", "config": wl.describe(),
                "rows_per_s": rows_s, "alg_pairs_per_s": alg_value * 1e9, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": wl.launches_per_step * args.steps, "clocks": clocks,
                "launch_ms": {"min": min(per), "median": statistics.median(per),
                              "p95": float(np.percentile(per, 95)), "max": max(per)}}
        line["config"]["parallelism"] = _parallelism(world)
        if hasattr(wl, "recall"):
            line["recall_vs_dense"] = recall
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
