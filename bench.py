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
FLOP_PER_PAIR = 2 * 64 * 128  # 2 * H * d


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
class Dense:
    name = "dense_bf16_32k"

    def __init__(self, device, size=None):
        from synthetic import CONFIGS, make_dense_inputs
        self.cfg = dict(CONFIGS[self.name])
        if size:
            self.cfg["T"] = self.cfg["N"] = int(size)
        self.inp = make_dense_inputs(self.name, device=device, T=self.cfg["T"], N=self.cfg["N"])
        self.T, self.N, self.k = self.cfg["T"], self.cfg["N"], self.cfg["k"]
        q0 = self.inp.q_pos0
        self.pairs = sum(q0 + t + 1 for t in range(self.T))
        self.rows = self.T

    def describe(self):
        c = self.cfg
        return {"workload": f"{self.name}: dense prefill T=N={c['T']} causal, H={c['H']}, d={c['d']}, "
                            f"k={c['k']}, bf16 q/k, fp32 w, low-rank AR(1) latent recipe, seed {c['seed']}",
                "T": c["T"], "N": c["N"], "H": c["H"], "d": c["d"], "k": c["k"],
                "l2": f"inputs larger than L2 (Q is {c['T'] * c['H'] * c['d'] * 2 >> 20} MiB), no flush"}

    def setup(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        T, H, d = i.q.shape
        self.ws = torch.zeros(dsa.dense_workspace_bytes(T, self.N, H, d, self.k, 0, 0), dtype=torch.uint8,
                              device=i.q.device)
        self.out = (torch.empty((T, self.k), dtype=torch.int32, device=i.q.device),
                    torch.empty((T, self.k), dtype=torch.float32, device=i.q.device))

    def step(self):
        import sparse_attention_token_index_b200 as dsa
        i = self.inp
        dsa.dsa_index_dense(i.q, i.w, i.k, self.k, q_pos0=i.q_pos0, out=self.out, workspace=self.ws)

    def check(self):
        import sparse_attention_token_index_b200 as dsa
        dsa.dsa_check_status(self.ws)

    launches_per_step = 1

    # end to end through the public API with host buffers
    def host_inputs(self):
        i = self.inp
        return [t.cpu().pin_memory() for t in (i.q, i.w, i.k)]

    def e2e_step(self, host, dev_bufs, host_out):
        import sparse_attention_token_index_b200 as dsa
        q, w, k = dev_bufs
        for d_, h_ in zip(dev_bufs, host):
            d_.copy_(h_, non_blocking=True)
        dsa.dsa_index_dense(q, w, k, self.k, q_pos0=self.inp.q_pos0, out=self.out, workspace=self.ws)
        host_out[0].copy_(self.out[0], non_blocking=True)
        host_out[1].copy_(self.out[1], non_blocking=True)

    def e2e_buffers(self):
        i = self.inp
        dev = [torch.empty_like(t) for t in (i.q, i.w, i.k)]
        hout = [torch.empty(self.out[0].shape, dtype=torch.int32).pin_memory(),
                torch.empty(self.out[1].shape, dtype=torch.float32).pin_memory()]
        h2d = sum(t.numel() * t.element_size() for t in dev)
        d2h = sum(t.numel() * t.element_size() for t in hout)
        return dev, hout, h2d, d2h

    # CPU oracle on a bounded sample of rows
    def oracle_sample(self, budget_s=15.0, seed=0):
        from oracle import dsa_oracle as O
        i = self.inp
        K = i.k.float().cpu().double().numpy()
        rng = np.random.default_rng(seed)
        t0 = time.perf_counter()
        pairs = 0
        nrows = 0
        while time.perf_counter() - t0 < budget_s:
            t = int(rng.integers(0, self.T))
            q = i.q[t:t + 1].float().cpu().double().numpy()
            w = i.w[t:t + 1].cpu().double().numpy()
            O.dense(q, w, K, self.k, q_pos0=i.q_pos0 + t)
            pairs += i.q_pos0 + t + 1
            nrows += 1
        el = time.perf_counter() - t0
        return pairs, nrows, el


WORKLOADS = {"dense_bf16_32k": Dense}


# ---------------------------------------------------------------------------
# clocks during the timed region
# ---------------------------------------------------------------------------
class ClockSampler:
    """SM clock and clock-event reasons sampled every 50 ms by NVML (reads only)."""
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
        self.err = None

    def _run(self):
        try:
            import pynvml as N
            N.nvmlInit()
            h = N.nvmlDeviceGetHandleByIndex(self.gpu)
            self.max_mhz = float(N.nvmlDeviceGetMaxClockInfo(h, N.NVML_CLOCK_SM))
            while not self._stop.is_set():
                self.samples.append(float(N.nvmlDeviceGetClockInfo(h, N.NVML_CLOCK_SM)))
                r = int(N.nvmlDeviceGetCurrentClocksEventReasons(h))
                for nm, bit in self.REASONS.items():
                    if r & bit:
                        self.reasons.add(nm)
                self._stop.wait(0.05)
            N.nvmlShutdown()
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
        self._thr = threading.Thread(target=self._run, daemon=True)
        self._thr.start()

    def stop(self):
        self._stop.set()
        if self._thr is not None:
            self._thr.join(timeout=5)
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


def _max_over_ranks(dist, x):
    if dist is None:
        return x
    t = torch.tensor([x], dtype=torch.float64, device="cuda")
    dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def run_reference(args):
    """The CPU oracle, as it stands, on a bounded sample of the workload."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    W = WORKLOADS[args.config]
    dev = "cuda" if torch.cuda.is_available() else "cpu"
    wl = W(dev, args.T)
    cores = torch.get_num_threads()
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
            "data": "synthetic", "config": wl.describe(),
            "cpu_baseline": {"value": v, "unit": "Gpairs/s", "cores": cores, "kind": "oracle",
                             "sample": f"{rows} random query rows of the workload, full causal prefix each, "
                                       f"numpy float64 scores + full stable sort"},
            "e2e": {"value": v, "unit": "Gpairs/s", "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(line))


def main():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=100)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--config", default="dense_bf16_32k", choices=sorted(WORKLOADS))
    ap.add_argument("--impl", default="ours", choices=["ours", "reference"])
    ap.add_argument("--T", type=int, default=None, help="smaller T = N for profiling captures")
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--no-e2e", action="store_true")
    args = ap.parse_args()
    args.warmup = max(3, args.warmup)
    if args.impl == "reference":
        run_reference(args)
        return

    dist, rank, world, local = _dist()
    torch.cuda.set_device(local)
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
    wl.check()
    per = [e0.elapsed_time(e1) for e0, e1 in ev]  # ms per launch
    total_ms = ev[0][0].elapsed_time(ev[-1][1])
    total_ms = _max_over_ranks(dist, total_ms)
    ms_step = total_ms / args.steps
    pairs = wl.pairs * world
    value = pairs * args.steps / (total_ms / 1e3) / 1e9
    rows_s = wl.rows * world * args.steps / (total_ms / 1e3)

    pk = _peaks()
    flops = wl.pairs * FLOP_PER_PAIR
    avg_launch = sum(per) / len(per)
    achieved = flops / (avg_launch / 1e3) / 1e12
    peak = pk["bf16_sus"]
    roof = {"bound": "tensor", "achieved": achieved, "peak": peak, "unit": "TFLOP/s",
            "frac": achieved / peak, "traffic": None,
            "note": f"algorithmic 2*H*d flop per causal pair; peak = {pk['src']} sustained cuBLAS bf16 "
                    f"(kernel timed inside a back-to-back loop); frac of burst peak "
                    f"{achieved / pk['bf16']:.3f}"}
    traffic_file = os.path.join(ROOT, "profiles", f"{args.config}_traffic.json")
    if os.path.exists(traffic_file):
        with open(traffic_file) as f:
            roof["traffic"] = json.load(f).get("bytes_per_launch")

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
        e2e = {"value": wl.pairs * world * n_e2e / (e2e_ms / 1e3) / 1e9, "unit": "Gpairs/s",
               "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h, "steps": n_e2e,
               "note": "pinned host inputs copied in, indexer run, idx/val copied out, every step"}

    cpu = None
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        p, r, el = wl.oracle_sample(budget_s=15.0)
        cpu = {"value": p / el / 1e9, "unit": "Gpairs/s", "cores": torch.get_num_threads(), "kind": "oracle",
               "sample": f"{r} random query rows of the workload ({p} causal pairs), full prefix each, "
                         f"numpy float64 + full stable sort, {el:.1f} s"}

    if rank == 0:
        line = {"metric": METRIC, "value": value, "unit": "Gpairs/s", "n_gpus": world, "steps": args.steps,
                "warmup": args.warmup, "ms_per_step": ms_step, "higher_is_better": True, "scaling": "weak",
                "vs_baseline": None, "dtype": "bf16", "data": "synthetic", "config": wl.describe(),
                "rows_per_s": rows_s, "roofline": roof, "cpu_baseline": cpu, "e2e": e2e,
                "gpu_launches": wl.launches_per_step * args.steps, "clocks": clocks,
                "launch_ms": {"min": min(per), "median": statistics.median(per), "max": max(per)}}
        line["config"]["parallelism"] = f"replicas x{world}" if world > 1 else "single GPU"
        print(json.dumps(line))
    if dist is not None:
        dist.destroy_process_group()


if __name__ == "__main__":
    main()
