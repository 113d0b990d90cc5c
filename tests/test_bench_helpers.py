"""bench.py's host helpers: the kernel-source hash that keeps a DRAM traffic
capture tied to the device code it measured."""
import os
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)

import bench  # noqa: E402

BASE = {
    "dsa_tc.cu": '#include "a.h"\n__global__ void k() { int x = 1; }  // note\nstatic int launch_tc(int g) { return g; }\n',
    "dsa_topk.cuh": "__device__ int f() { return 2; } /* doc */\n",
    "dsa_common.cuh": "__device__ int g() { return 3; }\n",
}


def _h(files):
    return bench.kernel_source_hash(lambda name: files[name])


def test_hash_ignores_comments_includes_and_host_launchers():
    h0 = _h(BASE)
    changed = dict(BASE)
    changed["dsa_tc.cu"] = ('#include <atomic>\n#include "a.h"\n// a new comment\n__global__ void k() {\n  int x = 1;\n}'
                            '\nstatic int launch_tc(int g) { return g + 1; }\n')
    changed["dsa_topk.cuh"] = "__device__ int f() { return 2; } /* other doc */\n"
    assert _h(changed) == h0


def test_hash_sees_device_code():
    h0 = _h(BASE)
    for name, new in (("dsa_tc.cu", BASE["dsa_tc.cu"].replace("x = 1", "x = 2")),
                      ("dsa_topk.cuh", "__device__ int f() { return 4; }\n"),
                      ("dsa_common.cuh", "__device__ int g() { return 5; }\n")):
        changed = dict(BASE)
        changed[name] = new
        assert _h(changed) != h0, name


def test_committed_traffic_is_tied_to_its_kernel():
    # every committed capture names the device code it measured; bench.py
    # reports its bytes only while that code is the current one
    cur = bench._kernel_source_hash()
    for cfg in ("dense_bf16_32k", "decode_bf16_32x128k", "group_bf16_128k_refine"):
        p = os.path.join(ROOT, "profiles", f"{cfg}_traffic.txt")
        kv = dict(line.split("=", 1) for line in open(p).read().splitlines() if "=" in line and line[0] != "#")
        kv = {a.strip(): b.strip() for a, b in kv.items()}
        assert int(kv["bytes_per_launch"]) > 0 and len(kv["kernel_source"]) == 16, cfg
        t = bench._traffic(cfg)
        assert t == (int(kv["bytes_per_launch"]) if kv["kernel_source"] == cur else None), cfg


def test_no_traffic_for_a_resized_run():
    # a capture of the full-size workload says nothing about a --T run
    assert bench._traffic("dense_bf16_32k", resized=True) is None
    assert bench._traffic("no_such_workload") is None


class _FakeNvml:
    """Reads only, like the sampler: a GPU at 1500 MHz of 1965 under the power cap."""
    NVML_CLOCK_SM = 1

    def __init__(self):
        self.calls = []

    def nvmlInit(self):
        self.calls.append("init")

    def nvmlShutdown(self):
        self.calls.append("shutdown")

    def nvmlDeviceGetHandleByIndex(self, i):
        return ("gpu", i)

    def nvmlDeviceGetMaxClockInfo(self, h, kind):
        return 1965

    def nvmlDeviceGetClockInfo(self, h, kind):
        return 1500

    def nvmlDeviceGetCurrentClocksEventReasons(self, h):
        return 0x4 | 0x1   # sw_power_cap, and a bit the sampler does not report


def test_clock_sampler_against_a_fake_nvml(monkeypatch):
    fake = _FakeNvml()
    monkeypatch.setitem(sys.modules, "pynvml", fake)
    monkeypatch.delenv("CUDA_VISIBLE_DEVICES", raising=False)
    c = bench.ClockSampler(0)
    c.start()
    out = c.stop()   # a timed region shorter than one interval still has samples
    assert out["samples"] >= 1 and out["sm_mhz"] == 1500.0 and out["sm_max_mhz"] == 1965.0
    assert out["reasons"] == ["sw_power_cap"] and "error" not in out
    assert fake.calls == ["init", "shutdown"]


def test_clock_sampler_without_nvml(monkeypatch):
    monkeypatch.setitem(sys.modules, "pynvml", None)   # import fails
    c = bench.ClockSampler(0)
    c.start()
    out = c.stop()
    assert out["sm_mhz"] is None and out["samples"] == 0 and "error" in out


def test_each_rank_indexes_its_own_batch(monkeypatch):
    # weak scaling: rank r's inputs are the workload's shape from seed + r
    a = bench.Dense("cpu", size=64)
    monkeypatch.setattr(bench, "SHARD", 1)
    b = bench.Dense("cpu", size=64)
    assert a.inp.q.shape == b.inp.q.shape and not bool((a.inp.q == b.inp.q).all())
    monkeypatch.setattr(bench, "SHARD", 0)
    c = bench.Dense("cpu", size=64)
    assert bool((a.inp.q == c.inp.q).all())
