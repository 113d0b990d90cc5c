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


def test_committed_traffic_matches_the_current_kernel():
    # the committed captures were taken on the current device code
    for cfg in ("dense_bf16_32k", "decode_bf16_32x128k", "group_bf16_128k_refine"):
        assert bench._traffic(cfg) is not None, cfg


def test_no_traffic_for_a_resized_run():
    # a capture of the full-size workload says nothing about a --T run
    assert bench._traffic("dense_bf16_32k", resized=True) is None
    assert bench._traffic("no_such_workload") is None
