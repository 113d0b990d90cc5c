"""bench.py's reference arm (the CPU oracle, as it stands) prints the
contract's JSON line on a machine without a GPU, and other ranks print
nothing."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(env_extra):
    env = dict(os.environ, **env_extra)
    r = subprocess.run([sys.executable, "bench.py", "--impl", "reference", "--steps", "1", "--warmup", "3"],
                       cwd=ROOT, env=env, capture_output=True, text=True, timeout=600)
    assert r.returncode == 0, r.stderr[-2000:]
    return r.stdout.strip()


def test_reference_line():
    j = json.loads(_run({}).splitlines()[-1])
    assert j["impl"] == "reference" and j["unit"] == "Gpairs/s" and j["value"] > 0
    assert j["higher_is_better"] is True and j["steps"] == 1 and j["warmup"] == 3
    assert j["cpu_baseline"]["kind"] == "oracle" and j["cpu_baseline"]["cores"] >= 1
    assert j["cpu_baseline"]["value"] == j["value"]
    assert j["e2e"] == {"value": j["value"], "unit": j["unit"], "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}
    assert j["config"]["workload"].startswith("dense_bf16_32k")


def test_reference_other_ranks_print_nothing():
    assert _run({"RANK": "1", "WORLD_SIZE": "2"}) == ""
