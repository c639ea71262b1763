"""bench.py's command-line contract on the CPU: the reference arm (the
oracle on the host cores) prints one JSON line with the required keys."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_prints_one_json_line():
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference", "--steps", "1",
                        "--warmup", "3"], capture_output=True, text=True, timeout=600, cwd=ROOT)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [l for l in r.stdout.splitlines() if l.strip().startswith("{")]
    assert len(lines) == 1, r.stdout[-2000:]
    d = json.loads(lines[0])
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step", "higher_is_better",
              "scaling", "vs_baseline", "dtype", "data", "config", "impl", "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["steps"] == 1 and d["warmup"] == 3
    assert d["config"]["workload"] == "llama31_8b_linears_b1"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0
    assert d["value"] > 0 and d["unit"] == "GB/s"


def test_committed_dram_traffic_matches_the_kernel_sources():
    """profiles/gemv_dram_traffic.txt was captured on the current kernel
    sources (its hash matches), so the bench's roofline carries a traffic
    figure, and that figure is the byte model up to the few KB of y."""
    sys.path.insert(0, ROOT)
    import bench
    traffic, kernel = bench._ncu_traffic()
    assert traffic is not None, "kernel sources changed since the committed ncu traffic capture"
    kv = {}
    for line in open(os.path.join(ROOT, "profiles", "gemv_dram_traffic.txt")):
        if line.strip() and not line.startswith("#") and " " in line:
            k, v = line.split(None, 1)
            kv[k] = v.strip()
    alg = float(kv["algorithmic_bytes"])
    assert traffic == float(kv["dram_bytes_read"]) + float(kv["dram_bytes_write"])
    assert alg <= traffic <= 1.01 * alg


def test_roofline_kernel_name_follows_the_kernel_choice():
    sys.path.insert(0, ROOT)
    import bench
    # every launch of the default step has K <= 30720: the single-vector kernel
    for key in ("qkv@p2", "o@p3", "gate_up@p4", "down@p4"):
        assert bench._launch_kernel(key) == "gemv1_kernel"
