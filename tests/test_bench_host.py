"""Host-side checks of bench.py that need no GPU: the reference arm's JSON line (the
CPU oracle timed on this host) reports what it timed, with the GPU arm's config."""
import json
import os
import subprocess
import sys
import time

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def test_reference_arm_line_is_consistent():
    sys.path.insert(0, ROOT)
    import bench
    from quantized_kv_cache_22_b200.inputs import WORKLOADS
    steps, warmup = 2, 3
    t0 = time.perf_counter()
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), "--impl", "reference",
                        "--steps", str(steps), "--warmup", str(warmup)],
                       capture_output=True, text=True, timeout=600,
                       env=dict(os.environ, RANK="0", WORLD_SIZE="1", LOCAL_RANK="0"))
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr
    line = json.loads(r.stdout.strip().splitlines()[-1])
    assert line["impl"] == "reference"
    # the same config dict as the GPU arm's line
    assert line["config"] == bench.bench_config(WORKLOADS[4], "K8V8", 1)
    # the timed steps fit inside the process's own wall time
    assert line["ms_per_step"] * (steps + warmup) / 1e3 < wall
    # value = the timed layer's KV bytes / its time
    per_layer = 2080 * 16 * 8192
    assert abs(line["value"] - per_layer / (line["ms_per_step"] * 1e-3) / 1e9) <= 1e-3 * line["value"]
    assert line["cpu_baseline"]["kind"] == "oracle" and line["cpu_baseline"]["cores"] >= 1
    assert line["e2e"]["h2d_bytes_per_step"] == 0
