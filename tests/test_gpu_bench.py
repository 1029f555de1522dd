"""bench.py on a B200: one JSON line with the contract's keys, from a short run of
a small workload (the graph, per-call events, back-to-back timing, the end-to-end
path with its copies, the oracle as checker and as the host baseline)."""
import json
import os
import subprocess
import sys

import pytest

pytestmark = pytest.mark.gpu

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _bench(*args):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=900)
    assert r.returncode == 0, r.stderr[-3000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    assert len(lines) == 1, r.stdout[-2000:]
    return json.loads(lines[0])


def test_bench_line_carries_the_contract():
    d = _bench("--workload", "gated_4096x128_bf16", "--steps", "24", "--warmup", "3",
               "--e2e-steps", "4")
    for k in ("metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "roofline", "cpu_baseline", "e2e", "gpu_launches", "clocks", "accuracy",
              "invariance", "back_to_back"):
        assert k in d, k
    assert d["n_gpus"] == 1 and d["steps"] == 24 and d["warmup"] == 3
    assert d["unit"] == "GB/s" and d["value"] > 0 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "gated_4096x128_bf16"
    # the library's own launches: one forward, one backward and one fold pass a step
    # at 4096 rows (128 leaves in 32 warps of four)
    assert d["gpu_launches"] % 24 == 0 and d["gpu_launches"] >= 2 * 24
    rl = d["roofline"]
    assert rl["bound"] == "hbm" and rl["unit"] == "GB/s" and rl["peak"] > 0
    assert 0 < rl["frac"] == pytest.approx(rl["achieved"] / rl["peak"], rel=1e-3)
    assert rl["algorithmic_bytes"] == 4096 * (5 * 128 * 2 + 4) + 2 * 128 * 4
    assert 0 < rl["per_call"]["frac"]
    b2b = d["back_to_back"]
    assert b2b["fwd_us"] > 0 and b2b["bwd_us"] > 0
    assert rl["achieved"] == pytest.approx(rl["algorithmic_bytes"] / b2b["bwd_us"] / 1e3,
                                           rel=1e-2)
    e2e = d["e2e"]
    assert e2e["value"] > 0 and e2e["steps"] == 4
    assert e2e["h2d_bytes_per_step"] == 3 * 4096 * 128 * 2 + 128 * 4
    assert e2e["d2h_bytes_per_step"] == 3 * 4096 * 128 * 2 + 4096 * 4 + 128 * 4
    assert d["invariance"]["result"] == "pass"
    acc = d["accuracy"]
    assert acc["rows_checked"] == 4096
    for t in ("y", "dx", "dz"):
        assert acc[t]["out_of_tolerance"] == 0, (t, acc[t])
    cpu = d["cpu_baseline"]
    assert cpu["kind"] == "oracle" and cpu["value"] > 0 and cpu["cores"] >= 1
    assert d["clocks"]["sm_max_mhz"] is None or d["clocks"]["sm_max_mhz"] > 0
