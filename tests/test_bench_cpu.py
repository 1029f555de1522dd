"""bench.py's reference arm on the CPU: one JSON line with the contract's keys
(the fp64 oracle timed on the host; no GPU involved)."""
import json
import os
import subprocess
import sys

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))


def _run(*args, env=None):
    r = subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], cwd=ROOT,
                       capture_output=True, text=True, timeout=600, env=env)
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.strip()]
    return lines


def test_reference_arm_prints_one_contract_line():
    lines = _run("--impl", "reference", "--steps", "2", "--warmup", "1",
                 "--workload", "norm_64x128_f32")
    assert len(lines) == 1
    d = json.loads(lines[0])
    for k in ("impl", "metric", "value", "unit", "n_gpus", "steps", "warmup", "ms_per_step",
              "higher_is_better", "scaling", "vs_baseline", "dtype", "data", "config",
              "cpu_baseline", "e2e"):
        assert k in d, k
    assert d["impl"] == "reference" and d["unit"] == "GB/s" and d["value"] > 0
    assert d["steps"] == 2 and d["warmup"] == 1 and d["higher_is_better"] is True
    assert d["config"]["workload"] == "norm_64x128_f32"
    assert d["cpu_baseline"]["kind"] == "oracle" and d["cpu_baseline"]["value"] == d["value"]
    host = d["cpu_baseline"]["host"]
    assert host["nproc"] >= 1 and host["cpu_model"]
    assert d["cpu_baseline"]["cores"] == host["nproc"]        # one worker per core
    assert d["e2e"]["h2d_bytes_per_step"] == 0 and d["e2e"]["d2h_bytes_per_step"] == 0


def test_reference_arm_on_non_zero_ranks_prints_nothing():
    env = dict(os.environ, RANK="1", WORLD_SIZE="2")
    assert _run("--impl", "reference", "--steps", "1", "--warmup", "0", env=env) == []


def test_oracle_pool_matches_one_process():
    """The all-cores oracle splits rows into blocks; the per-block dw add up to
    the one-process oracle's dw (fp64, up to summation order)."""
    import numpy as np
    sys.path.insert(0, ROOT)
    import bench
    import oracle
    from rollout_parity_b200 import workloads
    wl = workloads.make("gated", 300, 64, "bf16", seed=3)
    pool = bench.OraclePool(wl, 300, procs=3)
    try:
        parts = pool.pass_()
    finally:
        pool.close()
    assert len(parts) == 3
    f = workloads.as_f64
    _, _, want = oracle.gated_norm_bwd(f(wl.x), f(wl.z), f(wl.w), f(wl.dy), wl.eps)
    assert np.allclose(np.sum(parts, axis=0), want, rtol=1e-12, atol=1e-12)
