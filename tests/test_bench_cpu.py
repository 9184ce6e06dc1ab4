"""bench.py's host-side parts on CPU: the reference arm (the fp64 oracle timed on the
host cores) and the fit that turns the sparsity sweep into a throughput on flagged blocks."""
import json
import os
import subprocess
import sys

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
sys.path.insert(0, ROOT)


def _run(args, env_extra=None):
    env = dict(os.environ)
    env.update(env_extra or {})
    return subprocess.run([sys.executable, os.path.join(ROOT, "bench.py"), *args], capture_output=True, text=True,
                          env=env, timeout=600, cwd=ROOT)


def test_reference_arm_prints_one_line():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "1"])
    assert r.returncode == 0, r.stderr[-2000:]
    lines = [ln for ln in r.stdout.splitlines() if ln.startswith("{")]
    assert len(lines) == 1
    out = json.loads(lines[0])
    assert out["impl"] == "reference" and out["value"] > 0 and out["unit"] == "tokens/s"
    assert out["cpu_baseline"]["kind"] == "oracle" and out["cpu_baseline"]["cores"] >= 1
    assert out["e2e"]["h2d_bytes_per_step"] == 0 and out["e2e"]["d2h_bytes_per_step"] == 0
    assert out["config"]["workload"] == "long_causal_L8192"


def test_reference_arm_is_silent_on_other_ranks():
    r = _run(["--impl", "reference", "--steps", "1", "--warmup", "1"], {"RANK": "1"})
    assert r.returncode == 0 and r.stdout.strip() == ""


def test_marginal_throughput_recovers_the_slope():
    import bench

    # time = 0.2 ms + flops / (500 TFLOP/s), for five sparsity levels
    pts = []
    for flagged in (24000, 12000, 6000, 3000, 1500):
        s_tiles = 24960 + 2 * flagged
        fl = bench.UNIT_FLOP * (s_tiles + 2 * flagged)
        bl = bench.UNIT_FLOP * 5 * flagged
        f_ms = 0.2 + fl / 500e12 * 1e3
        b_ms = 0.05 + bl / 600e12 * 1e3
        pts.append({"s_tiles": s_tiles, "flagged_tiles": flagged, "fwd_ms": f_ms, "bwd_ms": b_ms, "ms": f_ms + b_ms})
    m = bench.marginal_throughput(pts)
    assert m["fwd"]["tflops_on_flagged_blocks"] == pytest.approx(500.0, rel=1e-6)
    assert m["bwd"]["tflops_on_flagged_blocks"] == pytest.approx(600.0, rel=1e-6)
    assert m["fwd"]["intercept_ms"] == pytest.approx(0.2, abs=1e-9)
