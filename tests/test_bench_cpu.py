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
        fl = bench.UNIT_FLOP * (s_tiles + flagged)
        bl = bench.UNIT_FLOP * 5 * flagged
        f_ms = 0.2 + fl / 500e12 * 1e3
        b_ms = 0.05 + bl / 600e12 * 1e3
        pts.append({"s_tiles": s_tiles, "flagged_tiles": flagged, "fwd_ms": f_ms, "bwd_ms": b_ms, "ms": f_ms + b_ms})
    m = bench.marginal_throughput(pts)
    assert m["fwd"]["tflops_on_flagged_blocks"] == pytest.approx(500.0, rel=1e-6)
    assert m["bwd"]["tflops_on_flagged_blocks"] == pytest.approx(600.0, rel=1e-6)
    assert m["fwd"]["intercept_ms"] == pytest.approx(0.2, abs=1e-9)


def test_reference_arm_is_self_consistent():
    """The reference line's config equals the GPU arm's, and ms_per_step x steps is time the
    run actually spent (each step is one measured oracle head)."""
    import bench
    from entmax_sm_attention_b200.workloads import WORKLOADS

    import time
    t0 = time.perf_counter()
    r = _run(["--impl", "reference", "--steps", "2", "--warmup", "1"])
    wall = time.perf_counter() - t0
    assert r.returncode == 0, r.stderr[-2000:]
    out = json.loads([ln for ln in r.stdout.splitlines() if ln.startswith("{")][0])
    w = WORKLOADS["long_causal_L8192"]
    assert out["config"] == bench.bench_config(w, 1.5, 0, 1)
    assert out["ms_per_step"] * out["steps"] / 1e3 < wall
    tokens = out["value"] * out["ms_per_step"] / 1e3
    assert tokens == pytest.approx(w.B * w.L / (w.B * w.H), rel=1e-9)


def test_pair_work_matches_brute_force():
    """pair_work counts active pairs, pairs in flagged blocks and the per-pair flop
    formulas; checked against a dense count on small causal / window / padded shapes."""
    import numpy as np
    import torch

    import bench
    from entmax_sm_attention_b200.workloads import small_case

    rng = np.random.default_rng(0)
    for w in (small_case("c", B=2, H=3, L=300, causal=True), small_case("wd", B=1, H=2, L=400, window=32),
              small_case("pad", B=2, H=1, L=260, kv_len=130)):
        T = -(-w.L // 128)
        W = -(-T // 32)
        bits = rng.random((w.B, w.H, T, T)) < 0.6
        words = np.zeros((w.B, w.H, T, W), np.uint32)
        for jt in range(T):
            words[..., jt // 32] |= bits[..., jt].astype(np.uint32) << np.uint32(jt % 32)
        R = rng.integers(1, 4, size=(w.B, w.H, T))
        st = np.zeros((w.B, w.H, T, 8), np.int32)
        st[..., 0] = R
        got = bench.pair_work(w, torch.from_numpy(words.view(np.int32)), torch.from_numpy(st))
        i = np.arange(w.L)[:, None]
        j = np.arange(w.L)[None, :]
        fwd = bwd = act_total = fl_total = 0
        for b in range(w.B):
            kv = w.L if w.kv_len is None else w.kv_len
            act = (j < kv) & np.ones((w.L, w.L), bool)
            if w.window >= 0:
                act &= (j <= i) & ((j == 0) | (i - j <= w.window))
            elif w.causal:
                act &= j <= i
            for h in range(w.H):
                blk = bits[b, h][i // 128, j // 128]
                a_i = act.sum(1)
                f_i = (act & blk).sum(1)
                r_i = R[b, h][np.arange(w.L) // 128]
                fwd += int(((1 + r_i) * a_i).sum() * 128 + 2 * f_i.sum() * 128)
                bwd += int(5 * f_i.sum() * 128)
                act_total += int(a_i.sum())
                fl_total += int(f_i.sum())
        assert got == {"fwd_flops": fwd, "bwd_flops": bwd, "active_pairs": act_total, "flagged_pairs": fl_total}
