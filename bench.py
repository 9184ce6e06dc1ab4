#!/usr/bin/env python
"""Throughput of fused alpha-entmax attention (forward + backward) on B200.

One step is one forward + backward pass over one batch of the long-context causal
workload: B=1, H=12, L=8192, d=64, bf16, alpha=1.5, with Q ~ N(0, 3^2) (the query
variance knob of AdaSplash-2 §4.2). Prints one JSON line.

  python bench.py [--gpus N] [--steps K] [--warmup W] [--impl ours|reference] [--alpha A]

With N > 1 (under torchrun) every rank runs its own batch with no data-path
collective (weak scaling). Only the timing uses a barrier and a max-reduce.
--impl reference times the fp64 CPU oracle on the host cores, on a bounded sample
of the same workload.
"""
from __future__ import annotations

import argparse
import json
import math
import os
import statistics
import subprocess
import sys
import threading
import time

ROOT = os.path.dirname(os.path.abspath(__file__))
sys.path.insert(0, ROOT)

METRIC = "fwd+bwd tokens/s & TFLOP/s at L=8192 vs tensor-core roofline, 1×B200"
UNIT = "tokens/s"
TILE = 128
UNIT_FLOP = 2 * TILE * TILE * 64      # one 128x128x64 (or 128x64x128) bf16 tile product
L2_BYTES = 126 * 1024 * 1024


def parse():
    ap = argparse.ArgumentParser()
    ap.add_argument("--gpus", type=int, default=1)
    ap.add_argument("--steps", type=int, default=200)
    ap.add_argument("--warmup", type=int, default=3)
    ap.add_argument("--impl", choices=["ours", "reference"], default="ours")
    ap.add_argument("--workload", default="long_causal_L8192")
    ap.add_argument("--alpha", type=float, default=1.5)
    ap.add_argument("--seed", type=int, default=0)
    ap.add_argument("--no-cpu-baseline", action="store_true")
    ap.add_argument("--cpu-seconds", type=float, default=10.0, help="target CPU-oracle sample time")
    ap.add_argument("--no-sweeps", action="store_true", help="skip the block-sparsity sweeps")
    return ap.parse_args()


def ncu_traffic(kernel: str, workload: str, alpha: float):
    """DRAM bytes per launch of `kernel` from the committed ncu summary, or None when the
    kernel source has changed since that capture (or no capture exists)."""
    import hashlib

    path = os.path.join(ROOT, "profiles", "traffic_per_launch.txt")
    if not os.path.exists(path):
        return None
    with open(path) as f:
        rec = json.load(f).get(kernel)
    if not rec or rec.get("workload") != workload or rec.get("alpha") != alpha:
        return None
    with open(os.path.join(ROOT, rec["source"]), "rb") as f:
        if hashlib.sha256(f.read()).hexdigest()[:16] != rec["sha256_16"]:
            return None
    return rec["bytes_per_launch"]


def load_peaks():
    path = os.path.join(ROOT, "MEASURED_PEAKS.json")
    if os.path.exists(path):
        with open(path) as f:
            p = json.load(f)
        return {"hbm_gbs": p["hbm_gbs"], "bf16_tflops": p["bf16_tflops"],
                "bf16_tflops_sustained": p.get("bf16_tflops_sustained", p["bf16_tflops"]), "source": "measured"}
    return {"hbm_gbs": 6650.0, "bf16_tflops": 1590.0, "bf16_tflops_sustained": 1400.0, "source": "fallback"}


# ------------------------------------------------------------ multi-rank plumbing
def rank_seed(seed: int, rank: int) -> int:
    """Seed of a rank's batch: every rank works on its own independent batch."""
    return seed + rank


def max_over_ranks(x: float, world: int, device) -> float:
    """The slowest rank's value (timings are taken as the max over ranks)."""
    import torch
    import torch.distributed as dist

    t = torch.tensor([x], dtype=torch.float64, device=device)
    if world > 1:
        dist.all_reduce(t, op=dist.ReduceOp.MAX)
    return float(t.item())


def job_throughput(world: int, tokens_per_step: int, steps: int, max_ms: float) -> float:
    """Whole-job tokens/s: the tokens all ranks processed over the slowest rank's time."""
    return world * tokens_per_step * steps / (max_ms / 1e3)


# ------------------------------------------------------------------ clock sampling
class ClockSampler:
    """nvidia-smi samples of SM clock and throttle reasons while the timed region runs."""
    FIELDS = ("clocks.sm,clocks.max.sm,power.draw,clocks_event_reasons.hw_slowdown,"
              "clocks_event_reasons.hw_thermal_slowdown,clocks_event_reasons.sw_thermal_slowdown,"
              "clocks_event_reasons.sw_power_cap")

    def __init__(self, gpu_index: int):
        self.gpu = gpu_index
        self.proc = None
        self.lines: list[str] = []

    def start(self):
        try:
            self.proc = subprocess.Popen(
                ["nvidia-smi", "-i", str(self.gpu), f"--query-gpu={self.FIELDS}", "--format=csv,noheader,nounits",
                 "-lms", "100"], stdout=subprocess.PIPE, stderr=subprocess.DEVNULL, text=True)
            self.thread = threading.Thread(target=self._read, daemon=True)
            self.thread.start()
        except (OSError, FileNotFoundError):
            self.proc = None

    def _read(self):
        for line in self.proc.stdout:
            self.lines.append(line.strip())

    def stop(self) -> dict:
        if self.proc is None:
            return {"sm_mhz": None, "sm_max_mhz": None, "reasons": ["nvidia-smi unavailable"]}
        self.proc.terminate()
        try:
            self.proc.wait(timeout=5)
        except subprocess.TimeoutExpired:
            self.proc.kill()
        self.thread.join(timeout=2)
        sm, mx, reasons = [], [], set()
        names = ["hw_slowdown", "hw_thermal_slowdown", "sw_thermal_slowdown", "sw_power_cap"]
        for ln in self.lines:
            parts = [p.strip() for p in ln.split(",")]
            if len(parts) < 7:
                continue
            try:
                sm.append(float(parts[0]))
                mx.append(float(parts[1]))
            except ValueError:
                continue
            for n, v in zip(names, parts[3:7]):
                if v.lower().startswith("active"):
                    reasons.add(n)
        return {"sm_mhz": statistics.median(sm) if sm else None, "sm_max_mhz": max(mx) if mx else None,
                "reasons": sorted(reasons), "samples": len(sm)}


# ------------------------------------------------------------------------ CPU oracle
def cpu_oracle_sample(w, alpha: float, seed: int, target_s: float, inp=None):
    """Times the fp64 oracle (as it stands) on whole heads of the workload, drawn with the
    GPU arm's seed (the same bytes the GPU arm computes on): forward and backward of head
    (0, 0), (0, 1), ... until target_s has passed. Returns tokens/s scaled to the full
    batch (heads done / (B*H) of B*L tokens), the thread count, a description, the oracle
    block sparsity of the first head, and the seconds per head."""
    import oracle
    from entmax_sm_attention_b200.workloads import make_inputs

    if inp is None:
        inp = make_inputs(w, seed)
    heads, t_total = 0, 0.0
    sparsity = None
    while heads < w.B * w.H and (heads == 0 or t_total < target_s):
        b, h = divmod(heads, w.H)
        one = {k: v[b:b + 1, h:h + 1] for k, v in inp.items()}
        pr = oracle.Problem(one["Q"], one["K"], one["V"], one["dO"], alpha=alpha, scale=w.scale,
                            causal=w.causal, window=w.window,
                            kv_len=None if w.kv_len is None else [w.kv_len])
        t0 = time.perf_counter()
        r = pr.rows(backward=True)
        pr.cols(r["tau"], r["delta"])
        t_total += time.perf_counter() - t0
        if heads == 0:
            sparsity = oracle_block_sparsity(pr, r["tau"], w)
        heads += 1
    tokens = w.B * w.L * heads / (w.B * w.H)
    return tokens / t_total, oracle.max_threads(), (
        f"{heads} of {w.B * w.H} heads (b,h) of {w.name} (seed {seed}, the GPU arm's inputs), full fwd+bwd "
        f"per head in fp64; tokens/s = heads/(B*H) * B*L / seconds"), sparsity, t_total / heads


def oracle_block_sparsity(pr, tau, w) -> dict:
    """Block sparsity of one head from the fp64 oracle, at the kernel's 128 x 128 blocks and
    at the 64 x 64 blocks of AdaSplash-2 Fig. 7: the share of structurally active blocks
    with no nonzero weight (causal workloads without padding or window)."""
    import numpy as np

    out = {}
    for blk in (128, 64):
        M, _, _ = pr.block_mask(tau, blk, blk)
        flagged = int(np.unpackbits(M.view(np.uint8)).sum())
        T = -(-w.L // blk)
        active = T * (T + 1) // 2 if w.causal else T * T
        out[f"{blk}x{blk}"] = 1.0 - flagged / active
    return out


def bench_config(w, alpha: float, seed: int, world: int) -> dict:
    """The `config` object of both arms' JSON lines (the same workload, same keys)."""
    return {"workload": w.name, "B": w.B, "H": w.H, "L": w.L, "d": w.d, "alpha": alpha,
            "causal": w.causal, "window": w.window, "kv_len": w.kv_len, "sigma_q": w.sigma_q,
            "seed": seed, "l2": "flushed (256 MB write) before every timed GPU step",
            "parallelism": f"replica x{world} (independent batches)"}


def run_reference(args):
    """--impl reference: the oracle on the host cores. Step k computes forward + backward
    of head k mod (B*H) of the GPU arm's own inputs (same seed); ms_per_step is the measured
    mean time of one such step, and value is the workload's tokens/s at that rate."""
    rank = int(os.environ.get("RANK", "0"))
    if rank != 0:
        return
    from entmax_sm_attention_b200.workloads import WORKLOADS, make_inputs

    w = WORKLOADS[args.workload]
    inp = make_inputs(w, args.seed)
    import oracle

    secs = []
    for k in range(args.warmup + args.steps):
        b, h = divmod(k % (w.B * w.H), w.H)
        one = {n: v[b:b + 1, h:h + 1] for n, v in inp.items()}
        pr = oracle.Problem(one["Q"], one["K"], one["V"], one["dO"], alpha=args.alpha, scale=w.scale,
                            causal=w.causal, window=w.window, kv_len=None if w.kv_len is None else [w.kv_len])
        t0 = time.perf_counter()
        r = pr.rows(backward=True)
        pr.cols(r["tau"], r["delta"])
        if k >= args.warmup:
            secs.append(time.perf_counter() - t0)
    ms_per_step = statistics.mean(secs) * 1e3
    tokens_per_step = w.B * w.L / (w.B * w.H)      # one head's share of the batch
    value = tokens_per_step / (ms_per_step * 1e-3)
    cores = oracle.max_threads()
    sample = (f"each step = full fwd+bwd in fp64 of one (b,h) head of {w.name} (head k mod {w.B * w.H}, "
              f"seed {args.seed}: the GPU arm's inputs); tokens/s = (B*L/(B*H)) / seconds per step")
    out = {"metric": METRIC, "value": value, "unit": UNIT, "n_gpus": args.gpus, "steps": args.steps,
           "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
           "vs_baseline": None, "dtype": "f64", "data": "synthetic", "impl": "reference",
           "config": bench_config(w, args.alpha, args.seed, args.gpus),
           "cpu_baseline": {"value": value, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample},
           "e2e": {"value": value, "unit": UNIT, "h2d_bytes_per_step": 0, "d2h_bytes_per_step": 0}}
    print(json.dumps(out), flush=True)


# ------------------------------------------------------------------------ GPU arm
def run_ours(args):
    import torch
    import torch.distributed as dist

    from entmax_sm_attention_b200 import binding as eb
    from entmax_sm_attention_b200.workloads import WORKLOADS, make_inputs

    world = int(os.environ.get("WORLD_SIZE", "1"))
    rank = int(os.environ.get("RANK", "0"))
    local = int(os.environ.get("LOCAL_RANK", "0"))
    if world > 1:
        from datetime import timedelta

        dist.init_process_group("nccl", timeout=timedelta(seconds=120))
    torch.cuda.set_device(local)
    dev = torch.device("cuda", local)
    w = WORKLOADS[args.workload]
    alpha = args.alpha

    host = make_inputs(w, seed=rank_seed(args.seed, rank))
    pinned = {k: v.pin_memory() for k, v in host.items()}
    d = {k: v.to(dev) for k, v in host.items()}
    kv = None if w.kv_len is None else torch.tensor(w.kv_len_list(), dtype=torch.int32, device=dev)
    desc = eb.make_desc(w.B, w.H, w.L, w.d, alpha=alpha, scale=w.scale, causal=w.causal, window=w.window,
                        kv_len=kv, dtype=eb.ENTMAX_BF16)
    ws = eb.alloc_workspace(desc, dev)
    shp = (w.B, w.H, w.L, w.d)
    O = torch.empty(shp, dtype=torch.float32, device=dev)
    tau = torch.empty(shp[:3], dtype=torch.float32, device=dev)
    dQ, dK, dV = (torch.empty(shp, dtype=torch.float32, device=dev) for _ in range(3))
    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)

    def step(src):
        eb.entmax_attn_fwd(desc, src["Q"], src["K"], src["V"], O, tau, ws, stream)
        eb.entmax_attn_bwd(desc, src["Q"], src["K"], src["V"], src["dO"], tau, ws, dQ, dK, dV, stream)

    def barrier():
        if world > 1:
            dist.barrier()

    for _ in range(args.warmup):
        step(d)
    torch.cuda.synchronize(dev)
    code, word = eb.entmax_last_device_status(desc, ws, stream)
    if code != eb.ENTMAX_OK:
        raise SystemExit(f"device status {eb.STATUS_NAMES[code]} (word {word}) after warm-up")

    # ---- device-timed region: inputs resident in HBM, L2 flushed before every step
    ev = [[torch.cuda.Event(enable_timing=True) for _ in range(3)] for _ in range(args.steps)]
    clocks = ClockSampler(local)
    clocks.start()
    time.sleep(0.3)
    barrier()
    torch.cuda.synchronize(dev)
    for k in range(args.steps):
        flush.zero_()
        ev[k][0].record(stream)
        eb.entmax_attn_fwd(desc, d["Q"], d["K"], d["V"], O, tau, ws, stream)
        ev[k][1].record(stream)
        eb.entmax_attn_bwd(desc, d["Q"], d["K"], d["V"], d["dO"], tau, ws, dQ, dK, dV, stream)
        ev[k][2].record(stream)
    torch.cuda.synchronize(dev)
    barrier()
    clk = clocks.stop()
    fwd_ms = [e[0].elapsed_time(e[1]) for e in ev]
    bwd_ms = [e[1].elapsed_time(e[2]) for e in ev]
    total_ms = max_over_ranks(sum(fwd_ms) + sum(bwd_ms), world, dev)
    ms_per_step = total_ms / args.steps
    tokens_per_step = w.B * w.L
    value = job_throughput(world, tokens_per_step, args.steps, total_ms)

    # ---- end to end through the public API: pinned host -> device, fwd+bwd, device -> host.
    # Every step copies its inputs in and its results out. The copies run on their own
    # streams with two buffer sets, so step k's kernels overlap step k+1's upload and step
    # k-1's download (as a training loop would pipeline them); events order each buffer
    # set's reuse. The time runs from the first upload to the last download.
    out_host = [{k: torch.empty(shp, dtype=torch.float32).pin_memory() for k in ("O", "dQ", "dK", "dV")}
                for _ in range(2)]
    h2d = sum(v.numel() * v.element_size() for v in pinned.values())
    d2h = sum(v.numel() * v.element_size() for v in out_host[0].values())
    s_in, s_out = torch.cuda.Stream(dev), torch.cuda.Stream(dev)
    din = [d, {k: torch.empty_like(v) for k, v in d.items()}]
    dout = [{"O": O, "dQ": dQ, "dK": dK, "dV": dV},
            {k: torch.empty(shp, dtype=torch.float32, device=dev) for k in ("O", "dQ", "dK", "dV")}]
    tau2 = [tau, torch.empty_like(tau)]
    ws2 = [ws, eb.alloc_workspace(desc, dev)]
    ev = lambda: torch.cuda.Event()  # noqa: E731
    in_ready, computed, out_done = [ev(), ev()], [ev(), ev()], [ev(), ev()]
    e0, e1 = torch.cuda.Event(enable_timing=True), torch.cuda.Event(enable_timing=True)
    barrier()
    torch.cuda.synchronize(dev)
    e0.record(s_in)
    for k in range(args.steps):
        b = k % 2
        if k >= 2:
            s_in.wait_event(computed[b])         # the kernels of step k-2 are done with din[b]
        with torch.cuda.stream(s_in):
            for n in ("Q", "K", "V", "dO"):
                din[b][n].copy_(pinned[n], non_blocking=True)
        in_ready[b].record(s_in)
        stream.wait_event(in_ready[b])
        if k >= 2:
            stream.wait_event(out_done[b])       # step k-2's results have left dout[b]
        src, dst = din[b], dout[b]
        eb.entmax_attn_fwd(desc, src["Q"], src["K"], src["V"], dst["O"], tau2[b], ws2[b], stream)
        eb.entmax_attn_bwd(desc, src["Q"], src["K"], src["V"], src["dO"], tau2[b], ws2[b], dst["dQ"], dst["dK"],
                           dst["dV"], stream)
        computed[b].record(stream)
        s_out.wait_event(computed[b])
        with torch.cuda.stream(s_out):
            for n in ("O", "dQ", "dK", "dV"):
                out_host[b][n].copy_(dst[n], non_blocking=True)
        out_done[b].record(s_out)
    e1.record(s_out)
    torch.cuda.synchronize(dev)
    e2e_value = job_throughput(world, tokens_per_step, args.steps,
                               max_over_ranks(e0.elapsed_time(e1), world, dev))
    code2, _ = eb.entmax_last_device_status(desc, ws2[1], stream)
    if code2 != eb.ENTMAX_OK:
        raise SystemExit(f"device status {eb.STATUS_NAMES[code2]} in the end-to-end run")

    # ---- work actually done (per-tile counters written by the forward and the backward)
    M, st = eb.block_mask((desc, ws))
    bst = eb.bwd_counters((desc, ws)).cpu().long()
    st = st.cpu().long()
    n_sweeps, n_s, n_out, n_act = (st[..., c] for c in range(4))
    s_tiles, out_tiles, act_tiles = int(n_s.sum()), int(n_out.sum()), int(n_act.sum())
    work = pair_work(w, M.cpu(), st)
    # Algorithmic tensor work (the scope table's per-pair figures): forward
    # (1+R) 2d |A_i| + 2 2d |F_i| summed over rows (max pass and R refinement passes over
    # the active keys; S and A V over the keys of flagged tiles: delta's g V term is not a
    # tensor product here, the backward's delta kernel sums it over the support lists),
    # backward 5 2d |F_i| (S, dA, dV, dK, dQ). R is each query tile's measured count.
    fwd_flops = work["fwd_flops"]
    bwd_flops = work["bwd_flops"]
    # The same at tile granularity (every 128x128 block counted whole, diagonal blocks
    # included), and the work the tensor cores are issued (dS enters dK and dQ as two
    # bf16 terms, hi + lo).
    fwd_tile_flops = UNIT_FLOP * (s_tiles + out_tiles)
    bwd_tile_flops = UNIT_FLOP * 5 * out_tiles
    fwd_issued = fwd_tile_flops
    bwd_issued = UNIT_FLOP * 7 * out_tiles
    fwd_avg, bwd_avg = statistics.mean(fwd_ms), statistics.mean(bwd_ms)
    peaks = load_peaks()
    # Each kernel runs for about half a millisecond inside a ~1 ms step: the burst peak
    # (cuBLAS timed alone) is its denominator, not the seconds-long sustained figure.
    peak = peaks["bf16_tflops"]
    dom = "bwd" if bwd_avg >= fwd_avg else "fwd"
    dom_ms = bwd_avg if dom == "bwd" else fwd_avg
    dom_flops = bwd_flops if dom == "bwd" else fwd_flops
    achieved = dom_flops / (dom_ms * 1e-3) / 1e12
    total_tflops = (fwd_flops + bwd_flops) / (ms_per_step * 1e-3) / 1e12
    phases = phase_shares(st, bst)
    # The threshold and mask passes (max pass, refinement, decision) read Q and K once per
    # head from HBM (2 B per element) and write tau (4 B per row) and the two masks.
    tm_bytes = 2 * 2 * w.B * w.H * w.L * w.d + 4 * w.B * w.H * w.L + 2 * M.numel() * 4
    tm_ms = fwd_avg * (phases["fwd"]["max_pass"] + phases["fwd"]["refine_and_mask"])
    # Softmax-equivalent work over structurally active pairs (4d fwd, 10d bwd per pair).
    pairs = act_pairs(w)
    sm_eq = (4 + 10) * w.d * pairs / (ms_per_step * 1e-3) / 1e12

    result = {
        "metric": METRIC, "value": value, "unit": UNIT, "n_gpus": world, "steps": args.steps,
        "warmup": args.warmup, "ms_per_step": ms_per_step, "higher_is_better": True, "scaling": "weak",
        "vs_baseline": None, "dtype": "bf16", "data": "synthetic",
        "config": bench_config(w, alpha, args.seed, world),
        "roofline": {"bound": "tensor",
                     "kernel": f"entmax {dom} (algorithmic bf16 work over active / flagged pairs)",
                     "achieved": achieved, "peak": peak, "unit": "TFLOP/s", "frac": achieved / peak,
                     "peak_source": f"{peaks['source']} bf16 burst (cuBLAS timed alone; of measured)",
                     "traffic": ncu_traffic(dom, w.name, alpha),
                     "traffic_unit": "bytes per launch (ncu dram read+write; null if the kernel changed)"},
        "clocks": clk,
        # per step: V -> fp16 copy, forward, dO -> fp16 copy, delta, backward
        "gpu_launches": 5 * args.steps,
        "e2e": {"value": e2e_value, "unit": UNIT, "h2d_bytes_per_step": h2d, "d2h_bytes_per_step": d2h},
        "detail": {
            "fwd_ms": fwd_avg, "bwd_ms": bwd_avg,
            "tflops_total_algorithmic": total_tflops,
            "tflops_fwd_algorithmic": fwd_flops / (fwd_avg * 1e-3) / 1e12,
            "tflops_bwd_algorithmic": bwd_flops / (bwd_avg * 1e-3) / 1e12,
            "fwd_flops_pairs": fwd_flops, "bwd_flops_pairs": bwd_flops,
            "fwd_flops_tiles": fwd_tile_flops, "bwd_flops_tiles": bwd_tile_flops,
            "tflops_fwd_tiles": fwd_tile_flops / (fwd_avg * 1e-3) / 1e12,
            "tflops_bwd_tiles": bwd_tile_flops / (bwd_avg * 1e-3) / 1e12,
            "frac_fwd_of_burst": fwd_flops / (fwd_avg * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "frac_bwd_of_burst": bwd_flops / (bwd_avg * 1e-3) / 1e12 / peaks["bf16_tflops"],
            "tflops_fwd_issued": fwd_issued / (fwd_avg * 1e-3) / 1e12,
            "tflops_bwd_issued": bwd_issued / (bwd_avg * 1e-3) / 1e12,
            "active_pairs": work["active_pairs"], "flagged_pairs": work["flagged_pairs"],
            "phase_cycle_shares": phases,
            "tau_mask_passes": {"ms_equiv": tm_ms, "algorithmic_bytes": tm_bytes,
                                "hbm_gbs": tm_bytes / (tm_ms * 1e-3) / 1e9 if tm_ms > 0 else None,
                                "note": "time = forward time x the max-pass and refinement cycle shares"},
            "softmax_equiv_tflops": sm_eq,
            "block_sparsity_128": 1.0 - out_tiles / max(1, act_tiles),
            "refine_sweeps_mean": float(n_sweeps.float().mean()), "refine_sweeps_max": int(n_sweeps.max()),
            "s_tiles": s_tiles, "flagged_tiles": out_tiles, "active_tiles": act_tiles,
            "memsets_per_step": 3,
        },
    }
    if rank == 0 and world == 1 and not args.no_sweeps:
        result["detail"]["sparsity_sweeps"] = sparsity_sweeps(w, alpha, dev)
        result["detail"]["variants"] = variant_points(w, dev)
    if rank == 0 and world == 1 and not args.no_cpu_baseline:
        v, cores, sample, osp, _ = cpu_oracle_sample(w, alpha, args.seed, args.cpu_seconds, inp=host)
        result["cpu_baseline"] = {"value": v, "unit": UNIT, "cores": cores, "kind": "oracle", "sample": sample}
        if osp is not None and w.window < 0 and w.kv_len is None:
            result["detail"]["block_sparsity_oracle_head0"] = osp
    if rank == 0:
        print(json.dumps(result), flush=True)
    if world > 1:
        dist.destroy_process_group()


def sparsity_sweeps(w, alpha, dev, steps: int = 10):
    """Wall time against measured block sparsity on the same shape as the timed workload.
    (a) planted block structure with rho in {1, 1/2, 1/4, 1/8, 1/16} (block sparsity about
    1 - rho); (b) iid Gaussian inputs with query scale sigma_Q in {1, 3, 8, 24} (AdaSplash-2
    §4.2's knob). Each point: 2 warm-up and `steps` timed forward+backward steps, L2 flushed
    before each step."""
    import torch

    from entmax_sm_attention_b200 import binding as eb
    from entmax_sm_attention_b200.workloads import make_inputs, make_planted_inputs

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    desc = eb.make_desc(w.B, w.H, w.L, w.d, alpha=alpha, scale=w.scale, causal=w.causal, window=w.window)
    ws = eb.alloc_workspace(desc, dev)
    desc64 = eb.make_desc(w.B, w.H, w.L, w.d, alpha=alpha, scale=w.scale, causal=w.causal, window=w.window,
                          mask64=True)
    ws64 = eb.alloc_workspace(desc64, dev)
    active64 = int(block_pair_counts(w, 64).astype(bool).sum()) * w.H   # structurally active 64 x 64 blocks
    shp = (w.B, w.H, w.L, w.d)
    O = torch.empty(shp, dtype=torch.float32, device=dev)
    tau = torch.empty(shp[:3], dtype=torch.float32, device=dev)
    dQ, dK, dV = (torch.empty(shp, dtype=torch.float32, device=dev) for _ in range(3))

    def timed(d, dsc, wsp):
        fwd, bwd = [], []
        for k in range(2 + steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            eb.entmax_attn_fwd(dsc, d["Q"], d["K"], d["V"], O, tau, wsp, stream)
            e[1].record(stream)
            eb.entmax_attn_bwd(dsc, d["Q"], d["K"], d["V"], d["dO"], tau, wsp, dQ, dK, dV, stream)
            e[2].record(stream)
            torch.cuda.synchronize(dev)
            if k >= 2:
                fwd.append(e[0].elapsed_time(e[1]))
                bwd.append(e[1].elapsed_time(e[2]))
        return fwd, bwd

    def point(inp, with64=False):
        d = {k: v.to(dev) for k, v in inp.items()}
        fwd, bwd = timed(d, desc, ws)
        _, st = eb.block_mask((desc, ws))
        st = st.cpu().long()
        extra = {}
        if with64:
            # The same inputs with the 64 x 64 mask built by the kernel (mask64): its block
            # sparsity over the structurally active 64 x 64 blocks, and the times of that
            # variant (the backward then leaves out empty 64-wide halves).
            f64, b64 = timed(d, desc64, ws64)
            M64 = eb.block_mask64((desc64, ws64)).cpu().numpy().view("uint32")
            nset = int(sum(bin(int(x)).count("1") for x in M64.ravel()))
            extra = {"block_sparsity_64": 1.0 - nset / max(1, active64),
                     "mask64_fwd_ms": statistics.mean(f64), "mask64_bwd_ms": statistics.mean(b64)}
        return {**extra, "block_sparsity_128": 1.0 - float(st[..., 2].sum()) / max(1, int(st[..., 3].sum())),
                "refine_sweeps_mean": float(st[..., 0].float().mean()),
                "s_tiles_per_active": float(st[..., 1].sum()) / max(1, int(st[..., 3].sum())),
                "s_tiles": int(st[..., 1].sum()), "flagged_tiles": int(st[..., 2].sum()),
                "fwd_ms": statistics.mean(fwd), "bwd_ms": statistics.mean(bwd),
                "ms": statistics.mean(fwd) + statistics.mean(bwd)}

    planted = []
    for rho in (1.0, 0.5, 0.25, 0.125, 0.0625):
        r = point(make_planted_inputs(w, rho, seed=7))
        r["rho"] = rho
        planted.append(r)
    sigma = []
    for sq in (1.0, 3.0, 8.0, 24.0):
        r = point(make_inputs(w.with_(sigma_q=sq), seed=7), with64=True)
        r["sigma_q"] = sq
        sigma.append(r)
    return {"planted_rho": planted, "iid_sigma_q": sigma, "marginal": marginal_throughput(planted),
            "note": "same shape as the timed workload; planted inputs are a builder-added family"}


def variant_points(w, dev, steps: int = 10) -> list:
    """The timed workload's shape and inputs through the other kernel variants: the run-time
    alpha kernels (alpha 1.25 and 1.75; alpha 2 has its own closed forms) and ALiBi on every
    head (AdaSplash-2 §4.3's NAPE heads) with the geometric slopes 2^(-8 h / H) of Press et
    al., h = 1..H, at alpha 1.5. Per point: 2 warm-up and `steps` timed forward+backward
    steps, L2 flushed before each; times, block sparsity and algorithmic TFLOP/s."""
    import torch

    from entmax_sm_attention_b200 import binding as eb
    from entmax_sm_attention_b200.workloads import make_inputs

    flush = torch.empty(2 * L2_BYTES // 4, dtype=torch.float32, device=dev)
    stream = torch.cuda.current_stream(dev)
    d = {k: v.to(dev) for k, v in make_inputs(w, seed=0).items()}
    shp = (w.B, w.H, w.L, w.d)
    O = torch.empty(shp, dtype=torch.float32, device=dev)
    tau = torch.empty(shp[:3], dtype=torch.float32, device=dev)
    dQ, dK, dV = (torch.empty(shp, dtype=torch.float32, device=dev) for _ in range(3))
    slopes = torch.tensor([2.0 ** (-8.0 * (h + 1) / w.H) for h in range(w.H)], dtype=torch.float32, device=dev)
    out = []
    for name, alpha, alibi in (("alpha_1.25", 1.25, None), ("alpha_1.75", 1.75, None), ("alpha_2", 2.0, None),
                               ("alibi_geometric_alpha_1.5", 1.5, slopes)):
        desc = eb.make_desc(w.B, w.H, w.L, w.d, alpha=alpha, scale=w.scale, causal=w.causal, window=w.window,
                            alibi=alibi)
        ws = eb.alloc_workspace(desc, dev)
        fwd, bwd = [], []
        for k in range(2 + steps):
            flush.zero_()
            e = [torch.cuda.Event(enable_timing=True) for _ in range(3)]
            e[0].record(stream)
            eb.entmax_attn_fwd(desc, d["Q"], d["K"], d["V"], O, tau, ws, stream)
            e[1].record(stream)
            eb.entmax_attn_bwd(desc, d["Q"], d["K"], d["V"], d["dO"], tau, ws, dQ, dK, dV, stream)
            e[2].record(stream)
            torch.cuda.synchronize(dev)
            if k >= 2:
                fwd.append(e[0].elapsed_time(e[1]))
                bwd.append(e[1].elapsed_time(e[2]))
        code, _ = eb.entmax_last_device_status(desc, ws, stream)
        M, st = eb.block_mask((desc, ws))
        work = pair_work(w, M.cpu(), st.cpu())
        st = st.cpu().long()
        f_ms, b_ms = statistics.mean(fwd), statistics.mean(bwd)
        out.append({"variant": name, "alpha": alpha, "status": eb.STATUS_NAMES[code],
                    "block_sparsity_128": 1.0 - float(st[..., 2].sum()) / max(1, int(st[..., 3].sum())),
                    "refine_sweeps_mean": float(st[..., 0].float().mean()),
                    "fwd_ms": f_ms, "bwd_ms": b_ms, "ms": f_ms + b_ms,
                    "tflops_fwd_algorithmic": work["fwd_flops"] / (f_ms * 1e-3) / 1e12,
                    "tflops_bwd_algorithmic": work["bwd_flops"] / (b_ms * 1e-3) / 1e12})
    return out


def marginal_throughput(points) -> dict:
    """Throughput on non-skipped blocks: a least-squares line of time against algorithmic
    tile products over the planted points (block sparsity 0.06 .. 0.93). The slope is the
    cost of the work that grows with the flagged blocks (the intercept holds the fixed and
    the max-pass costs), so 1 / slope is the rate at which flagged blocks are processed."""
    def fit(xs, ys):
        n = len(xs)
        mx, my = sum(xs) / n, sum(ys) / n
        sxx = sum((x - mx) ** 2 for x in xs)
        b = sum((x - mx) * (y - my) for x, y in zip(xs, ys)) / sxx
        return b, my - b * mx
    out = {}
    fl = [UNIT_FLOP * (p["s_tiles"] + p["flagged_tiles"]) for p in points]
    bl = [UNIT_FLOP * 5 * p["flagged_tiles"] for p in points]
    for name, xs, ys in (("fwd", fl, [p["fwd_ms"] for p in points]), ("bwd", bl, [p["bwd_ms"] for p in points]),
                         ("fwd+bwd", [a + b for a, b in zip(fl, bl)], [p["ms"] for p in points])):
        b, a = fit(xs, ys)
        out[name] = {"tflops_on_flagged_blocks": 1e-9 / b if b > 0 else None, "intercept_ms": a}
    return out


def block_pair_counts(w, tile: int = TILE):
    """Structurally active (query, key) pairs in every tile x tile block, per batch entry:
    int64 [B, T, T] with T = ceil(L / tile) (the same for every head)."""
    import numpy as np

    TILE_ = tile
    L, T = w.L, -(-w.L // TILE_)
    out = np.zeros((w.B, T, T), np.int64)
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    for b in range(w.B):
        kv = L if w.kv_len is None else min(max(w.kv_len, 1), L)
        act = np.broadcast_to(j < kv, (L, L))
        if w.window >= 0:
            act = act & (j <= i) & ((j == 0) | (i - j <= w.window))
        elif w.causal:
            act = act & (j <= i)
        pad = np.zeros((T * TILE_, T * TILE_), np.int64)
        pad[:L, :L] = act
        out[b] = pad.reshape(T, TILE_, T, TILE_).sum((1, 3))
    return out


def pair_work(w, M, st) -> dict:
    """Algorithmic tensor work at pair granularity from the block mask M (int32 bit
    patterns [B, H, T, words]) and the forward counters st ([B, H, T, 8]): forward
    sum_i (1+R_i) 2d |A_i| + 2 2d |F_i|, backward 5 2d |F_i|, where A_i are the active keys
    of row i, F_i the active keys of row i inside flagged blocks, and R_i the refinement
    passes of row i's query tile."""
    import numpy as np

    cnt = block_pair_counts(w)                                      # [B, T, T]
    T = cnt.shape[1]
    words = M.numpy().view(np.uint32).astype(np.int64)              # [B, H, T, W]
    bits = np.zeros(words.shape[:3] + (T,), bool)
    for jt in range(T):
        bits[..., jt] = (words[..., jt // 32] >> (jt % 32)) & 1 == 1
    flagged = (bits * cnt[:, None]).sum(-1)                         # [B, H, T] pairs in flagged blocks
    active = np.broadcast_to(cnt.sum(-1)[:, None], flagged.shape)   # [B, H, T] active pairs per query tile
    R = st[..., 0].numpy().astype(np.int64)
    two_d = 2 * w.d
    fwd = int(((1 + R) * active).sum() * two_d + 2 * flagged.sum() * two_d)
    bwd = int(5 * flagged.sum() * two_d)
    return {"fwd_flops": fwd, "bwd_flops": bwd, "active_pairs": int(active.sum()),
            "flagged_pairs": int(flagged.sum())}


def phase_shares(st, bst) -> dict:
    """Cycle shares of the phases, summed over CTAs, from the kernels' clock64 counters:
    forward max pass / refinement + mask decision / output pass; backward (first
    row-owner warp) waiting for S and dA / waiting for the previous tile's MMAs / forming
    A and dS / staging dQ."""
    f = st[..., 4:8].double().sum((0, 1, 2))
    b = bst[..., 1:6].double().sum((0, 1, 2))
    ft = float(f[3]) or 1.0
    bt = float(b[0]) or 1.0
    return {"fwd": {"max_pass": float(f[0]) / ft, "refine_and_mask": float(f[1]) / ft,
                    "output_pass": float(f[2]) / ft, "cta_cycles": float(f[3])},
            "bwd": {"wait_s_dA": float(b[1]) / bt, "wait_prev_mma": float(b[2]) / bt,
                    "form_A_dS": float(b[3]) / bt, "stage_dQ": float(b[4]) / bt, "cta_cycles": float(b[0])}}


def act_pairs(w) -> int:
    """Structurally active (query, key) pairs of the workload."""
    L = w.L
    kv = L if w.kv_len is None else w.kv_len
    if w.window >= 0:
        per = sum(1 + max(0, min(i, kv - 1) - max(1, i - w.window) + 1) for i in range(L))
    elif w.causal:
        per = sum(min(i + 1, kv) for i in range(L))
    else:
        per = L * kv
    return w.B * w.H * per


def main():
    args = parse()
    if args.impl == "reference":
        run_reference(args)
    else:
        run_ours(args)


if __name__ == "__main__":
    main()
