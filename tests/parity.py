"""Shared helpers of the GPU-vs-oracle parity tests (imported by tests only).

Tolerances are the ones the target states for bf16 inputs with fp32 accumulation:
|tau - tau_ref| <= 1e-3 (Eq. 3 units), max|O - O_ref| <= 1e-2,
max|dQ, dK, dV - ref| <= 2e-2. The zero pattern must agree wherever
|z - tau| > 1e-3. Block-skip decisions must be exact, except for tiles whose only
deciding entries lie within that same margin of tau.
"""
from __future__ import annotations

import math

import numpy as np
import torch

import oracle
from entmax_sm_attention_b200 import binding as eb
from entmax_sm_attention_b200.workloads import Workload, make_inputs

TOL_TAU = 1e-3
TOL_O = 1e-2
TOL_GRAD = 2e-2
MARGIN = 1e-3
# alpha = 2 has g = [u > 0], so an entry whose fp32 and fp64 support decisions can differ
# flips g by 1: dS of that entry, and through sum g and Ot also delta_i of its row, change
# by O(1). Such entries are found per entry with a band derived from the arithmetic (see
# alpha2_exclusions); dQ of their rows and dK of their keys and of their rows' support keys
# are reported, not compared. A = [z - tau]_+ is continuous, so dV is always compared.


def gpu_run(inp: dict, w: Workload, alpha: float, backward: bool = True, max_sweeps: int = 0,
            mask64: bool = False):
    dev = {k: v.cuda() for k, v in inp.items()}
    kv = None if w.kv_len is None else torch.tensor(w.kv_len_list(), dtype=torch.int32, device="cuda")
    ab = None if w.alibi is None else torch.tensor(w.alibi, dtype=torch.float32, device="cuda")
    O, tau, ctx = eb.forward(dev["Q"], dev["K"], dev["V"], alpha=alpha, scale=w.scale, causal=w.causal,
                             window=w.window, kv_len=kv, max_sweeps=max_sweeps, alibi=ab, mask64=mask64)
    out = {"O": O, "tau": tau}
    if backward:
        out["dQ"], out["dK"], out["dV"] = eb.backward(ctx, dev["Q"], dev["K"], dev["V"], dev["dO"], tau)
    M, stats = eb.block_mask(ctx)
    M64 = eb.block_mask64(ctx) if mask64 else None
    code, word = eb.entmax_last_device_status(ctx[0], ctx[1])
    torch.cuda.synchronize()
    res = {k: v.cpu().double().numpy() for k, v in out.items()}
    res["M"] = M.cpu().numpy().view(np.uint32)
    if M64 is not None:
        res["M64"] = M64.cpu().numpy().view(np.uint32)
    res["stats"] = stats.cpu().numpy()
    res["status"] = (code, word)
    return res


def oracle_problem(inp: dict, w: Workload, alpha: float) -> oracle.Problem:
    return oracle.Problem(inp["Q"], inp["K"], inp["V"], inp["dO"], alpha=alpha, scale=w.scale, causal=w.causal,
                          window=w.window, kv_len=w.kv_len_list(), alibi=w.alibi)


def alpha2_exclusions(pr: oracle.Problem, tau_ref: np.ndarray, tau_gpu: np.ndarray):
    """Rows (dQ) and keys (dK) that an ambiguous alpha = 2 support decision can move.

    Entry (i, k) is ambiguous when |z_ik - tau_i| lies within the band where fp32 and fp64
    can disagree: 4 |tau_gpu - tau_ref| (the measured threshold difference) plus
    2^-15 (alpha-1) scale sum_d |q_id k_kd| (fp32 accumulation of the 64 exact bf16
    products: at most 64 roundings of 2^-24 relative to the running sum, times 4 for
    safety) plus 2^-20.

    A flip of (i, k) changes g_ik by 1, so dS_ik changes by |dA_ik - delta_i|: row i (dQ)
    and key k (dK) are excluded. It also moves delta_i = sum_j g_ij dA_ij / sum_j g_ij by at
    most max_k |dA_ik - delta_i| / (|S_i| - 1), which reaches every support key j of row i
    as scale * that * max_d |Q_id| in dK_j. A support key is excluded only when those
    bounds, summed over its ambiguous rows, exceed a quarter of the gradient tolerance.
    Returns boolean [B,H,L] arrays (rows, keys)."""
    B, H, L = pr.B, pr.H, pr.L
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    rows = np.zeros((B, H, L), bool)
    keys = np.zeros((B, H, L), bool)
    c = (pr.alpha - 1) * pr.scale
    for b in range(B):
        kv = L if pr.kv_len is None else int(pr.kv_len[b])
        act = np.broadcast_to(j < kv, (L, L)).copy()
        if pr.window >= 0:
            act &= (j <= i) & ((j == 0) | (i - j <= pr.window))
        elif pr.causal:
            act &= j <= i
        for h in range(H):
            Q, K = pr.Q[b, h], pr.K[b, h]
            z = c * (Q @ K.T)
            if pr.alibi is not None:   # ALiBi: the penalty m_h |i - j| on the scores
                z = z - (pr.alpha - 1) * pr.alibi[h] * np.abs(i - j)
            t = tau_ref[b, h][:, None]
            band = (4 * np.abs(tau_gpu[b, h] - tau_ref[b, h])[:, None]
                    + 2.0 ** -15 * c * (np.abs(Q) @ np.abs(K).T) + 2.0 ** -20)
            amb = act & (np.abs(z - t) <= band)
            r = amb.any(1)
            rows[b, h] = r
            k_own = amb.any(0)
            if r.any():
                supp = act & (z > t)
                dA = pr.dO[b, h][r] @ pr.V[b, h].T                      # [rows r, L]
                sr = supp[r]
                n = np.maximum(sr.sum(1), 1)
                delta = (np.where(sr, dA, 0.0)).sum(1) / n
                shift = np.where(amb[r], np.abs(dA - delta[:, None]), 0.0).max(1) / np.maximum(n - 1, 1)
                per_row = pr.scale * shift * np.abs(Q[r]).max(1)        # bound on |d dK_j| per row
                bound = (sr * per_row[:, None]).sum(0)
                k_own |= bound > TOL_GRAD / 4
            keys[b, h] = k_own
    return rows, keys


def check_mask(pr: oracle.Problem, tau_ref: np.ndarray, M_gpu: np.ndarray, block: int = 128):
    """Bits of the GPU block mask that disagree with the oracle's, away from the ambiguity
    margin, and the number of ambiguous bits. block = 64: the 64 x 64 mask, whose GPU copy
    has 2 ceil(L/128) rows per head (a last row past L must be empty)."""
    M, Mlo, Mhi = pr.block_mask(tau_ref, block, block, margin=MARGIN)
    G = M_gpu
    if G.shape != M.shape:
        extra = G[..., M.shape[2]:, :]
        assert not extra.any(), "64 x 64 mask rows past L must be empty"
        G = G[..., : M.shape[2], : M.shape[3]]
    decided = ~(Mlo ^ Mhi)
    bad = (G ^ M) & decided
    n_amb = int(sum(bin(int(x)).count("1") for x in (Mlo ^ Mhi).ravel()))
    return int(np.count_nonzero(bad)), n_amb


def compare(w: Workload, alpha: float, backward: bool = True, seed: int = 0, report: dict | None = None,
            mask64: bool = True):
    """GPU against the oracle on one small case. mask64 (default on here) also builds the
    64 x 64 mask, checks it bit for bit, and runs the backward variant that skips empty
    64-wide halves."""
    inp = make_inputs(w, seed)
    g = gpu_run(inp, w, alpha, backward, mask64=mask64)
    pr = oracle_problem(inp, w, alpha)
    ref = pr.backward() if backward else pr.forward()
    err = {"tau": np.abs(g["tau"] - ref["tau"]).max(), "O": np.abs(g["O"] - ref["O"]).max()}
    assert g["status"][0] == eb.ENTMAX_OK, g["status"]
    nbad, namb = check_mask(pr, ref["tau"], g["M"])
    err["mask_bad"], err["mask_ambiguous"] = nbad, namb
    nbad64 = 0
    if mask64:
        nbad64, namb64 = check_mask(pr, ref["tau"], g["M64"], 64)
        err["mask64_bad"], err["mask64_ambiguous"] = nbad64, namb64
    if backward:
        if alpha == 2.0:
            xr, xk = alpha2_exclusions(pr, ref["tau"], g["tau"])
            rmask, cmask = ~xr[..., None], ~xk[..., None]
            err["excluded_rows"] = int(xr.sum())
            err["excluded_keys"] = int(xk.sum())
        else:
            rmask = cmask = np.ones(ref["tau"].shape + (1,), bool)
        err["dQ"] = np.abs(np.where(rmask, g["dQ"] - ref["dQ"], 0)).max()
        err["dK"] = np.abs(np.where(cmask, g["dK"] - ref["dK"], 0)).max()
        err["dV"] = np.abs(g["dV"] - ref["dV"]).max()
    if report is not None:
        report.update(err)
    assert err["tau"] <= TOL_TAU, err
    assert err["O"] <= TOL_O, err
    assert nbad == 0, err
    assert nbad64 == 0, err
    if backward:
        assert max(err["dQ"], err["dK"], err["dV"]) <= TOL_GRAD, err
    return err, g, ref
