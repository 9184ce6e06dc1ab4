"""Full-size workloads on the GPU, checked against the oracle on sampled heads.

The GPU runs the whole batch, in the launch configuration the bench uses. The oracle
recomputes a few complete (batch, head) pairs in fp64: every row's tau, O and dQ,
every key's dK and dV, and the head's block mask. All are compared element by
element at the stated tolerances.
"""
import numpy as np
import pytest
import torch

import oracle
from entmax_sm_attention_b200 import binding as eb
from entmax_sm_attention_b200.workloads import WORKLOADS, make_inputs

from parity import MARGIN, TOL_GRAD, TOL_O, TOL_TAU, alpha2_exclusions, gpu_run

pytestmark = pytest.mark.gpu

# Three or more whole heads per workload: the first (0, 0), the last (B-1, H-1) and one
# or two in between.
FULL = [
    ("gpt2_causal_L1024", 1.5, [(0, 0), (3, 5), (7, 11)]),
    ("long_causal_L8192", 1.5, [(0, 0), (0, 5), (0, 11)]),
    ("long_causal_L8192", 2.0, [(0, 0), (0, 3), (0, 11)]),
    ("encoder_padded_L4096", 1.5, [(0, 0), (3, 2), (3, 11)]),
    ("encoder_padded_L4096", 2.0, [(0, 0), (1, 7), (3, 11)]),
    ("window_sink_L2048", 1.5, [(0, 0), (4, 0), (9, 6), (15, 11)]),
]


def head_problem(inp, w, alpha, b, h):
    sl = lambda x: x[b:b + 1, h:h + 1]  # noqa: E731
    kv = None if w.kv_len is None else [w.kv_len]
    return oracle.Problem(sl(inp["Q"]), sl(inp["K"]), sl(inp["V"]), sl(inp["dO"]), alpha=alpha, scale=w.scale,
                          causal=w.causal, window=w.window, kv_len=kv)


@pytest.mark.parametrize("name,alpha,heads", FULL, ids=[f"{n}-a{a}" for n, a, _ in FULL])
def test_full_size(name, alpha, heads):
    w = WORKLOADS[name]
    inp = make_inputs(w, seed=0)
    g = gpu_run(inp, w, alpha, backward=True)
    assert g["status"][0] == eb.ENTMAX_OK, g["status"]
    for (b, h) in heads:
        pr = head_problem(inp, w, alpha, b, h)
        ref = pr.backward()
        tau_ref = ref["tau"][0, 0]
        assert np.abs(g["tau"][b, h] - tau_ref).max() <= TOL_TAU
        assert np.abs(g["O"][b, h] - ref["O"][0, 0]).max() <= TOL_O
        rows_ok = np.ones(w.L, bool)
        keys_ok = np.ones(w.L, bool)
        if alpha == 2.0:
            xr, xk = alpha2_exclusions(pr, ref["tau"], g["tau"][b:b + 1, h:h + 1])
            rows_ok, keys_ok = ~xr[0, 0], ~xk[0, 0]
        errs = {
            "dQ": np.abs(g["dQ"][b, h] - ref["dQ"][0, 0])[rows_ok].max(),
            "dK": np.abs(g["dK"][b, h] - ref["dK"][0, 0])[keys_ok].max(),
            "dV": np.abs(g["dV"][b, h] - ref["dV"][0, 0]).max(),
            "excluded_rows": int((~rows_ok).sum()), "excluded_keys": int((~keys_ok).sum()),
        }
        print(name, alpha, (b, h), {k: float(v) for k, v in errs.items()},
              "tau", float(np.abs(g["tau"][b, h] - tau_ref).max()),
              "O", float(np.abs(g["O"][b, h] - ref["O"][0, 0]).max()))
        assert max(errs["dQ"], errs["dK"], errs["dV"]) <= TOL_GRAD, errs
        M, Mlo, Mhi = pr.block_mask(ref["tau"], 128, 128, margin=MARGIN)
        decided = ~(Mlo ^ Mhi)
        assert np.count_nonzero((g["M"][b, h] ^ M[0, 0]) & decided[0, 0]) == 0

