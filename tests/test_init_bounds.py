"""The forward's initial threshold against the pages' histogram initialisation (CPU).

"AdaSplash-2" §3.1 and Appendix C.3 start the refinement from tau_h, the root of Eq. 4
with every score replaced by the left edge of its histogram bin (B bins); Proposition 3.1
bounds it by tau* - 1/B <= tau_h <= tau*. The forward kernel starts instead from tau_T, the
root of Eq. 4 on a subset of the row's scores: the four largest of its part-tile maxima
(maxima over 32 consecutive keys of a 128-key tile) in each of the four column parts. A
subset has f_T <= f, so tau_T <= tau* as well. Its use in the kernel is to bound the
candidate copies: every score above the initial threshold is copied, so a tighter bound
means fewer copies.

On the iid workloads of AdaSplash-2 §4.2 (Gaussian Q, K with d = 64 and query scale
sigma_Q), one causal head of length 1024: both are lower bounds on every row, and tau_T
leaves no more candidates on average than tau_h with 8 bins (the B of the pages' kernel).
tau_T has no worst-case bound like 1/B; a row whose support is spread over more part-tiles
than the sixteen kept can have a loose tau_T, which only costs copies.
"""
import numpy as np
import pytest

import oracle
from entmax_sm_attention_b200.workloads import WORKLOADS, make_inputs


def tile_max_bound(z, alpha):
    """tau on the four largest part-tile maxima of each column part (-inf entries inactive)."""
    n = z.size
    nt = -(-n // 128)
    zp = np.full(nt * 128, -np.inf)
    zp[:n] = z
    pm = zp.reshape(nt, 4, 32).max(-1)               # [tile, part]
    top = -np.sort(-pm.T, axis=1)[:, :4].ravel()      # four largest per part
    top = top[np.isfinite(top)]
    return oracle.tau_sort(top, alpha)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("sigma_q", [1.0, 3.0, 8.0, 24.0])
def test_tile_max_bound_against_histogram(alpha, sigma_q):
    w = WORKLOADS["long_causal_L8192"].with_(B=1, H=1, L=1024, sigma_q=sigma_q)
    inp = make_inputs(w, seed=0)
    Q = inp["Q"][0, 0].double().numpy()
    K = inp["K"][0, 0].double().numpy()
    cz = (alpha - 1.0) * w.scale
    gap_t, gap_h, cand_t, cand_h, supp = [], [], [], [], []
    for i in range(16, 1024, 13):
        z = cz * (Q[i] @ K[: i + 1].T)
        ts = oracle.tau_sort(z, alpha)
        tt = tile_max_bound(z, alpha)
        th = oracle.tau_hist(z, alpha, 8)
        assert tt <= ts + 1e-12 and th <= ts + 1e-12
        gap_t.append(ts - tt)
        gap_h.append(ts - th)
        cand_t.append(int((z > tt).sum()))
        cand_h.append(int((z > th).sum()))
        supp.append(int((z > ts).sum()))
    print(f"alpha {alpha} sigma_Q {sigma_q}: mean tau* - tau_T {np.mean(gap_t):.4f} (max {np.max(gap_t):.4f}), "
          f"tau* - tau_h(B=8) {np.mean(gap_h):.4f}; candidates tau_T {np.mean(cand_t):.2f}, "
          f"tau_h {np.mean(cand_h):.2f}, support {np.mean(supp):.2f}")
    assert np.mean(cand_t) <= np.mean(cand_h)
