"""GPU parity at alpha outside {1.5, 2} (the run-time alpha variant), against the fp64
oracle's bisection of Eq. 4 (AdaSplash-2 §2.4; §3.2 covers general alpha).

Forward and backward at alpha = 1.25 and 1.75: p = u^{1/(alpha-1)} and g = u^{(2-alpha)/
(alpha-1)} are continuous at the support boundary, so the same tolerances apply as at
alpha = 1.5. At alpha > 2, g = p^{2-alpha} is unbounded as p -> 0 (a property of the
method's Jacobian, not of the kernels), so fp32 and fp64 gradients of keys just inside
the support cannot agree to an absolute tolerance; alpha = 3 is checked on the forward
(tau, O and the block mask).
"""
import numpy as np
import pytest

from entmax_sm_attention_b200.workloads import small_case

from parity import compare

pytestmark = pytest.mark.gpu

CASES = [
    (small_case("causal_L300", L=300, causal=True), 1.25, True),
    (small_case("causal_L300", L=300, causal=True), 1.75, True),
    (small_case("window_L300", L=300, causal=True, window=32), 1.25, True),
    (small_case("padded_L300", B=2, L=300, kv_len=200), 1.75, True),
    (small_case("peaked_causal_L520", L=520, causal=True, sigma_q=3.0), 1.25, True),
    (small_case("sigma8_L384", L=384, causal=True, sigma_q=8.0), 1.75, True),
    # flat rows: the candidate copies overflow, so refinement takes Newton sweeps and the
    # backward recomputes the support of the rows it could not list
    (small_case("flat_sigma005_L512", L=512, sigma_q=0.05), 1.25, True),
    (small_case("causal_L1100", B=1, H=1, L=1100, causal=True), 1.25, True),
    (small_case("full_L300", L=300), 3.0, False),
    (small_case("causal_L520", L=520, causal=True, sigma_q=2.0), 3.0, False),
]


@pytest.mark.parametrize("mask64", [True, False], ids=["mask64", "default"])
@pytest.mark.parametrize("w,alpha,backward", CASES, ids=[f"{w.name}-a{a}" for w, a, _ in CASES])
def test_general_alpha(w, alpha, backward, mask64):
    """Each case in both kernel variants (with and without the 64 x 64 mask)."""
    rep = {}
    compare(w, alpha, backward=backward, report=rep, mask64=mask64)
    print(w.name, alpha, {k: (float(v) if not isinstance(v, int) else v) for k, v in rep.items()})
