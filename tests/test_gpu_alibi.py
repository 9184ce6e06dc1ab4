"""GPU parity with ALiBi slopes (AdaSplash-2 §4.3: NAPE heads, half without positional
encoding, half with ALiBi) against the fp64 oracle, element by element.

The slopes are per head, in score units per position; a zero slope is a NoPE head, so
mixed slopes check both kinds in one launch. Large slopes push every far key below the
threshold, so whole key tiles drop out of the mask: the last case checks that the mask
is still exact and that block sparsity appears on iid inputs.
"""
import numpy as np
import pytest

from entmax_sm_attention_b200 import binding as eb
from entmax_sm_attention_b200.workloads import small_case

from parity import compare

pytestmark = pytest.mark.gpu

CASES = [
    (small_case("alibi_causal_L300", H=3, L=300, causal=True, alibi=(0.0, 0.1, 0.5)), 1.5),
    (small_case("alibi_causal_L300", H=3, L=300, causal=True, alibi=(0.0, 0.1, 0.5)), 2.0),
    (small_case("alibi_causal_L300", H=3, L=300, causal=True, alibi=(0.0, 0.1, 0.5)), 1.25),
    (small_case("alibi_full_L260", H=2, L=260, alibi=(0.05, 0.3)), 1.5),
    (small_case("alibi_window_L300", H=2, L=300, causal=True, window=32, alibi=(0.2, 0.0)), 1.5),
    (small_case("alibi_padded_L300", B=2, H=2, L=300, kv_len=200, alibi=(0.1, 0.02)), 2.0),
    (small_case("alibi_causal_L1100", H=2, L=1100, causal=True, sigma_q=2.0, alibi=(0.02, 0.2)), 1.5),
    # near-uniform rows with a gentle slope: the candidate copies overflow, and the
    # backward recomputes those rows' support (with the penalty) over their flagged tiles
    (small_case("alibi_flat_L512", H=2, L=512, sigma_q=0.05, alibi=(0.0005, 0.002)), 1.5),
]


@pytest.mark.parametrize("mask64", [True, False], ids=["mask64", "default"])
@pytest.mark.parametrize("w,alpha", CASES, ids=[f"{w.name}-a{a}" for w, a in CASES])
def test_alibi(w, alpha, mask64):
    """Each case in both kernel variants: with the 64 x 64 mask (checked bit for bit) and
    the default kernels."""
    rep = {}
    compare(w, alpha, backward=True, report=rep, mask64=mask64)
    print(w.name, alpha, {k: (float(v) if not isinstance(v, int) else v) for k, v in rep.items()})


def test_alibi_gives_block_sparsity_L4096():
    """One causal head of L = 4096 with a slope that keeps each row's support within a few
    hundred positions: the far key tiles are skipped (block sparsity well above 0 on iid
    inputs), and the result, mask included, matches the oracle."""
    w = small_case("alibi_L4096", B=1, H=1, L=4096, causal=True, alibi=(0.02,))
    err, g, _ = compare(w, 1.5, backward=True)
    st = g["stats"].reshape(-1, eb.FWD_STATS)
    sparsity = 1.0 - st[:, 2].sum() / st[:, 3].sum()
    print("alibi_L4096 block sparsity", sparsity, {k: float(v) for k, v in err.items()})
    assert sparsity > 0.5
