"""GPU (B200) vs fp64 oracle, element by element, through the C ABI.

Sizes are small enough for the oracle to finish in seconds, yet span several 128-wide
tiles with a ragged tail. The edge cases are L = 1, single-tile and tile-boundary
lengths, key padding, window + sink, peaked rows, and the refinement cap.
"""
import numpy as np
import pytest
import torch

import oracle
from entmax_sm_attention_b200 import binding as eb
from entmax_sm_attention_b200.workloads import make_inputs, make_score_rows, small_case

from parity import TOL_TAU, compare, gpu_run

pytestmark = pytest.mark.gpu

CASES = [
    small_case("full_L300", L=300),
    small_case("causal_L300", L=300, causal=True),
    small_case("window_L300", L=300, causal=True, window=32),
    small_case("padded_L300", B=2, L=300, kv_len=200),
    small_case("peaked_causal_L520", L=520, causal=True, sigma_q=3.0),
    small_case("single_row", L=1),
    small_case("one_tile_L128", L=128, causal=True),
    small_case("tile_plus_one_L129", L=129),
    small_case("padded_short_kv", B=1, L=260, kv_len=5),
    small_case("window0_L200", L=200, causal=True, window=0),
    small_case("wide_sigma8_L384", L=384, causal=True, sigma_q=8.0),
    # Near-uniform rows: at alpha = 1.5 almost every key is in the support, so the
    # candidate lists overflow and the threshold takes Newton sweeps; at alpha = 2 the
    # support (28+ keys) still fits and is solved in the max pass.
    small_case("flat_sigma005_L512", L=512, sigma_q=0.05),
    # Exactly uniform rows (Q = 0, all scores tie): p = 1/n, tau = -n^{1-alpha}; every key is
    # in the support, so both alphas take the sweep path.
    small_case("uniform_sigma0_L512", L=512, sigma_q=0.0),
]


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("w", CASES, ids=lambda w: w.name)
def test_fwd_bwd_small(w, alpha):
    """Every case with the 64 x 64 mask built (checked bit for bit) and the backward variant
    that leaves out empty 64-wide halves."""
    rep = {}
    compare(w, alpha, backward=True, report=rep)
    print(w.name, alpha, {k: (float(v) if not isinstance(v, int) else v) for k, v in rep.items()})


@pytest.mark.parametrize("alpha", [1.5, 2.0])
@pytest.mark.parametrize("w", [c for c in CASES if c.name in ("causal_L300", "window_L300", "padded_L300",
                                                                  "peaked_causal_L520", "tile_plus_one_L129")],
                         ids=lambda w: w.name)
def test_fwd_bwd_small_without_mask64(w, alpha):
    """The default kernels (no 64 x 64 mask) on the cases whose structure leaves 64-wide
    halves empty."""
    compare(w, alpha, backward=True, mask64=False)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_entmax_rows(alpha):
    # The 128 x 128 score rows of the single-head workload, plus long rows with inactive entries.
    for rows, n, sigma in ((128, 128, 1.0), (64, 1000, 2.0), (16, 4096, 0.5)):
        S = make_score_rows(rows, n, seed=n, sigma=sigma)
        if n == 1000:
            S[3, 10:] = -float("inf")
            S[4, :999] = -float("inf")
        P, tau, st = eb.rows(S.cuda(), alpha, return_status=True)
        assert st == 0
        P, tau = P.cpu().double().numpy(), tau.cpu().double().numpy()
        Pr, taur = oracle.entmax_rows(S, alpha)
        assert np.abs(tau - taur).max() <= 1e-5
        assert np.abs(P - Pr).max() <= 1e-5
        z = (alpha - 1) * S.double().numpy()
        decided = np.abs(z - taur[:, None]) > 1e-3
        assert np.array_equal((P > 0)[decided], (Pr > 0)[decided])
    # Uniform rows (all scores tie): p = 1/n and tau = (alpha-1) s - n^{1-alpha}, the upper
    # end of the §2.4 bracket.
    for n, v in ((300, 0.0), (1000, 3.7)):
        S = torch.full((3, n), v, dtype=torch.float32)
        P, tau = eb.rows(S.cuda(), alpha)
        P, tau = P.cpu().double().numpy(), tau.cpu().double().numpy()
        assert np.abs(P - 1.0 / n).max() <= 1e-6
        assert np.abs(tau - ((alpha - 1) * v - n ** (1 - alpha))).max() <= 1e-5


def test_refinement_cap_reports_no_convergence():
    """Refinement capped at one sweep on rows that need several (near-uniform rows whose
    support, 174+ keys per column half at both alphas, overflows the on-chip candidate
    lists): the status word says so. Per §2.4 tau stays inside the bracket, so O stays
    finite."""
    w = small_case("capped", L=512, causal=False, sigma_q=0.002)
    from parity import gpu_run
    from entmax_sm_attention_b200.workloads import make_inputs
    for alpha in (1.5, 2.0):
        g = gpu_run(make_inputs(w), w, alpha, backward=False, max_sweeps=1)
        assert g["status"][0] == eb.ENTMAX_ENOCONVERGE, alpha
        assert np.isfinite(g["O"]).all() and np.isfinite(g["tau"]).all()
        g = gpu_run(make_inputs(w), w, alpha, backward=False)
        assert g["status"][0] == eb.ENTMAX_OK, alpha
        assert g["stats"].reshape(-1, eb.FWD_STATS)[:, 0].max() > 1   # it took more than one sweep


def test_repeatable():
    """Two forward+backward calls give bit-identical O, tau and dK/dV. dQ uses float
    atomics and is only compared to tolerance."""
    w = small_case("rep", L=384, causal=True)
    from parity import gpu_run
    from entmax_sm_attention_b200.workloads import make_inputs
    inp = make_inputs(w)
    a, b = gpu_run(inp, w, 1.5), gpu_run(inp, w, 1.5)
    for k in ("O", "tau", "dK", "dV", "M"):
        assert np.array_equal(a[k], b[k]), k
    assert np.abs(a["dQ"] - b["dQ"]).max() < 1e-5


def test_single_head_fp32_workload():
    """B=H=1, L=128, fp32 Q, K, V, non-causal: forward against the oracle, plus
    entmax_rows on the same 128 x 128 score matrix S = Q K^T / sqrt(d)."""
    from entmax_sm_attention_b200.workloads import WORKLOADS, make_inputs
    from parity import check_mask, gpu_run, oracle_problem

    w = WORKLOADS["single_head_L128_fp32"]
    inp = make_inputs(w, seed=0)
    assert inp["Q"].dtype == torch.float32
    g = gpu_run(inp, w, 1.5, backward=False)
    assert g["status"][0] == eb.ENTMAX_OK
    pr = oracle_problem(inp, w, 1.5)
    ref = pr.forward()
    assert np.abs(g["tau"] - ref["tau"]).max() <= TOL_TAU
    assert np.abs(g["O"] - ref["O"]).max() <= 1e-2
    assert check_mask(pr, ref["tau"], g["M"])[0] == 0
    if "M64" in g:
        assert check_mask(pr, ref["tau"], g["M64"], 64)[0] == 0
    # entmax_rows on the explicit scores (computed in fp32 on the GPU by torch: plumbing)
    S = (inp["Q"][0, 0].cuda() @ inp["K"][0, 0].cuda().T) * w.scale
    P, tau = eb.rows(S.contiguous(), 1.5)
    Pr, taur = oracle.entmax_rows(S.cpu(), 1.5)
    assert np.abs(tau.cpu().numpy() - taur).max() <= 1e-5
    assert np.abs(P.cpu().numpy() - Pr).max() <= 1e-5


def test_fp32_uniform_rows():
    """fp32 forward on exactly uniform rows (Q = 0): tau sits at the upper end of the
    bracket, -n^{1-alpha}, and O is the mean of the active values."""
    from parity import gpu_run, oracle_problem
    from entmax_sm_attention_b200.workloads import make_inputs

    for causal in (False, True):
        w = small_case("uniform_fp32", L=200, dtype="fp32", sigma_q=0.0, causal=causal)
        inp = make_inputs(w)
        for alpha in (1.5, 2.0):
            g = gpu_run(inp, w, alpha, backward=False)
            assert g["status"][0] == eb.ENTMAX_OK
            ref = oracle_problem(inp, w, alpha).forward()
            assert np.abs(g["tau"] - ref["tau"]).max() <= TOL_TAU
            assert np.abs(g["O"] - ref["O"]).max() <= 1e-2


def test_fp32_backward_is_rejected():
    d = {k: torch.zeros(1, 1, 128, 64, device="cuda") for k in ("Q", "K", "V", "dO")}
    O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"])
    with pytest.raises(eb.EntmaxError) as e:
        eb.backward(ctx, d["Q"], d["K"], d["V"], d["dO"], tau)
    assert e.value.code == eb.ENTMAX_EUNSUPPORTED


def test_out_of_fp16_range_is_reported():
    """V and dO feed fp16 products; a bf16 value beyond fp16's range is flagged."""
    from entmax_sm_attention_b200.workloads import make_inputs

    w = small_case("range", L=256)
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    d["V"][0, 1, 7, 3] = 1.0e5
    O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"], alpha=1.5, scale=w.scale)
    code, word = eb.entmax_last_device_status(*ctx)
    assert code == eb.ENTMAX_ERANGE and word & 4
    d["V"][0, 1, 7, 3] = 0.5
    O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"], alpha=1.5, scale=w.scale)
    assert eb.entmax_last_device_status(*ctx)[0] == eb.ENTMAX_OK
    d["dO"][0, 0, 3, 1] = -7.0e4
    eb.backward(ctx, d["Q"], d["K"], d["V"], d["dO"], tau)
    assert eb.entmax_last_device_status(*ctx)[0] == eb.ENTMAX_ERANGE


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_planted_block_structure(alpha):
    """Block-structured inputs (support confined to a fraction rho of the key tiles):
    parity with the oracle, an exact mask, real block sparsity, and a backward that
    visits only the flagged tiles."""
    from entmax_sm_attention_b200.workloads import make_planted_inputs
    from parity import check_mask, gpu_run, oracle_problem

    w = small_case("planted", B=1, H=2, L=1100, causal=True)
    inp = make_planted_inputs(w, 0.25, seed=3)
    g = gpu_run(inp, w, alpha, backward=True)
    pr = oracle_problem(inp, w, alpha)
    ref = pr.backward()
    assert np.abs(g["tau"] - ref["tau"]).max() <= TOL_TAU
    assert np.abs(g["O"] - ref["O"]).max() <= 1e-2
    for k in ("dQ", "dK", "dV"):
        assert np.abs(g[k] - ref[k]).max() <= 2e-2, k
    assert check_mask(pr, ref["tau"], g["M"])[0] == 0
    if "M64" in g:
        assert check_mask(pr, ref["tau"], g["M64"], 64)[0] == 0
    st = g["stats"].reshape(-1, eb.FWD_STATS)
    sparsity = 1.0 - st[:, 2].sum() / st[:, 3].sum()
    assert sparsity > 0.5, sparsity


def test_long_head_L12288():
    """One long head (L = 12288, 96 key tiles; 48 KB of per-tile maxima in shared
    memory), causal, alpha = 1.5, checked element by element."""
    w = small_case("long_L12288", B=1, H=1, L=12288, causal=True, sigma_q=3.0)
    rep = {}
    compare(w, 1.5, backward=True, report=rep)
    print(w.name, {k: (float(v) if not isinstance(v, int) else v) for k, v in rep.items()})


def test_max_length_head():
    """L = ENTMAX_MAX_L = 16384 (128 key tiles: every bit of the four mask words), one head,
    causal, alpha = 1.5, checked element by element. Shared memory: 217 KB of 227."""
    w = small_case("max_L16384", B=1, H=1, L=16384, causal=True, sigma_q=3.0)
    rep = {}
    compare(w, 1.5, backward=True, report=rep)
    print(w.name, {k: (float(v) if not isinstance(v, int) else v) for k, v in rep.items()})


@pytest.mark.parametrize("stage", ["fwd", "bwd"])
def test_wait_expiry_reports_timeout_and_context_survives(stage):
    """The bounded-wait failure path, without faulting or hanging anything: with
    ENTMAX_SELFTEST_STALL one thread of every CTA waits on a barrier that nothing
    completes, so its wait expires after wait_limit_us (200 us here). The call must report
    ENTMAX_ETIMEOUT; every other wait then returns at once, no copy or MMA is issued after
    the abort, the CTA frees its tensor memory and exits. A normal call on the same stream
    afterwards returns ENTMAX_OK and matches the oracle."""
    from entmax_sm_attention_b200.workloads import make_inputs

    w = small_case("stall", B=1, H=1, L=256, causal=True)
    inp = make_inputs(w)
    d = {k: v.cuda() for k, v in inp.items()}
    kw = dict(alpha=1.5, scale=w.scale, causal=True)
    if stage == "fwd":
        O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"], wait_limit_us=200, selftest=eb.ENTMAX_SELFTEST_STALL, **kw)
        code, word = eb.entmax_last_device_status(*ctx)
        assert code == eb.ENTMAX_ETIMEOUT and word & 2, (code, word)
    else:
        O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"], **kw)
        assert eb.entmax_last_device_status(*ctx)[0] == eb.ENTMAX_OK
        desc, ws = ctx
        stall = eb.make_desc(1, 1, w.L, alpha=1.5, scale=w.scale, causal=True, wait_limit_us=200,
                             selftest=eb.ENTMAX_SELFTEST_STALL)
        dQ, dK, dV = eb.backward((stall, ws), d["Q"], d["K"], d["V"], d["dO"], tau)
        code, word = eb.entmax_last_device_status(stall, ws)
        assert code == eb.ENTMAX_ETIMEOUT and word & 2, (code, word)
    # The context is intact: a normal forward + backward on the same stream is correct.
    O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"], **kw)
    dQ, dK, dV = eb.backward(ctx, d["Q"], d["K"], d["V"], d["dO"], tau)
    assert eb.entmax_last_device_status(*ctx)[0] == eb.ENTMAX_OK
    ref = oracle.Problem(inp["Q"], inp["K"], inp["V"], inp["dO"], alpha=1.5, scale=w.scale, causal=True).backward()
    assert np.abs(tau.cpu().double().numpy() - ref["tau"]).max() <= TOL_TAU
    assert np.abs(O.cpu().double().numpy() - ref["O"]).max() <= 1e-2
    for k, v in (("dQ", dQ), ("dK", dK), ("dV", dV)):
        assert np.abs(v.cpu().double().numpy() - ref[k]).max() <= 2e-2, k


def test_backward_counters():
    """The per-key-tile counters of the backward: flagged query tiles visited equal the set
    bits of the transposed mask, and the phase cycles add up to at most the CTA total."""
    from entmax_sm_attention_b200.workloads import make_inputs

    w = small_case("bcount", B=1, H=2, L=700, causal=True)
    d = {k: v.cuda() for k, v in make_inputs(w).items()}
    O, tau, ctx = eb.forward(d["Q"], d["K"], d["V"], alpha=1.5, scale=w.scale, causal=True)
    eb.backward(ctx, d["Q"], d["K"], d["V"], d["dO"], tau)
    M, st = eb.block_mask(ctx)
    bst = eb.bwd_counters(ctx).cpu().numpy().reshape(-1, eb.BWD_STATS).astype(np.int64)
    Mb = M.cpu().numpy().view(np.uint32).reshape(2, -1)
    T = Mb.shape[1]
    per_key = np.array([[sum((int(Mb[h, it]) >> kt) & 1 for it in range(T)) for kt in range(T)] for h in range(2)])
    assert np.array_equal(bst[:, 0], per_key.ravel())
    assert (bst[:, 1] > 0).all()
    assert (bst[:, 2:6].sum(1) <= bst[:, 1]).all()
    fst = st.cpu().numpy().reshape(-1, eb.FWD_STATS).astype(np.int64)
    assert (fst[:, 4:7].sum(1) <= fst[:, 7]).all() and (fst[:, 7] > 0).all()


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_mask64_variant_matches_default(alpha):
    """The 64 x 64 variant only adds the finer mask and leaves out MMA steps whose products
    are exactly zero, so O, tau, dK and dV are bit-identical to the default kernels' (dQ is
    a sum of reduce-adds in no fixed order, so it is compared to fp32 rounding)."""
    w = small_case("peaked_causal_L520", L=520, causal=True, sigma_q=3.0)
    inp = make_inputs(w, seed=4)
    a = gpu_run(inp, w, alpha, backward=True, mask64=False)
    b = gpu_run(inp, w, alpha, backward=True, mask64=True)
    for k in ("O", "tau", "dK", "dV"):
        assert np.array_equal(a[k], b[k]), k
    assert np.abs(a["dQ"] - b["dQ"]).max() <= 1e-5
    assert np.array_equal(a["M"], b["M"])
