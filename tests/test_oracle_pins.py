"""Pins for the fp64 oracle: each check compares it with something other than itself.

These checks are closed forms (tests/golden/closed_forms.json), brute-force
support enumeration, a library optimiser on the variational definition,
finite differences, invariants, and dense numpy compositions. Every test runs
on the CPU.
"""
import itertools
import json
import math
import os

import numpy as np
import pytest
from scipy.optimize import brentq, minimize

import oracle

GOLD = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")
ALPHAS = (1.5, 2.0)
GENERAL = (1.25, 3.0)            # alpha outside {1.5, 2}: the oracle takes the bisection of Eq. 4
ALL_ALPHAS = ALPHAS + GENERAL


def _row(vals):
    return np.array([-np.inf if v == "-inf" else float(v) for v in vals])


# --------------------------------------------------------------------------- closed forms
@pytest.mark.parametrize("case", json.load(open(GOLD))["cases"], ids=lambda c: c["name"])
def test_closed_forms(case):
    alpha, s = case["alpha"], _row(case["s"])
    n = int(np.isfinite(s).sum())
    env = {"s": case["s_value"], "n": n, "alpha": alpha, "sqrt": math.sqrt}
    if "tau_score" in case:
        want_eq3 = (alpha - 1) * eval(case["tau_score"], {}, env)
    else:
        want_eq3 = eval(case["tau_eq3"], {}, env)
    methods = (oracle.METHOD_SORT, oracle.METHOD_BISECT) if alpha in ALPHAS else (oracle.METHOD_BISECT,)
    for method in methods + (oracle.METHOD_AUTO,):
        P, tau = oracle.entmax_rows(s[None, :], alpha, method)
        tol = 1e-13 if method == oracle.METHOD_SORT else 1e-12
        assert abs(tau[0] - want_eq3) < tol, (method, tau[0], want_eq3)
        np.testing.assert_allclose(P[0], case["p"], atol=1e-12)


# ------------------------------------------------------------------ brute-force supports
def _brute_tau(z, alpha):
    """Enumerate every support S, root-find sum_{S} (z - t)^{1/(alpha-1)} = 1 with brentq
    (not the closed form), and keep the self-consistent one: min_S z > t >= max_notS z."""
    e = 1.0 / (alpha - 1.0)
    n = len(z)
    found = []
    for k in range(1, n + 1):
        for S in itertools.combinations(range(n), k):
            zS = z[list(S)]
            lo, hi = zS.max() - 1.0 - 1e-9, zS.min()
            g = lambda t: np.sum(np.maximum(zS - t, 0.0) ** e) - 1.0  # noqa: E731
            if g(hi) > 0:   # even at t = min z_S the piece sums to more than 1 -> S too big
                continue
            t = brentq(lambda t: np.sum((zS - t) ** e) - 1.0 if t <= zS.min() else g(t), lo, hi,
                       xtol=1e-15, rtol=1e-15)
            rest = np.delete(z, list(S))
            if zS.min() > t and (rest.size == 0 or t >= rest.max()):
                found.append(t)
    return found


@pytest.mark.parametrize("alpha", ALL_ALPHAS)
@pytest.mark.parametrize("n", [1, 2, 3, 5, 8])
def test_brute_force_supports(alpha, n):
    rng = np.random.default_rng(100 + n)
    for trial in range(6):
        s = rng.normal(0, 1.0 + trial, size=n)
        z = (alpha - 1) * s
        found = _brute_tau(z, alpha)
        assert len(found) == 1, found          # exactly one consistent support (uniqueness)
        if alpha in ALPHAS:
            assert abs(oracle.tau_sort(z, alpha) - found[0]) < 1e-12
        assert abs(oracle.tau_bisect(z, alpha) - found[0]) < 1e-11
        _, tau = oracle.entmax_rows(s[None, :], alpha)   # the row solver the attention uses
        assert abs(tau[0] - found[0]) < 1e-11


# ------------------------------------------------------------ variational definition
def _tsallis_obj(p, s, alpha):
    # p^T s + H_alpha(p), H_alpha(p) = 1/(alpha(alpha-1)) sum_j (p_j - p_j^alpha);
    # alpha = 1.5 gives the 4/3 (p - p^1.5) of the distilbert-mnli model card.
    return p @ s + np.sum(p - np.maximum(p, 0) ** alpha) / (alpha * (alpha - 1))


@pytest.mark.parametrize("alpha", ALL_ALPHAS)
def test_tsallis_argmax(alpha):
    """distilbert-mnli-full-adasplash card, 'Tsallis alpha-Entropy Simplex Formulation':
    entmax is the argmax over the simplex of p^T s + H_alpha(p). Checked two ways:
    random simplex perturbations never do better, and SLSQP finds the same p."""
    rng = np.random.default_rng(7)
    for n in (4, 9, 17):
        s = rng.normal(0, 2.0, size=n)
        P, _ = oracle.entmax_rows(s[None, :], alpha)
        p = P[0]
        best = _tsallis_obj(p, s, alpha)
        for _ in range(2000):
            q = np.abs(p + rng.normal(0, 0.05, size=n) * (rng.random(n) < 0.5))
            q /= q.sum()
            assert _tsallis_obj(q, s, alpha) <= best + 1e-12
        res = minimize(lambda x: -_tsallis_obj(np.maximum(x, 0), s, alpha), np.full(n, 1.0 / n),
                       method="SLSQP", bounds=[(0, 1)] * n,
                       constraints=[{"type": "eq", "fun": lambda x: x.sum() - 1}],
                       options={"ftol": 1e-14, "maxiter": 500})
        np.testing.assert_allclose(res.x, p, atol=2e-5)


def test_sparsemax_is_simplex_projection():
    """alpha = 2 is sparsemax (AdaSplash-2 §2.3, citing Martins & Astudillo): the
    Euclidean projection of s onto the simplex, found here by SLSQP."""
    rng = np.random.default_rng(3)
    for n in (3, 6, 11):
        s = rng.normal(0, 1.0, size=n)
        P, _ = oracle.entmax_rows(s[None, :], 2.0)
        res = minimize(lambda x: np.sum((x - s) ** 2), np.full(n, 1.0 / n), method="SLSQP",
                       bounds=[(0, None)] * n,
                       constraints=[{"type": "eq", "fun": lambda x: x.sum() - 1}],
                       options={"ftol": 1e-15, "maxiter": 500})
        np.testing.assert_allclose(res.x, P[0], atol=1e-6)


# ------------------------------------------------------------------------- invariants
@pytest.mark.parametrize("alpha", ALL_ALPHAS)
def test_row_invariants(alpha):
    rng = np.random.default_rng(11)
    S = rng.normal(0, 2.0, size=(64, 257))
    S[5, 100:] = -np.inf                     # a partly masked row
    P, tau = oracle.entmax_rows(S, alpha)
    assert np.all(P >= 0)
    np.testing.assert_allclose(P.sum(1), 1.0, atol=1e-12)
    z = (alpha - 1) * S
    assert np.array_equal(P > 0, z > tau[:, None])          # p_j = 0 exactly when z_j <= tau
    # Sort-based and bisection solvers agree (§2.4: two different solvers of Eq. 4).
    if alpha in ALPHAS:
        _, tau_b = oracle.entmax_rows(S, alpha, oracle.METHOD_BISECT)
        np.testing.assert_allclose(tau, tau_b, atol=1e-12, rtol=0)
    else:
        f = [oracle.f_root(z[r][np.isfinite(z[r])], alpha, tau[r]) for r in range(S.shape[0])]
        assert np.abs(f).max() < 1e-10
    # Shift invariance: s + c gives the same p and tau shifted by (alpha-1) c.
    P2, tau2 = oracle.entmax_rows(S + 3.25, alpha)
    np.testing.assert_allclose(P2, P, atol=1e-12)
    np.testing.assert_allclose(tau2, tau + (alpha - 1) * 3.25, atol=1e-12)
    # Permutation equivariance.
    perm = rng.permutation(S.shape[1])
    P3, tau3 = oracle.entmax_rows(S[:, perm], alpha)
    np.testing.assert_allclose(P3, P[:, perm], atol=1e-12)
    # tau lies in the §2.4 bracket [m - 1, m - n^{1-alpha}].
    n = np.isfinite(S).sum(1)
    m = z.max(1)
    assert np.all(tau >= m - 1 - 1e-12) and np.all(tau <= m - n ** (1 - alpha) + 1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.75, 3.0])
def test_bisection_general_alpha(alpha):
    """Eq. 4 root for alpha outside {1.5, 2}: f(tau) ~ 0 and tau in the bracket."""
    rng = np.random.default_rng(5)
    s = rng.normal(0, 1.0, size=300)
    z = (alpha - 1) * s
    t = oracle.tau_bisect(z, alpha)
    assert abs(oracle.f_root(z, alpha, t)) < 1e-10
    assert z.max() - 1 <= t <= z.max() - 300 ** (1 - alpha)
    assert math.isnan(oracle.tau_sort(z, alpha))   # the sorting solver covers {1.5, 2} only


# ------------------------------------------------------------------- attention forward
def _dense_masks(L, causal, window, kv_len):
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    act = np.broadcast_to(j < kv_len, (L, L)).copy()
    if window >= 0:
        act &= (j <= i) & ((j == 0) | (i - j <= window))
    elif causal:
        act &= j <= i
    return act


ATTN_CASES = [
    dict(causal=False, window=-1, kv=None),
    dict(causal=True, window=-1, kv=None),
    dict(causal=True, window=3, kv=None),
    dict(causal=False, window=-1, kv=[9, 5]),
]


@pytest.mark.parametrize("alpha", ALL_ALPHAS)
@pytest.mark.parametrize("case", ATTN_CASES, ids=lambda c: f"c{int(c['causal'])}w{c['window']}kv{c['kv']}")
def test_attention_forward_vs_dense_composition(alpha, case):
    """The oracle's row loops against S = scale Q K^T and O = P V done with numpy matmul,
    masks built with numpy (window: model card 'Causal Splash Masking'), and P from the
    pinned row solver."""
    rng = np.random.default_rng(21)
    B, H, L, d = 2, 2, 13, 8
    Q, K, V = (rng.normal(0, s, size=(B, H, L, d)) for s in (2.0, 1.0, 1.0))
    scale = 1 / math.sqrt(d)
    pr = oracle.Problem(Q, K, V, alpha=alpha, scale=scale, causal=case["causal"], window=case["window"],
                        kv_len=case["kv"])
    out = pr.forward()
    for b in range(B):
        kv = L if case["kv"] is None else case["kv"][b]
        act = _dense_masks(L, case["causal"], case["window"], kv)
        for h in range(H):
            S = scale * Q[b, h] @ K[b, h].T
            S[~act] = -np.inf
            P, tau = oracle.entmax_rows(S, alpha)
            np.testing.assert_allclose(out["tau"][b, h], tau, atol=1e-13)
            np.testing.assert_allclose(out["O"][b, h], P @ V[b, h], atol=1e-12)
            G = np.where(P > 0, P ** (2 - alpha), 0.0)
            np.testing.assert_allclose(out["sumg"][b, h], G.sum(1), atol=1e-12)
            np.testing.assert_allclose(out["Ot"][b, h], G @ V[b, h], atol=1e-12)


# ------------------------------------------------------------------ attention backward
def _loss(pr, dO):
    return float(np.sum(pr.forward()["O"] * dO))


@pytest.mark.parametrize("alpha", ALL_ALPHAS)
@pytest.mark.parametrize("case", ATTN_CASES[:3], ids=["full", "causal", "window"])
def test_backward_finite_differences(alpha, case):
    """dQ, dK, dV from the derived Jacobian against central differences of <dO, O>
    (fp64, h = 1e-6). The Jacobian is not printed on the pages (§3.3 only says it lives
    on the support), so this is its pin."""
    rng = np.random.default_rng(31 + int(alpha * 10))
    B, H, L, d = 1, 1, 10, 6
    # Query spread 1.25 / (alpha - 1): z = (alpha-1) s has the same spread at every alpha,
    # so rows keep supports of several keys (nonzero gradients) at alpha = 3 as well.
    Q, K, V, dO = (rng.normal(0, s, size=(B, H, L, d)) for s in (1.25 / (alpha - 1), 1.0, 1.0, 1.0))
    kw = dict(alpha=alpha, scale=1 / math.sqrt(d), causal=case["causal"], window=case["window"])
    g = oracle.Problem(Q, K, V, dO, **kw).backward()
    h = 1e-6
    for name, X in (("dQ", Q), ("dK", K), ("dV", V)):
        fd = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args = {"Q": Q, "K": K, "V": V}
            key = name[1]
            args[key] = Xp
            lp = _loss(oracle.Problem(args["Q"], args["K"], args["V"], **kw), dO)
            args[key] = Xm
            lm = _loss(oracle.Problem(args["Q"], args["K"], args["V"], **kw), dO)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.abs(fd - g[name]).max() / max(1e-3, np.abs(fd).max())
        assert err < 1e-6, (name, err)


def test_backward_sparsemax_jacobian():
    """alpha = 2: the derived Jacobian must equal the textbook sparsemax Jacobian
    diag(1_S) - 1_S 1_S^T / |S| (Martins & Astudillo, cited in AdaSplash-2 §2.3).
    Checked through dQ on a single query row: dQ = scale * K^T J (V dO)."""
    rng = np.random.default_rng(41)
    L, d = 12, 5
    Q, K, V, dO = (rng.normal(0, s, size=(1, 1, L, d)) for s in (3.0, 1.0, 1.0, 1.0))
    scale = 1 / math.sqrt(d)
    g = oracle.Problem(Q, K, V, dO, alpha=2.0, scale=scale).backward()
    for i in range(L):
        s = scale * K[0, 0] @ Q[0, 0, i]
        P, _ = oracle.entmax_rows(s[None, :], 2.0)
        supp = (P[0] > 0).astype(float)
        J = np.diag(supp) - np.outer(supp, supp) / supp.sum()
        dp = V[0, 0] @ dO[0, 0, i]
        np.testing.assert_allclose(g["dQ"][0, 0, i], scale * K[0, 0].T @ (J @ dp), atol=1e-12)


@pytest.mark.parametrize("alpha", ALL_ALPHAS)
def test_backward_invariants(alpha):
    """Gradients vanish off the support (§3.3 'Backward pass'), and the score
    gradient of every row sums to zero (softmax-like shift invariance). So
    sum_j dK_j = scale * sum_i Q_i * (sum_j dS_ij) = 0."""
    rng = np.random.default_rng(51)
    B, H, L, d = 1, 2, 40, 8
    Q, K, V, dO = (rng.normal(0, s, size=(B, H, L, d)) for s in (3.0, 1.0, 1.0, 1.0))
    g = oracle.Problem(Q, K, V, dO, alpha=alpha, scale=1 / math.sqrt(d), causal=True).backward()
    np.testing.assert_allclose(g["dK"].sum(2), 0.0, atol=1e-11)
    # A key that no row keeps in its support gets zero dK and dV.
    pr = oracle.Problem(Q, K, V, dO, alpha=alpha, scale=1 / math.sqrt(d), causal=True)
    f = pr.forward()
    for h in range(H):
        S = (Q[0, h] @ K[0, h].T) / math.sqrt(d)
        S[np.triu(np.ones((L, L), bool), 1)] = -np.inf
        P, _ = oracle.entmax_rows(S, alpha)
        np.testing.assert_allclose(f["tau"][0, h], _, atol=1e-13)
        dead = ~(P > 0).any(0)
        assert dead.any()
        assert np.all(g["dK"][0, h][dead] == 0) and np.all(g["dV"][0, h][dead] == 0)


# -------------------------------------------------------------------------- block mask
@pytest.mark.parametrize("alpha", ALL_ALPHAS)
def test_block_mask_brute_force(alpha):
    """Appendix C.4 packing, against a dense numpy reduction of A > 0 over tiles."""
    rng = np.random.default_rng(61)
    B, H, L, d, Br, Bc = 1, 2, 70, 8, 16, 8
    Q, K, V = (rng.normal(0, s, size=(B, H, L, d)) for s in (4.0, 1.0, 1.0))
    pr = oracle.Problem(Q, K, V, alpha=alpha, scale=1 / math.sqrt(d), causal=True)
    tau = pr.forward()["tau"]
    M, Mlo, Mhi = pr.block_mask(tau, Br, Bc, margin=1e-3)
    Tr, Tc = -(-L // Br), -(-L // Bc)
    for h in range(H):
        S = (Q[0, h] @ K[0, h].T) / math.sqrt(d)
        S[np.triu(np.ones((L, L), bool), 1)] = -np.inf
        P, _ = oracle.entmax_rows(S, alpha)
        for it in range(Tr):
            for jt in range(Tc):
                want = (P[it * Br:(it + 1) * Br, jt * Bc:(jt + 1) * Bc] > 0).any()
                got = bool((M[0, h, it, jt // 32] >> (jt % 32)) & 1)
                assert got == want, (h, it, jt)
    # margin masks bracket the exact one
    assert np.all((Mlo & ~M) == 0) and np.all((M & ~Mhi) == 0)


# ---------------------------------------------------------------- ALiBi (NAPE heads)
# AdaSplash-2 §4.3: NAPE heads use no positional encoding or ALiBi (Press et al.), a
# per-head linear penalty m_h |i - j| subtracted from the scores.
SLOPES = np.array([0.0, 0.25, 0.7])


@pytest.mark.parametrize("alpha", (1.5, 2.0, 1.25))
@pytest.mark.parametrize("causal", (True, False))
def test_alibi_forward_vs_dense_composition(alpha, causal):
    rng = np.random.default_rng(81)
    B, H, L, d = 1, 3, 19, 8
    Q, K, V = (rng.normal(0, s, size=(B, H, L, d)) for s in (1.5, 1.0, 1.0))
    scale = 1 / math.sqrt(d)
    out = oracle.Problem(Q, K, V, alpha=alpha, scale=scale, causal=causal, alibi=SLOPES).forward()
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    for h in range(H):
        S = scale * Q[0, h] @ K[0, h].T - SLOPES[h] * np.abs(i - j)
        if causal:
            S[j > i] = -np.inf
        P, tau = oracle.entmax_rows(S, alpha)
        np.testing.assert_allclose(out["tau"][0, h], tau, atol=1e-13)
        np.testing.assert_allclose(out["O"][0, h], P @ V[0, h], atol=1e-12)
        G = np.where(P > 0, P ** (2 - alpha), 0.0)
        np.testing.assert_allclose(out["Ot"][0, h], G @ V[0, h], atol=1e-12)
    # A zero slope is no bias at all.
    plain = oracle.Problem(Q, K, V, alpha=alpha, scale=scale, causal=causal).forward()
    np.testing.assert_allclose(out["O"][0, 0], plain["O"][0, 0], atol=1e-14)


@pytest.mark.parametrize("m", (0.3, 0.8, 1.5))
def test_alibi_two_keys_sparsemax_closed_form(m):
    """Q = 0 makes every raw score 0, so row 1 of a causal head sees the biased scores
    (-m, 0). At alpha = 2 (sparsemax, Eq. 3) two scores a < b give p = ((1-(b-a))/2,
    (1+(b-a))/2) while b - a < 1, and (0, 1) beyond."""
    L, d = 2, 4
    Q = np.zeros((1, 1, L, d))
    rng = np.random.default_rng(3)
    K, V = rng.normal(size=(1, 1, L, d)), rng.normal(size=(1, 1, L, d))
    out = oracle.Problem(Q, K, V, alpha=2.0, scale=0.5, causal=True, alibi=[m]).forward()
    p0 = max(0.0, (1 - m) / 2)
    p = np.array([p0, 1 - p0])
    np.testing.assert_allclose(out["O"][0, 0, 1], p @ V[0, 0], atol=1e-14)
    np.testing.assert_allclose(out["tau"][0, 0, 1], (-m - 1) / 2 if m < 1 else -1.0, atol=1e-14)


@pytest.mark.parametrize("alpha", (1.5, 1.25))
def test_alibi_backward_finite_differences(alpha):
    """The bias has no parameters, so the Jacobian formulas are unchanged; central
    differences of <dO, O> check dQ, dK, dV with ALiBi on."""
    rng = np.random.default_rng(91)
    B, H, L, d = 1, 2, 9, 5
    Q, K, V, dO = (rng.normal(0, s, size=(B, H, L, d)) for s in (1.25 / (alpha - 1), 1.0, 1.0, 1.0))
    kw = dict(alpha=alpha, scale=1 / math.sqrt(d), causal=True, alibi=[0.2, 0.6])
    g = oracle.Problem(Q, K, V, dO, **kw).backward()
    h = 1e-6
    for name, X in (("dQ", Q), ("dK", K), ("dV", V)):
        fd = np.zeros_like(X)
        for idx in np.ndindex(X.shape):
            Xp, Xm = X.copy(), X.copy()
            Xp[idx] += h
            Xm[idx] -= h
            args = {"Q": Q, "K": K, "V": V}
            args[name[1]] = Xp
            lp = _loss(oracle.Problem(args["Q"], args["K"], args["V"], **kw), dO)
            args[name[1]] = Xm
            lm = _loss(oracle.Problem(args["Q"], args["K"], args["V"], **kw), dO)
            fd[idx] = (lp - lm) / (2 * h)
        err = np.abs(fd - g[name]).max() / max(1e-3, np.abs(fd).max())
        assert err < 1e-6, (name, err)


def test_alibi_block_mask_brute_force():
    rng = np.random.default_rng(97)
    B, H, L, d, Br, Bc = 1, 2, 70, 8, 16, 8
    Q, K, V = (rng.normal(0, s, size=(B, H, L, d)) for s in (2.0, 1.0, 1.0))
    pr = oracle.Problem(Q, K, V, alpha=1.5, scale=1 / math.sqrt(d), causal=True, alibi=[0.1, 0.5])
    tau = pr.forward()["tau"]
    M, _, _ = pr.block_mask(tau, Br, Bc)
    i = np.arange(L)[:, None]
    j = np.arange(L)[None, :]
    for h, m in enumerate((0.1, 0.5)):
        S = (Q[0, h] @ K[0, h].T) / math.sqrt(d) - m * np.abs(i - j)
        S[j > i] = -np.inf
        P, _ = oracle.entmax_rows(S, 1.5)
        for it in range(-(-L // Br)):
            for jt in range(-(-L // Bc)):
                want = (P[it * Br:(it + 1) * Br, jt * Bc:(jt + 1) * Bc] > 0).any()
                assert bool((M[0, h, it, jt // 32] >> (jt % 32)) & 1) == want


# ---------------------------------------------------------------- histogram initialisation
def _hist_root_brute(z, alpha, B):
    """The root of the histogram objective of AdaSplash-2 §3.1, written out directly: shift
    so that max z = 1, replace each score in [0, 1] by the left edge of its bin
    min(floor(B z), B - 1) / B, and bisect f_h(t) = -1 + sum [edge - t]_+^{1/(alpha-1)}."""
    z = np.asarray(z, dtype=np.float64)
    m = z.max()
    zt = z - (m - 1.0)
    zt = zt[zt >= 0]
    edges = np.minimum(np.floor(B * zt), B - 1) / B
    e = 1.0 / (alpha - 1.0)
    lo, hi = -1.0 / B, 1.0
    for _ in range(200):
        mid = 0.5 * (lo + hi)
        f = -1.0 + np.sum(np.clip(edges - mid, 0.0, None) ** e)
        lo, hi = (mid, hi) if f > 0 else (lo, mid)
    return 0.5 * (lo + hi) + (m - 1.0)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
@pytest.mark.parametrize("B", [4, 8, 16, 64])
def test_histogram_bound_proposition(alpha, B):
    """Proposition 3.1 (AdaSplash-2 §3.2): tau* - 1/B <= tau_h <= tau*, on rows of several
    sizes and spreads, with tau* from the exact solvers of §2.4 (a different algorithm).
    The page states the left inequality strictly, but its proof needs z < edge + 1/B for
    every score, which fails for the row maximum: the clamp min(floor(B z), B - 1) puts
    z = 1 exactly 1/B above its edge. When the support is that maximum alone (a dominant
    key), tau_h = tau* - 1/B; otherwise the inequality is strict."""
    rng = np.random.default_rng(11)
    for n in (1, 2, 7, 64, 4096):
        for spread in (0.05, 0.5, 3.0):
            z = (alpha - 1.0) * rng.normal(size=n) * spread
            ts = oracle.tau_sort(z, alpha) if alpha in (1.5, 2.0) else oracle.tau_bisect(z, alpha)
            th = oracle.tau_hist(z, alpha, B)
            assert ts - 1.0 / B - 1e-12 <= th <= ts + 1e-12, (n, spread, ts, th)
            single = np.sum(z > ts + 1e-12) <= 1   # support = the maximum alone
            if not single:
                assert ts - 1.0 / B < th, (n, spread, ts, th)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 3.0])
def test_histogram_solve_matches_brute_force(alpha):
    """The oracle's exact solve on bin counts (α in {1.5, 2}) or bisection on bins gives the
    root of the histogram objective computed directly from the binned scores."""
    rng = np.random.default_rng(5)
    for n, B in ((3, 4), (50, 8), (1000, 16), (4096, 8)):
        z = rng.normal(size=n) * 0.7
        assert abs(oracle.tau_hist(z, alpha, B) - _hist_root_brute(z, alpha, B)) < 1e-9


def test_histogram_converges_with_bins():
    """tau_h -> tau* as B grows (error below 1/B for B up to 2^14)."""
    rng = np.random.default_rng(3)
    z = 0.5 * rng.normal(size=2000)
    ts = oracle.tau_sort(z, 1.5)
    for k in range(2, 15):
        B = 2 ** k
        assert 0.0 <= ts - oracle.tau_hist(z, 1.5, B) < 1.0 / B
