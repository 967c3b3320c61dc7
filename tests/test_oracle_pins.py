"""Pins of the float64 oracle against facts that do not come from the oracle.

Closed forms, exact rational arithmetic, brute-force enumeration, numerical
quadrature, a library rounding routine, the variational definition of
α-entmax and the invariants stated by the source page ("Résumé Technique :
EntmaxKV", §2–§3).  CPU only.
"""
import itertools
import math
import os
from fractions import Fraction

import numpy as np
import pytest
import torch
from scipy import integrate, optimize

import oracle as O

HERE = os.path.dirname(os.path.abspath(__file__))


# ---------------------------------------------------------------- rounding
def test_round_bf16_matches_torch_fp32_to_bf16():
    rng = np.random.default_rng(1)
    x32 = np.concatenate([
        rng.standard_normal(20000).astype(np.float32),
        (rng.standard_normal(2000) * 1e-38).astype(np.float32),   # bf16 subnormal range
        (rng.standard_normal(2000) * 1e30).astype(np.float32),
    ])
    # exact ties between two bf16 neighbours (bit 15 set, lower bits clear)
    ties = (rng.integers(0, 2 ** 16, 4000, dtype=np.uint32) << 16) | np.uint32(0x8000)
    ties = ties[(ties & 0x7F800000) != 0x7F800000]
    x32 = np.concatenate([x32, ties.view(np.float32)])
    want = torch.from_numpy(x32).to(torch.bfloat16).double().numpy()
    got = O.round_bf16(x32.astype(np.float64))
    assert np.array_equal(got, want)


def test_round_bf16_hand_cases():
    cases = {1 + 2 ** -8: 1.0, 1 + 3 * 2 ** -8: 1 + 2 ** -6, 2 - 2 ** -9: 2.0,
             1.5 * 2 ** -133: 2 ** -132, 2.5 * 2 ** -133: 2 ** -132, -(1 + 2 ** -8 + 2 ** -40): -(1 + 2 ** -7)}
    for x, y in cases.items():
        assert O.round_bf16(np.array([x]))[0] == y, x


def _exact_round(v: Fraction, dtype: str) -> float:
    """Round a rational to the nearest bf16 / fp32 value, ties to even (exact)."""
    if v == 0:
        return 0.0
    sign = -1 if v < 0 else 1
    a = abs(v)
    e = math.floor(math.log2(a.numerator) - math.log2(a.denominator)) + 1
    while Fraction(2) ** (e - 1) > a:
        e -= 1
    while Fraction(2) ** e <= a:
        e += 1
    bits, emin = (8, -133) if dtype == "bf16" else (24, -149)
    qexp = max(e - bits, emin)
    r = a / Fraction(2) ** qexp
    fl = r.numerator // r.denominator
    rem = r - fl
    if rem > Fraction(1, 2) or (rem == Fraction(1, 2) and fl % 2 == 1):
        fl += 1
    return sign * float(Fraction(fl) * Fraction(2) ** qexp)


@pytest.mark.parametrize("dtype", ["bf16", "f32"])
def test_metadata_against_exact_rationals(dtype):
    g = torch.Generator().manual_seed(7)
    P, S, d = 40, 8, 5
    tdt = torch.bfloat16 if dtype == "bf16" else torch.float32
    k = (torch.randn(P, S, d, generator=g) * torch.exp(torch.randn(P, 1, d, generator=g))).to(tdt).double().numpy()
    n_valid = torch.randint(1, S + 1, (P,), generator=g).numpy()
    meta = O.page_metadata(k, n_valid, dtype)
    mism = 0
    for p in range(P):
        n = int(n_valid[p])
        for j in range(d):
            xs = [Fraction(float(k[p, t, j])) for t in range(n)]
            mean = sum(xs) / n
            var = sum((x - mean) ** 2 for x in xs) / n
            assert meta["kmax"][p, j] == float(max(xs))
            assert meta["kmin"][p, j] == float(min(xs))
            for name, val in (("mean", mean), ("var", var)):
                want = _exact_round(val, dtype)
                got = meta[name][p, j]
                if dtype == "bf16":
                    assert got == want, (name, p, j)   # fp64 sums of bf16 are exact here
                elif got != want:
                    mism += 1                          # fp32 input: fp64 rounding may differ by 1 ulp
                    assert abs(got - want) <= np.spacing(np.float32(abs(want))), (name, p, j)
    assert mism <= 2


def test_metadata_variance_is_population_and_single_token_zero():
    k = np.array([[[1.0, 2.0], [3.0, 2.0], [5.0, 9.0]]])
    m = O.page_metadata(k, [3], "f32")
    assert m["mean"][0].tolist() == [3.0, pytest.approx(13 / 3, rel=1e-7)]
    assert m["var"][0, 0] == pytest.approx(8 / 3, rel=1e-7)        # divides by n, not n − 1
    m1 = O.page_metadata(k, [1], "f32")
    assert m1["var"][0].tolist() == [0.0, 0.0] and m1["kmax"][0].tolist() == [1.0, 2.0]


# ---------------------------------------------------------------- bound / top-k
def test_bound_dominates_every_token_score():
    rng = np.random.default_rng(3)
    for trial in range(20):
        G, P, S, d = 4, 30, 16, 32
        q = rng.standard_normal((G, d))
        K = rng.standard_normal((P, S, d)) * rng.exponential(1.0, (P, 1, d)) + rng.standard_normal((P, 1, d))
        n_valid = rng.integers(1, S + 1, P)
        meta = O.page_metadata(K, n_valid, "f32")
        # exact stored bounds must hold on the unrounded keys (min/max are exact)
        ub = O.bbox_upper_bound(q, meta["kmax"], meta["kmin"], 0.25)
        for p in range(P):
            z = 0.25 * q @ K[p, : n_valid[p]].T                      # [G, n]
            slack = 1e-12 * 0.25 * (np.abs(q) @ np.abs(K[p, : n_valid[p]]).T)
            assert np.all(ub[:, p, None] >= z - slack)
            # the bound is tight on at least the box corner: ub ≥ max z, and equal for n=1
            if n_valid[p] == 1:
                assert np.allclose(ub[:, p], z[:, 0], rtol=1e-12, atol=1e-12)


def test_bound_sign_convention():
    # one coordinate: q>0 uses kmax, q<0 uses kmin
    ub = O.bbox_upper_bound(np.array([[2.0], [-3.0]]), np.array([[5.0]]), np.array([[-1.0]]), 1.0)
    assert ub[:, 0].tolist() == [10.0, 3.0]


def test_page_size_one_topk_equals_token_topk():
    rng = np.random.default_rng(5)
    G, T, d = 3, 200, 16
    q = rng.standard_normal((G, d))
    K = rng.standard_normal((T, 1, d))
    meta = O.page_metadata(K, np.ones(T, int), "f32")
    ub = O.bbox_upper_bound(q, meta["kmax"], meta["kmin"], 0.5)
    z = 0.5 * q @ K[:, 0].T
    assert np.allclose(ub, z, rtol=1e-12, atol=1e-13)
    score = O.page_scores(ub)
    want = np.sort(np.argsort(-z.max(0))[:17])
    assert np.array_equal(O.select_topk(score, 17), want)


def test_topk_bruteforce_with_ties():
    rng = np.random.default_rng(11)
    for trial in range(200):
        P = int(rng.integers(1, 60))
        s = rng.integers(-5, 6, P).astype(float)
        k = int(rng.integers(1, 70))
        want = sorted(sorted(range(P), key=lambda i: (-s[i], i))[:k])
        assert O.select_topk(s, k).tolist() == want


# ---------------------------------------------------------------- entmax
def _golden_rows():
    rows = []
    with open(os.path.join(HERE, "golden", "entmax_closed_forms.txt")) as f:
        for line in f:
            if line.startswith("#") or not line.strip():
                continue
            a, z, p, _ = [x.strip() for x in line.split("|")]
            rows.append((float(a), np.array(z.split(), float), np.array(p.split(), float)))
    return rows


@pytest.mark.parametrize("row", _golden_rows())
def test_entmax_golden_closed_forms(row):
    alpha, z, p_want = row
    for method in ([None, "bisect"] if alpha in O.ENTMAX_SORT_ALPHAS else [None]):
        p, _ = O.entmax_probs(z, alpha, method)
        assert np.allclose(p, p_want, rtol=0, atol=1e-12), (method, p)


def test_sparsemax_two_element_closed_form():
    rng = np.random.default_rng(2)
    for z in rng.standard_normal((300, 2)) * 2:
        p, _ = O.entmax_probs(z, 2.0)
        p1 = min(max((z[0] - z[1] + 1) / 2, 0.0), 1.0)
        assert p[0] == pytest.approx(p1, abs=1e-12) and p[1] == pytest.approx(1 - p1, abs=1e-12)


def test_entmax15_two_element_closed_form():
    rng = np.random.default_rng(4)
    for z in rng.standard_normal((300, 2)) * 3:
        p, _ = O.entmax_probs(z, 1.5)
        D = abs(z[0] - z[1]) / 2
        top = ((D + math.sqrt(2 - D * D)) / 2) ** 2 if D < 1 else 1.0
        hi = 0 if z[0] >= z[1] else 1
        assert p[hi] == pytest.approx(top, abs=1e-12)
        assert p[1 - hi] == pytest.approx(1 - top, abs=1e-12)


def _tsallis_objective(p, z, alpha):
    return p @ z + (np.sum(p - p ** alpha)) / (alpha * (alpha - 1))


@pytest.mark.parametrize("alpha", [1.25, 1.5, 1.7, 2.0, 3.0])
def test_entmax_is_the_variational_maximiser(alpha):
    """α-entmax(z) = argmax_{p ∈ simplex} p·z + H^T_α(p) (Tsallis entropy)."""
    rng = np.random.default_rng(int(alpha * 100))
    for trial in range(30):
        n = int(rng.integers(2, 40))
        z = rng.standard_normal(n) * rng.uniform(0.5, 4)
        p, _ = O.entmax_probs(z, alpha)
        assert np.all(p >= 0) and abs(p.sum() - 1) < 1e-12
        best = _tsallis_objective(p, z, alpha)
        for eps in (1e-1, 1e-2, 1e-4):
            for r in rng.dirichlet(np.ones(n) * 0.3, 20):
                pp = (1 - eps) * p + eps * r
                assert _tsallis_objective(pp, z, alpha) <= best + 1e-13


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 1.8])
def test_entmax_bruteforce_support_enumeration(alpha):
    beta = 1 / (alpha - 1)
    rng = np.random.default_rng(17)
    for trial in range(40):
        n = int(rng.integers(1, 9))
        u = (alpha - 1) * rng.standard_normal(n) * rng.uniform(0.3, 3)
        found = []
        for r in range(1, n + 1):
            for S in itertools.combinations(range(n), r):
                us = u[list(S)]
                lo_edge = us.min()
                g = lambda t: np.sum((us - t) ** beta) - 1
                if g(lo_edge) > 0:          # all of S stays active beyond the root: no root below min
                    continue
                tau = optimize.brentq(g, lo_edge - 2.0, lo_edge, xtol=1e-15, rtol=1e-15)
                outside = np.delete(u, list(S))
                if tau < lo_edge and (outside.size == 0 or tau >= outside.max()):
                    found.append((set(S), tau))
        assert len(found) == 1, found
        tau_o = O.entmax_threshold(u, alpha)
        assert tau_o == pytest.approx(found[0][1], abs=1e-11)
        assert set(np.nonzero(u > tau_o)[0].tolist()) == found[0][0]


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_sort_forms_match_bisection(alpha):
    rng = np.random.default_rng(23)
    for trial in range(100):
        z = rng.standard_normal(int(rng.integers(1, 500))) * rng.uniform(0.1, 10)
        u = (alpha - 1) * z
        assert O.entmax_threshold(u, alpha, "sort") == pytest.approx(
            O.entmax_threshold(u, alpha, "bisect"), abs=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_entmax_shift_and_permutation(alpha):
    rng = np.random.default_rng(29)
    for trial in range(30):
        z = rng.standard_normal(50) * 2
        p, _ = O.entmax_probs(z, alpha)
        p2, _ = O.entmax_probs(z + 3.7, alpha)
        assert np.allclose(p, p2, atol=1e-12)
        perm = rng.permutation(50)
        p3, _ = O.entmax_probs(z[perm], alpha)
        assert np.allclose(p3, p[perm], atol=1e-12)


# ---------------------------------------------------------------- Gaussian policy
def _quad_expect(mu, sigma, tau, beta):
    c = (tau - mu) / sigma
    lo, hi = max(c, -40.0), max(c, 0.0) + 40.0       # φ is below 1e-300 outside
    pts = [x for x in (-5.0, 0.0, 5.0) if lo < x < hi]
    val, _ = integrate.quad(lambda x: (x - c) ** beta * math.exp(-0.5 * x * x) / math.sqrt(2 * math.pi),
                            lo, hi, points=pts or None, epsabs=1e-15, epsrel=1e-12, limit=400)
    return sigma ** beta * val


def test_gauss_truncated_power_mean_vs_quadrature():
    rng = np.random.default_rng(31)
    for trial in range(400):
        beta = int(rng.integers(1, 5))
        mu, sigma, tau = rng.uniform(-2, 2), rng.uniform(0.05, 2), rng.uniform(-3, 3)
        got = float(O.gauss_truncated_power_mean(mu, sigma, tau, beta))
        want = _quad_expect(mu, sigma, tau, beta)
        scale = sigma ** beta + abs(mu - tau) ** beta
        assert abs(got - want) <= 1e-9 * abs(want) + 1e-12 * scale, (mu, sigma, tau, beta, got, want)


def test_gauss_truncated_power_mean_small_sigma_limit():
    for beta in (1, 2, 3, 4):
        for mu, tau in ((0.7, 0.2), (0.1, 0.5)):
            got = float(O.gauss_truncated_power_mean(mu, 1e-9, tau, beta))
            assert got == pytest.approx(max(mu - tau, 0) ** beta, abs=1e-8)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_gauss_tau_hat_zero_variance_is_exact_entmax(alpha):
    """Identical tokens inside each page: the Gaussian model is exact, so τ̂
    equals α-entmax's τ on the page scores repeated n_p times."""
    beta = round(1 / (alpha - 1))
    rng = np.random.default_rng(37)
    for trial in range(20):
        P = int(rng.integers(1, 60))
        mu_u = (alpha - 1) * rng.standard_normal(P) * 2
        n = rng.integers(1, 17, P)
        tokens = np.repeat(mu_u, n)
        want = O.entmax_threshold(tokens, alpha)
        assert O.gauss_tau_hat(mu_u, np.zeros(P), n, beta) == pytest.approx(want, abs=1e-12)
        assert O.gauss_tau_hat(mu_u, np.full(P, 1e-10), n, beta) == pytest.approx(want, abs=1e-8)


def test_gauss_tau_hat_solves_the_equation_by_quadrature():
    rng = np.random.default_rng(41)
    for beta in (1, 2, 4):
        P = 25
        mu, sig, n = rng.standard_normal(P), rng.uniform(0.05, 0.6, P), rng.integers(1, 17, P)
        tau = O.gauss_tau_hat(mu, sig, n, beta)
        total = sum(n[p] * _quad_expect(mu[p], sig[p], tau, beta) for p in range(P))
        assert total == pytest.approx(1.0, abs=1e-9)


def test_gauss_selection_monotone_in_delta_and_limits():
    rng = np.random.default_rng(43)
    G, P, d = 4, 120, 32
    q = rng.standard_normal((G, d))
    mean = rng.standard_normal((P, d))
    var = rng.uniform(0.01, 0.2, (P, d))
    n = rng.integers(1, 17, P)
    prev = None
    for delta in (-1.0, 0.0, 0.25, 0.5, 1.0, 2.0):
        sel = O.select_gauss(q, mean, var, n, 0.2, 1.5, delta)["sel"]
        if prev is not None:
            assert set(prev) <= set(sel.tolist())
        prev = sel.tolist()
    assert O.select_gauss(q, mean, var, n, 0.2, 1.5, 1e9)["sel"].tolist() == list(range(P))
    gs = O.select_gauss(q, mean, var, n, 0.2, 1.5, -1e9)
    assert gs["sel"].tolist() == [int(np.argmax(gs["margin"].max(0)))]


def test_gauss_score_moments_match_the_page_tokens():
    """m and s are the mean and standard deviation of the page's token scores
    when the keys vary along independent coordinates (here: one coordinate)."""
    rng = np.random.default_rng(61)
    q = np.array([[0.3, -2.5, 1.7, 0.9], [1.1, 0.4, -0.6, 2.0]])
    n = 16
    K = np.tile(rng.standard_normal(4), (n, 1))
    K[:, 2] += rng.standard_normal(n) * 0.7
    meta = O.page_metadata(K[None], [n], "f32")
    gs = O.select_gauss(q, meta["mean"], meta["var"], [n], 0.5, 1.5, 0.0)
    z = 0.5 * q @ K.T
    assert np.allclose(gs["m"][:, 0], z.mean(axis=1), rtol=1e-6)
    assert np.allclose(gs["s"][:, 0], z.std(axis=1), rtol=1e-6)


def test_gauss_estimated_max_bounds_the_expected_max():
    """ŝ = m + s·√(2 ln n) upper-bounds E[max of n Gaussian scores] (and is
    within a modest factor of it); n = 1 gives ŝ = m."""
    rng = np.random.default_rng(67)
    for n in (1, 2, 4, 16, 32):
        mean, var = np.array([[0.2]]), np.array([[0.09]])
        gs = O.select_gauss(np.array([[1.0]]), mean, var, [n], 1.0, 2.0, 0.0)
        m, s, shat = gs["m"][0, 0], gs["s"][0, 0], gs["shat"][0, 0]
        draws = m + s * rng.standard_normal((200000, n))
        emax = draws.max(axis=1).mean()
        if n == 1:
            assert shat == pytest.approx(m)
        else:
            assert emax <= shat and (shat - m) <= 2.2 * (emax - m)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_gauss_zero_variance_selects_exactly_the_support_pages(alpha):
    """Identical tokens per page and Δ = 0: the kept pages are exactly those
    holding α-entmax support tokens."""
    rng = np.random.default_rng(71)
    for trial in range(20):
        P, d = 50, 8
        q = rng.standard_normal((1, d))
        mean = O.round_to(rng.standard_normal((P, d)), "f32")
        n = rng.integers(1, 17, P)
        gs = O.select_gauss(q, mean, np.zeros((P, d)), n, 0.4, alpha, 0.0)
        u_pages = (alpha - 1) * 0.4 * (q @ mean.T)[0]
        tau = O.entmax_threshold(np.repeat(u_pages, n), alpha)
        want = np.nonzero(u_pages > tau + 1e-12)[0]
        got = gs["sel"]
        ambiguous = np.abs(u_pages - tau) <= 1e-10
        assert np.array_equal(np.setdiff1d(got, np.nonzero(ambiguous)[0]), want)


# ---------------------------------------------------------------- §3 guarantees
def _random_unit(rng, P=40, S=8, d=16, G=3, L=None):
    L = L or P * S - 3
    k_pool = (rng.standard_normal((P, 1, 1, d)) + 0.3 * rng.standard_normal((P, 1, S, d)))
    v_pool = rng.standard_normal((P, 1, S, d))
    q = rng.standard_normal((G, d)) * 1.5
    return k_pool, v_pool, np.arange(P), L, q


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_exactness_when_selection_contains_support(alpha):
    """[EntmaxKV] §3 'Récupération du Support': S ⊆ I_keep ⇒ identical output."""
    rng = np.random.default_rng(47)
    for trial in range(10):
        k_pool, v_pool, pt, L, q = _random_unit(rng)
        kw = dict(page_size=8, scale=0.25, alpha=alpha, dtype="f32")
        full = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="all", **kw)
        support_pages = set(full["token_page"][np.any(full["p"] > 0, axis=0)].tolist())
        extra = set(rng.choice(len(full["n_valid"]), 5).tolist())
        sel = sorted(support_pages | extra)
        sparse = O.decode_unit(k_pool, v_pool, pt, L, 0, q, sel=sel, **kw)
        assert np.allclose(sparse["tau"], full["tau"], rtol=0, atol=1e-12)
        assert np.allclose(sparse["o"], full["o"], rtol=0, atol=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_error_bound_two_B_delta(alpha):
    """[EntmaxKV] §3 'Borne d'Erreur': ‖o − õ‖ ≤ 2·B·δ."""
    rng = np.random.default_rng(53)
    for trial in range(20):
        k_pool, v_pool, pt, L, q = _random_unit(rng)
        kw = dict(page_size=8, scale=0.25, alpha=alpha, dtype="f32")
        full = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="all", **kw)
        P = len(full["n_valid"])
        sel = np.sort(rng.choice(P, int(rng.integers(1, P)), replace=False))
        sparse = O.decode_unit(k_pool, v_pool, pt, L, 0, q, sel=sel, **kw)
        kept = np.isin(full["token_page"], sel)
        delta = full["p"][:, ~kept].sum(axis=1)
        V = np.concatenate([v_pool[p, 0, : full["n_valid"][p]] for p in range(P)])
        B = np.linalg.norm(V, axis=1).max()
        err = np.linalg.norm(full["o"] - sparse["o"], axis=1)
        assert np.all(err <= 2 * B * delta + 1e-12)


@pytest.mark.parametrize("alpha", [1.5, 2.0])
def test_threshold_monotone_and_bound_certificate(alpha):
    """τ over a subset never exceeds τ over the full set, and when every
    unselected page's bound sits at or below the subset τ, sparse = full."""
    rng = np.random.default_rng(59)
    certified = 0
    for trial in range(40):
        k_pool, v_pool, pt, L, q = _random_unit(rng)
        kw = dict(page_size=8, scale=0.25, alpha=alpha, dtype="f32")
        full = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="all", **kw)
        sparse = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="topk", k=int(rng.integers(1, 20)), **kw)
        assert np.all(sparse["tau"] <= full["tau"] + 1e-12)
        rest = np.setdiff1d(np.arange(len(full["n_valid"])), sparse["sel"])
        if rest.size == 0:
            continue
        cert = (alpha - 1) * sparse["ub"][:, rest].max(axis=1) <= sparse["tau"]
        for h in np.nonzero(cert)[0]:
            certified += 1
            assert np.allclose(sparse["o"][h], full["o"][h], atol=1e-12)
    assert certified > 0


# ---------------------------------------------------------------- softmax attention (full-cache baseline)
def test_softmax_attention_matches_scipy_and_two_token_closed_form():
    """The dense softmax decode of the full-cache baseline ([EntmaxKV] §4):
    weights against scipy's softmax, the two-token case against the logistic
    function, and invariance to shifting every score."""
    from scipy.special import softmax, expit
    rng = np.random.default_rng(7)
    q = rng.normal(size=(3, 16))
    K = rng.normal(size=(50, 16))
    V = rng.normal(size=(50, 16))
    scale = 0.25
    r = O.softmax_attention(q, K, V, scale)
    w = softmax(scale * (q @ K.T), axis=1)
    assert np.allclose(r["p"], w, rtol=1e-13, atol=1e-15)
    assert np.allclose(r["o"], w @ V, rtol=1e-12, atol=1e-13)
    # two tokens: weight of the first = logistic(z1 − z2)
    K2 = rng.normal(size=(2, 16))
    r2 = O.softmax_attention(q, K2, np.eye(2, 16), scale)
    z = scale * (q @ K2.T)
    assert np.allclose(r2["p"][:, 0], expit(z[:, 0] - z[:, 1]), rtol=1e-13)
    # adding c·q to every key shifts every score of a head equally: nothing changes
    r3 = O.softmax_attention(q[:1], K + 0.0, V, scale)
    Ks = K + 3.0 * q[0] / (q[0] @ q[0])
    r4 = O.softmax_attention(q[:1], Ks, V, scale)
    assert np.allclose(r3["o"], r4["o"], rtol=1e-11, atol=1e-12)


def test_entmax_tends_to_softmax_as_alpha_tends_to_one():
    """α-entmax → softmax as α → 1⁺ (the Tsallis family's limit): the gap
    shrinks in proportion to α − 1, tying the two oracle functions together."""
    from scipy.special import softmax
    rng = np.random.default_rng(11)
    z = rng.normal(size=40)
    gaps = []
    for eps in (1e-2, 1e-3, 1e-4):
        p, _ = O.entmax_probs(z, 1.0 + eps)
        gaps.append(np.abs(p - softmax(z)).max())
    assert gaps[2] < 1e-4 and gaps[1] < 1e-3
    assert 5 < gaps[0] / gaps[1] < 20 and 5 < gaps[1] / gaps[2] < 20


# ---------------------------------------------------------------- exactness certificate (unit scores)
@pytest.mark.parametrize("alpha", [1.5, 2.0, 1.25])
def test_unit_score_certificate_implies_full_cache_output(alpha):
    """[EntmaxKV] §3: a head certified from the unit's page scores (the bound
    maximised over the group) has the full-cache output exactly; the test
    sees both certified and uncertified heads."""
    rng = np.random.default_rng(61)
    seen = {True: 0, False: 0}
    for trial in range(40):
        k_pool, v_pool, pt, L, q = _random_unit(rng)
        kw = dict(page_size=8, scale=0.25, alpha=alpha, dtype="f32")
        full = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="all", **kw)
        sparse = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="topk", k=int(rng.integers(1, 30)), **kw)
        cert = O.exactness_certificate(sparse["score"], sparse["sel"], sparse["tau"], alpha)
        for h in range(q.shape[0]):
            seen[bool(cert[h])] += 1
            if cert[h]:
                assert np.allclose(sparse["o"][h], full["o"][h], atol=1e-12)
                assert abs(sparse["tau"][h] - full["tau"][h]) <= 1e-12
    assert seen[True] > 0 and seen[False] > 0


def test_adaptive_budget_reaches_the_full_cache_output():
    """Doubling k until every head is certified ends at the full-cache output,
    and the budget before the last doubling was not certified."""
    rng = np.random.default_rng(67)
    for trial in range(15):
        k_pool, v_pool, pt, L, q = _random_unit(rng)
        kw = dict(page_size=8, scale=0.25, alpha=1.5, dtype="f32")
        full = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="all", **kw)
        k, r = O.adaptive_topk(k_pool, v_pool, pt, L, 0, q, k0=2, **kw)
        assert np.allclose(r["o"], full["o"], atol=1e-12)
        if k > 2:
            prev = O.decode_unit(k_pool, v_pool, pt, L, 0, q, policy="topk", k=k // 2, **kw)
            assert not np.all(O.exactness_certificate(prev["score"], prev["sel"], prev["tau"], 1.5))


# ---------------------------------------------------------------- paged cache plumbing
def _paged_from_flat(rng, lens, S, Hkv, d, spare=2):
    """A paged pool built from flat per-sequence token arrays through a random
    page table (a permutation of a shared pool with spare pages per sequence),
    plus the flat arrays themselves: tokens[b] is [Hkv, n_pages·S, d]."""
    n_pages = [-(-L // S) + spare for L in lens]
    num_phys = sum(n_pages)
    perm = rng.permutation(num_phys)
    max_pages = max(n_pages)
    page_table = np.zeros((len(lens), max_pages), np.int64)
    k_pool = np.zeros((num_phys, Hkv, S, d))
    v_pool = np.zeros((num_phys, Hkv, S, d))
    flat_k, flat_v, off = [], [], 0
    for b, P in enumerate(n_pages):
        page_table[b, :P] = perm[off:off + P]
        off += P
        fk = O.round_bf16(rng.normal(size=(Hkv, P * S, d)))
        fv = O.round_bf16(rng.normal(size=(Hkv, P * S, d)))
        flat_k.append(fk)
        flat_v.append(fv)
        for p in range(P):
            k_pool[page_table[b, p]] = fk[:, p * S:(p + 1) * S]
            v_pool[page_table[b, p]] = fv[:, p * S:(p + 1) * S]
    return k_pool, v_pool, page_table, flat_k, flat_v


def _flat_of(pool, page_table_row, P):
    """Read a sequence back out of the pool: its pages in logical order."""
    return np.concatenate([pool[page_table_row[p]] for p in range(P)], axis=1)


def test_append_token_writes_position_L_minus_1_of_the_flat_sequence():
    """[EntmaxKV] §2.A: the cache grows by one token per decode step.  After
    append_token, reading each sequence back through its page table must give
    the flat token array with exactly token L−1 replaced (L = the length that
    already counts the new token), whatever slot of whatever page that is: a
    mid-page slot, slot 0 of a fresh page and the last slot of a page are all
    in the batch.  The returned n_valid is the page's token count after it."""
    rng = np.random.default_rng(71)
    S, Hkv, d = 8, 3, 5
    lens = [13, 17, 24, 1, 9]          # slots 4, 0 (fresh page), 7 (last), 0 (first token), 0
    k_pool, v_pool, pt, flat_k, flat_v = _paged_from_flat(rng, lens, S, Hkv, d)
    before_k, before_v = k_pool.copy(), v_pool.copy()
    k_new = O.round_bf16(rng.normal(size=(len(lens), Hkv, d)))
    v_new = O.round_bf16(rng.normal(size=(len(lens), Hkv, d)))
    touched = O.append_token(k_pool, v_pool, pt, lens, k_new, v_new, S)
    assert [t[0] for t in touched] == list(range(len(lens)))
    changed_pages = set()
    for b, L in enumerate(lens):
        P = -(-L // S) + 2
        want_k = flat_k[b].copy()
        want_v = flat_v[b].copy()
        want_k[:, L - 1] = k_new[b]
        want_v[:, L - 1] = v_new[b]
        assert np.array_equal(_flat_of(k_pool, pt[b], P), want_k), b
        assert np.array_equal(_flat_of(v_pool, pt[b], P), want_v), b
        _, phys, n_valid = touched[b]
        assert phys == pt[b][(L - 1) // S]
        assert n_valid == L - S * ((L - 1) // S)       # tokens of that page up to L−1
        changed_pages.add(phys)
    # nothing outside the touched pages moved
    untouched = np.setdiff1d(np.arange(k_pool.shape[0]), sorted(changed_pages))
    assert np.array_equal(k_pool[untouched], before_k[untouched])
    assert np.array_equal(v_pool[untouched], before_v[untouched])


def test_build_page_meta_matches_flat_slices_on_a_permuted_pool():
    """[EntmaxKV] §2.A: metadata of every (physical page, KV head) of a
    scattered pool equals page_metadata of that page's tokens sliced straight
    out of the flat sequence (logical page p = tokens p·S .. p·S + n_p − 1),
    including a partial last page; pages no sequence uses get no entry."""
    rng = np.random.default_rng(73)
    S, Hkv, d = 8, 2, 6
    lens = [21, 8, 30]
    k_pool, _, pt, flat_k, _ = _paged_from_flat(rng, lens, S, Hkv, d, spare=1)
    meta = O.build_page_meta(k_pool, pt, lens, S, "bf16")
    used = set()
    for b, L in enumerate(lens):
        P = -(-L // S)
        for p in range(P):
            n = min(S, L - p * S)
            phys = int(pt[b, p])
            used.add(phys)
            for h in range(Hkv):
                ref = O.page_metadata(flat_k[b][h, p * S:p * S + S][None], [n], "bf16")
                for f in ("kmax", "kmin", "mean", "var"):
                    assert np.array_equal(meta[phys][f][h], ref[f][0]), (b, p, h, f)
    assert set(meta) == used


def test_softmax_lse_consistent_with_weights_and_equal_score_closed_form():
    """The softmax log-sum-exp: n equal scores give z + ln n exactly in closed
    form, and every weight (pinned against scipy above) equals e^(z_i − lse)."""
    rng = np.random.default_rng(79)
    d = 8
    q = rng.normal(size=(2, d))
    K = np.tile(rng.normal(size=(1, d)), (37, 1))
    r = O.softmax_attention(q, K, np.ones((37, 1)), 0.5)
    z = 0.5 * (q @ K[0])
    assert np.allclose(r["lse"], z + math.log(37), rtol=0, atol=1e-13)
    K2 = rng.normal(size=(50, d)) * 3.0
    r2 = O.softmax_attention(q, K2, np.ones((50, 1)), 0.5)
    assert np.allclose(np.exp(0.5 * (q @ K2.T) - r2["lse"][:, None]), r2["p"], rtol=1e-12, atol=1e-300)


def test_softmax_dropped_mass_identity_and_limits():
    """[EntmaxKV] §3 "Borne d'Erreur": the dropped softmax mass δ of a kept set
    equals 1 − e^(lse_kept − lse_all) (the kept tokens' share of Σ e^z), is 0
    when everything is kept and 1 − (kept/T) for equal scores."""
    rng = np.random.default_rng(83)
    q = rng.normal(size=(3, 10))
    K = rng.normal(size=(60, 10))
    kept = rng.random(60) < 0.3
    delta = O.softmax_dropped_mass(q, K, kept, 0.4)
    lse_all = O.softmax_attention(q, K, np.zeros((60, 1)), 0.4)["lse"]
    lse_kept = O.softmax_attention(q, K[kept], np.zeros((int(kept.sum()), 1)), 0.4)["lse"]
    assert np.allclose(delta, 1.0 - np.exp(lse_kept - lse_all), rtol=1e-12, atol=1e-14)
    assert np.allclose(O.softmax_dropped_mass(q, K, np.ones(60, bool), 0.4), 0.0)
    Keq = np.tile(K[:1], (60, 1))
    assert np.allclose(O.softmax_dropped_mass(q, Keq, kept, 0.4), 1.0 - kept.sum() / 60.0, atol=1e-14)
