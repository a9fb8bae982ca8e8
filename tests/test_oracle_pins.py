"""Pins of the fp64 CPU oracle against facts that do not come from the oracle.

Each test checks one oracle function against something independent of its
code: a textbook closed form, an exact rational computation, numerical
quadrature, a constrained optimiser, brute force over supports, or an
invariant the EntmaxKV summary states (gist.science paper 2605.21649:
section 2 exact zeros / support recovery, section 2.A upper bound,
section 3 error bound 2*B*delta).
"""
import json
import math
import os
from fractions import Fraction

import numpy as np
import pytest
from scipy import integrate, optimize

from tests.helpers import bf16_bits_to_f64, f32_to_bf16_bits

GOLD = os.path.join(os.path.dirname(__file__), "golden", "closed_forms.json")


def _gold(case_id):
    for c in json.load(open(GOLD))["cases"]:
        if c["id"] == case_id:
            return c
    raise KeyError(case_id)


# ---------------------------------------------------------------- entmax tau

def _p_from_tau(z, tau, alpha):
    r = 1.0 / (alpha - 1.0)
    return np.where(z > tau, np.maximum(z - tau, 0.0) ** r, 0.0)


def _brute_tau(z, alpha):
    """Enumerate the support size k (the support is always a top-k set) and
    solve sum_{top k} (z - tau)^r = 1 with a bracketing root finder; return
    the one k whose root is consistent with the ordering."""
    r = 1.0 / (alpha - 1.0)
    s = np.sort(z)[::-1]
    found = []
    for k in range(1, len(s) + 1):
        top = s[:k]
        f = lambda t: np.sum((top - t) ** r) - 1.0
        lo, hi = top[-1] - 1.0 - 1e-9, top[-1]
        if f(hi) > 0 or f(lo) < 0:
            continue
        t = optimize.brentq(f, lo, hi, xtol=1e-15, rtol=1e-15)
        nxt = s[k] if k < len(s) else -np.inf
        if t < top[-1] and t >= nxt - 1e-12:
            found.append(t)
    assert len(found) >= 1
    return found[0]


@pytest.mark.parametrize("case_id", ["sparsemax_3", "entmax15_3", "entmax_single"])
def test_entmax_golden_closed_forms(orc, case_id):
    c = _gold(case_id)
    z = np.array(c["z"], np.float64)
    tau = orc.entmax_tau(z, c["alpha"])
    assert tau == pytest.approx(c["tau"], abs=1e-14)
    p = _p_from_tau(z, tau, c["alpha"])
    np.testing.assert_allclose(p, c["p"], atol=1e-13)


@pytest.mark.parametrize("seed", range(20))
def test_general_solver_matches_sparsemax_closed_form(orc, seed):
    rng = np.random.default_rng(seed)
    z = rng.normal(size=rng.integers(1, 200)) * rng.uniform(0.1, 5)
    # closed form written out here: sort, cumulative sums, k*
    s = np.sort(z)[::-1]
    cs = np.cumsum(s)
    ks = np.arange(1, len(s) + 1)
    kstar = ks[1 + ks * s > cs].max()
    tau_cf = (cs[kstar - 1] - 1.0) / kstar
    assert orc.entmax_tau(z, 2.0) == pytest.approx(tau_cf, abs=1e-12)
    assert orc.sparsemax_tau(z) == pytest.approx(tau_cf, abs=1e-12)


@pytest.mark.parametrize("seed", range(20))
def test_general_solver_matches_sort_based_entmax15(orc, seed):
    rng = np.random.default_rng(100 + seed)
    z = rng.normal(size=rng.integers(1, 300)) * rng.uniform(0.1, 5)
    t_gen = orc.entmax_tau(z, 1.5)
    t_sort = orc.entmax15_tau(z)
    assert t_gen == pytest.approx(t_sort, abs=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0, 1.1, 3.0])
@pytest.mark.parametrize("seed", range(6))
def test_entmax_tau_brute_force_support(orc, alpha, seed):
    rng = np.random.default_rng(200 + seed)
    z = rng.normal(size=rng.integers(1, 9)) * rng.uniform(0.2, 3)
    t = orc.entmax_tau(z, alpha)
    assert t == pytest.approx(_brute_tau(z, alpha), abs=1e-11)
    p = _p_from_tau(z, t, alpha)
    assert p.min() >= 0.0
    assert p.sum() == pytest.approx(1.0, abs=1e-12)
    # exact zeros exactly off the support
    assert np.all((p > 0) == (z > t))


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
@pytest.mark.parametrize("seed", range(4))
def test_entmax_is_the_tsallis_regularised_argmax(orc, alpha, seed):
    """alpha-entmax(s) = argmax_{p in simplex} p.s + sum_j (p_j - p_j^alpha)/(alpha(alpha-1));
    the optimiser knows nothing of thresholds, so this pins the (alpha-1)
    scaling of z and the 1/(alpha-1) exponent."""
    rng = np.random.default_rng(300 + seed)
    n = 6
    s = rng.normal(size=n) * 1.5
    z = (alpha - 1.0) * s
    t = orc.entmax_tau(z, alpha)
    p_orc = _p_from_tau(z, t, alpha)

    def negobj(p):
        p = np.maximum(p, 0.0)
        return -(p @ s + np.sum(p - p ** alpha) / (alpha * (alpha - 1.0)))

    res = optimize.minimize(negobj, np.full(n, 1.0 / n), method="SLSQP",
                            bounds=[(0.0, 1.0)] * n,
                            constraints=[{"type": "eq", "fun": lambda p: p.sum() - 1.0}],
                            options={"ftol": 1e-14, "maxiter": 500})
    np.testing.assert_allclose(p_orc, np.maximum(res.x, 0), atol=2e-5)


# ------------------------------------------------ Gaussian partial moments

@pytest.mark.parametrize("r", [0, 1, 2, 3, 4, 8])
@pytest.mark.parametrize("c", [-6.0, -2.5, -0.3, 0.0, 0.7, 2.0, 4.5, 7.0])
def test_gauss_J_matches_quadrature(orc, r, c):
    phi = lambda z: math.exp(-0.5 * z * z) / math.sqrt(2 * math.pi)
    ref, _ = integrate.quad(lambda z: (z - c) ** r * phi(z), c, np.inf,
                            epsabs=1e-300, epsrel=1e-13, limit=200)
    got = orc.gauss_J(r, c)
    assert got == pytest.approx(ref, rel=1e-9, abs=1e-14 * max(1.0, abs(c)) ** r * phi(c) + 1e-300)


def test_gauss_J_golden_at_zero(orc):
    for r, v in _gold("gauss_J_at_zero")["values"].items():
        assert orc.gauss_J(int(r), 0.0) == pytest.approx(v, rel=1e-14)


def test_gauss_J_monte_carlo(orc):
    rng = np.random.default_rng(7)
    zs = rng.standard_normal(4_000_000)
    for r, c in [(1, 0.5), (2, -1.0), (4, 0.25)]:
        mc = np.mean(np.maximum(zs - c, 0.0) ** r)
        se = np.std(np.maximum(zs - c, 0.0) ** r) / math.sqrt(len(zs))
        assert abs(orc.gauss_J(r, c) - mc) < 5 * se


# --------------------------------------------------------------- tau_hat

def test_tau_hat_golden_point_masses(orc):
    c = _gold("tau_hat_point_masses")
    a1 = c["alpha"] - 1.0
    mu = np.array(c["mu_z"]) / a1
    t = orc.tau_hat(mu, np.zeros_like(mu), np.array(c["n_tok"]), c["alpha"])
    assert t == pytest.approx(c["tau_hat"], abs=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
@pytest.mark.parametrize("seed", range(4))
def test_tau_hat_zero_variance_is_entmax_of_page_means(orc, alpha, seed):
    """sigma -> 0 turns every page into n_p identical scores m_p, so tau_hat
    must equal the exact entmax threshold of that multiset."""
    rng = np.random.default_rng(400 + seed)
    npg = rng.integers(1, 40)
    mu = rng.normal(size=npg).astype(np.float32)
    n_tok = rng.integers(1, 65, size=npg)
    t = orc.tau_hat(mu, np.zeros(npg, np.float32), n_tok, alpha)
    z = np.repeat((alpha - 1.0) * mu.astype(np.float64), n_tok)
    assert t == pytest.approx(_brute_tau(z, alpha) if len(z) < 9 else orc.entmax_tau(z, alpha),
                              abs=1e-10)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
@pytest.mark.parametrize("seed", range(3))
def test_tau_hat_solves_normalisation_with_quadrature(orc, alpha, seed):
    """Re-evaluate F(tau_hat) with J computed by quadrature: it must be 1."""
    rng = np.random.default_rng(500 + seed)
    npg = 12
    mu = rng.normal(size=npg).astype(np.float32)
    sigma = rng.uniform(0.05, 1.5, size=npg).astype(np.float32)
    n_tok = rng.integers(1, 65, size=npg)
    t = orc.tau_hat(mu, sigma, n_tok, alpha)
    a1 = alpha - 1.0
    r = round(1.0 / a1)

    def F(tau):
        tot = 0.0
        for m, s, n in zip(mu, sigma, n_tok):
            m, s = a1 * float(m), a1 * float(s)
            f = lambda x: (x - tau) ** r * math.exp(-0.5 * ((x - m) / s) ** 2) / (s * math.sqrt(2 * math.pi))
            v, _ = integrate.quad(f, tau, m + 40 * s + abs(tau), epsabs=1e-15, epsrel=1e-12, limit=200)
            tot += n * v
        return tot

    assert F(t) == pytest.approx(1.0, rel=1e-7)
    # F decreases, so a slightly smaller tau gives more than one
    assert F(t - 1e-3) > 1.0 > F(t + 1e-3)


def test_tau_hat_rejects_non_integer_exponent(orc):
    assert math.isnan(orc.tau_hat(np.zeros(3, np.float32), np.ones(3, np.float32),
                                  np.ones(3, np.int32), 1.3))


# ------------------------------------------------------------- metadata

def _random_pages(rng, n_blk, Hkv, P, d, scale=1.0):
    x = (rng.normal(size=(n_blk, Hkv, P, d)) * scale).astype(np.float32)
    return f32_to_bf16_bits(x).reshape(n_blk, Hkv, P, d)


@pytest.mark.parametrize("seed", range(3))
def test_build_meta_exact_rationals(orc, seed):
    rng = np.random.default_rng(600 + seed)
    B, Hkv, d, P, npg = 2, 2, 8, 16, 3
    nb = B * npg
    K = _random_pages(rng, nb, Hkv, P, d, scale=rng.uniform(0.01, 10))
    pt = rng.permutation(nb).astype(np.int32).reshape(B, npg)
    seq = np.array([npg * P, npg * P - 5], np.int32)   # second sequence ragged
    kmin, kmax, mean, var = orc.build_meta(K, pt, seq, Hkv, d, P, nb)
    for b in range(B):
        for p in range(npg):
            n = min(P, seq[b] - p * P)
            blk = pt[b, p]
            for kvh in range(Hkv):
                rec = blk * Hkv + kvh
                x = bf16_bits_to_f64(K[blk, kvh, :n])          # [n, d]
                np.testing.assert_array_equal(bf16_bits_to_f64(kmin[rec]), x.min(0))
                np.testing.assert_array_equal(bf16_bits_to_f64(kmax[rec]), x.max(0))
                for j in range(d):
                    col = [Fraction(float(v)) for v in x[:, j]]
                    m = sum(col) / n
                    v = sum(c * c for c in col) / n - m * m
                    assert mean[rec, j] == np.float32(float(m))
                    # var: within the rounding of the fp64 steps plus one fp32 rounding
                    s2n = float(sum(c * c for c in col) / n)
                    bound = 4 * 2.0 ** -52 * s2n + np.spacing(np.float32(float(v)))
                    assert abs(float(var[rec, j]) - float(v)) <= bound


def test_build_meta_single_token_page(orc):
    rng = np.random.default_rng(11)
    K = _random_pages(rng, 1, 1, 16, 64)
    kmin, kmax, mean, var = orc.build_meta(K, np.zeros((1, 1), np.int32),
                                           np.array([1], np.int32), 1, 64, 16, 1)
    np.testing.assert_array_equal(kmin[0], K[0, 0, 0])
    np.testing.assert_array_equal(kmax[0], K[0, 0, 0])
    np.testing.assert_array_equal(mean[0], bf16_bits_to_f64(K[0, 0, 0]).astype(np.float32))
    assert np.all(var[0] == 0.0)


# ---------------------------------------------------------- page scores

def _scores_setup(seed, B=2, Hq=4, Hkv=2, d=16, P=8, npg=5, ragged=True):
    rng = np.random.default_rng(seed)
    nb = B * npg
    K = _random_pages(rng, nb, Hkv, P, d)
    q = f32_to_bf16_bits(rng.normal(size=(B, Hq, d)).astype(np.float32))
    pt = rng.permutation(nb).astype(np.int32).reshape(B, npg)
    seq = np.array([npg * P - (3 if ragged and b % 2 else 0) for b in range(B)], np.int32)
    return K, q, pt, seq, dict(B=B, Hq=Hq, Hkv=Hkv, d=d, P=P, npg=npg, nb=nb)


@pytest.mark.parametrize("seed", range(4))
def test_bbox_is_an_upper_bound_and_exact_sum(orc, seed):
    K, q, pt, seq, s = _scores_setup(700 + seed)
    meta = orc.build_meta(K, pt, seq, s["Hkv"], s["d"], s["P"], s["nb"])
    bbox, mu, sig = orc.score_pages(q, meta, pt, seq, s["Hkv"], s["P"])
    G = s["Hq"] // s["Hkv"]
    inv = 1.0 / math.sqrt(s["d"])
    for b in range(s["B"]):
        for h in range(s["Hq"]):
            qv = bf16_bits_to_f64(q[b, h])
            for p in range(s["npg"]):
                n = min(s["P"], seq[b] - p * s["P"])
                blk = pt[b, p]
                keys = bf16_bits_to_f64(K[blk, h // G, :n])
                smax = (keys @ qv).max() * inv
                assert float(bbox[b, h, p]) >= smax * (1 - 1e-6) - 1e-30
                # exact rational value of the bound, rounded once
                rec = blk * s["Hkv"] + h // G
                lo = bf16_bits_to_f64(meta[0][rec])
                hi = bf16_bits_to_f64(meta[1][rec])
                S = sum(max(Fraction(float(a)) * Fraction(float(l)), Fraction(float(a)) * Fraction(float(u)))
                        for a, l, u in zip(qv, lo, hi))
                assert bbox[b, h, p] == np.float32(float(S) * inv)


def test_bbox_is_tight_on_single_token_pages(orc):
    K, q, pt, seq, s = _scores_setup(71, P=1, npg=6, ragged=False)
    meta = orc.build_meta(K, pt, seq, s["Hkv"], s["d"], 1, s["nb"])
    bbox, _, _ = orc.score_pages(q, meta, pt, seq, s["Hkv"], 1)
    G = s["Hq"] // s["Hkv"]
    for b in range(s["B"]):
        for h in range(s["Hq"]):
            for p in range(s["npg"]):
                k = bf16_bits_to_f64(K[pt[b, p], h // G, 0])
                sc = k @ bf16_bits_to_f64(q[b, h]) / math.sqrt(s["d"])
                assert float(bbox[b, h, p]) == pytest.approx(sc, rel=1e-6, abs=1e-6)


@pytest.mark.parametrize("seed", range(3))
def test_mu_is_the_mean_token_score(orc, seed):
    K, q, pt, seq, s = _scores_setup(800 + seed)
    meta = orc.build_meta(K, pt, seq, s["Hkv"], s["d"], s["P"], s["nb"])
    _, mu, _ = orc.score_pages(q, meta, pt, seq, s["Hkv"], s["P"])
    G = s["Hq"] // s["Hkv"]
    for b in range(s["B"]):
        for h in range(s["Hq"]):
            qv = bf16_bits_to_f64(q[b, h])
            for p in range(s["npg"]):
                n = min(s["P"], seq[b] - p * s["P"])
                keys = bf16_bits_to_f64(K[pt[b, p], h // G, :n])
                emp = (keys @ qv).mean() / math.sqrt(s["d"])
                scale = np.abs(qv).sum() * np.abs(keys).max() / math.sqrt(s["d"])
                assert float(mu[b, h, p]) == pytest.approx(emp, abs=2e-7 * scale)


def test_sigma_is_exact_when_one_coordinate_varies(orc):
    """With keys that differ in one coordinate j only, the page's token
    scores have variance q_j^2 var_j / d exactly: the diagonal model is exact."""
    rng = np.random.default_rng(9)
    d, P = 16, 32
    base = rng.normal(size=d).astype(np.float32)
    x = np.tile(base, (P, 1))
    x[:, 5] = rng.normal(size=P).astype(np.float32) * 2.0
    K = f32_to_bf16_bits(x).reshape(1, 1, P, d)
    q = f32_to_bf16_bits(rng.normal(size=(1, 1, d)).astype(np.float32))
    pt = np.zeros((1, 1), np.int32)
    seq = np.array([P], np.int32)
    meta = orc.build_meta(K, pt, seq, 1, d, P, 1)
    _, mu, sig = orc.score_pages(q, meta, pt, seq, 1, P)
    sc = bf16_bits_to_f64(K[0, 0]) @ bf16_bits_to_f64(q[0, 0]) / math.sqrt(d)
    assert float(sig[0, 0, 0]) == pytest.approx(sc.std(), rel=1e-6)
    assert float(mu[0, 0, 0]) == pytest.approx(sc.mean(), rel=1e-6, abs=1e-7)


# ------------------------------------------------------------- selection

@pytest.mark.parametrize("seed", range(10))
def test_topk_matches_lexicographic_sort_with_ties(orc, seed):
    rng = np.random.default_rng(900 + seed)
    n = int(rng.integers(1, 400))
    sc = np.round(rng.normal(size=n), 1).astype(np.float32)     # many ties
    k = int(rng.integers(1, n + 5))
    got = orc.select_topk(sc, k)
    order = np.lexsort((np.arange(n), -sc.astype(np.float64)))
    want = np.sort(order[:min(k, n)])
    np.testing.assert_array_equal(got, want)


def test_gauss_select_keeps_support_pages_when_threshold_is_low(orc):
    """Section 2.B/2.C: a page holding a support token has (alpha-1)*bound >= z > tau,
    so any threshold at or below the exact tau keeps every support page."""
    rng = np.random.default_rng(12)
    B, Hq, Hkv, d, P, npg = 1, 2, 1, 16, 8, 20
    nb = npg
    K = _random_pages(rng, nb, Hkv, P, d)
    V = _random_pages(rng, nb, Hkv, P, d)
    q = f32_to_bf16_bits(rng.normal(size=(B, Hq, d)).astype(np.float32) * 2)
    pt = np.arange(nb, dtype=np.int32).reshape(1, npg)
    seq = np.array([npg * P], np.int32)
    alpha = 1.5
    meta = orc.build_meta(K, pt, seq, Hkv, d, P, nb)
    bbox, _, _ = orc.score_pages(q, meta, pt, seq, Hkv, P)
    o, tau, pw, _ = orc.decode(q, K, V, pt, seq, Hkv, P, alpha, want_p=True)
    for h in range(Hq):
        sel = orc.select_gauss(bbox[0, h], alpha, tau[0, h], 0.0)
        supp_pages = set(np.nonzero(pw[0, h])[0] // P)
        assert supp_pages <= set(sel.tolist())


def test_zmax_of_closed_forms(orc):
    """z(n)^2 = 2 ln n: z(64)^2 = 12 ln 2, z(e^2) would be 2; one token: 0."""
    assert orc.zmax_of(64) ** 2 == pytest.approx(12 * math.log(2), rel=1e-15)
    assert orc.zmax_of(2) ** 2 == pytest.approx(2 * math.log(2), rel=1e-15)
    assert orc.zmax_of(1) == 0.0


def test_gauss_est_hand_example(orc):
    """Three pages worked by hand: alpha 1.5, tau_hat 1, Delta 0.5 (cut 0.5 on z).
    Estimate: p0 min(2, 1 + 0.5 sqrt(2 ln 64)) = 2 -> z 1.0, kept; p1 min(1, 0.5 +
    0.1 sqrt(2 ln 64)) = 0.788 -> 0.394, dropped; p2 min(3, 0.2 + 0.3 sqrt(2 ln 10))
    = 0.844 -> 0.422, dropped.  Bound alone: z = 1.0, 0.5 (not above the cut), 1.5."""
    bbox = np.array([2.0, 1.0, 3.0], np.float32)
    mu = np.array([1.0, 0.5, 0.2], np.float32)
    sig = np.array([0.5, 0.1, 0.3], np.float32)
    n = np.array([64, 64, 10], np.int32)
    np.testing.assert_array_equal(orc.select_gauss_est(bbox, mu, sig, n, 1.5, 1.0, 0.5), [0])
    np.testing.assert_array_equal(orc.select_gauss(bbox, 1.5, 1.0, 0.5), [0, 2])


@pytest.mark.parametrize("seed", range(6))
def test_gauss_est_keeps_a_subset_of_the_bound_rule(orc, seed):
    """min(u, mu + z sigma) <= u, so the estimate keeps a subset of what the
    bound keeps, and the same pages where mu + z sigma >= u."""
    rng = np.random.default_rng(1300 + seed)
    n = 500
    bbox = rng.normal(2.0, 1.0, n).astype(np.float32)
    mu = (bbox - np.abs(rng.normal(1.0, 0.5, n))).astype(np.float32)
    sig = np.abs(rng.normal(0.3, 0.3, n)).astype(np.float32)
    nt = rng.integers(1, 65, n).astype(np.int32)
    tau_hat, delta, alpha = float(rng.normal(1.0, 0.3)), 0.25, 1.5
    est = set(orc.select_gauss_est(bbox, mu, sig, nt, alpha, tau_hat, delta).tolist())
    bnd = set(orc.select_gauss(bbox, alpha, tau_hat, delta).tolist())
    assert est <= bnd
    capped = {p for p in range(n) if mu[p] + orc.zmax_of(int(nt[p])) * float(sig[p]) >= float(bbox[p])}
    assert {p for p in bnd if p in capped} <= est


def test_gauss_est_equals_bound_rule_on_constant_pages(orc):
    """Pages whose tokens are all the same key: sigma = 0 and mu equals the bound
    (both are q.k/sqrt(d) summed in the same order), so both rules agree."""
    rng = np.random.default_rng(77)
    Hq, Hkv, d, P, npg = 2, 1, 16, 8, 30
    base = _random_pages(rng, npg, Hkv, 1, d)
    K = np.repeat(base, P, axis=2)
    q = f32_to_bf16_bits(rng.normal(size=(1, Hq, d)).astype(np.float32))
    pt = np.arange(npg, dtype=np.int32).reshape(1, npg)
    seq = np.array([npg * P], np.int32)
    meta = orc.build_meta(K, pt, seq, Hkv, d, P, npg)
    bbox, mu, sig = orc.score_pages(q, meta, pt, seq, Hkv, P)
    assert np.all(sig == 0.0)
    np.testing.assert_array_equal(mu, bbox)
    nt = np.full(npg, P, np.int32)
    for h in range(Hq):
        t = float(np.median(bbox[0, h])) * 0.5
        np.testing.assert_array_equal(orc.select_gauss_est(bbox[0, h], mu[0, h], sig[0, h], nt, 1.5, t, 0.1),
                                      orc.select_gauss(bbox[0, h], 1.5, t, 0.1))


# ----------------------------------------------------------------- decode

def _decode_setup(seed, alpha, Hq=2, Hkv=1, d=16, P=8, npg=12):
    rng = np.random.default_rng(seed)
    nb = npg
    K = _random_pages(rng, nb, Hkv, P, d)
    V = _random_pages(rng, nb, Hkv, P, d)
    q = f32_to_bf16_bits(rng.normal(size=(1, Hq, d)).astype(np.float32) * 3)
    pt = rng.permutation(nb).astype(np.int32).reshape(1, npg)
    seq = np.array([npg * P - 3], np.int32)
    return K, V, q, pt, seq


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_decode_matches_brute_force(orc, alpha):
    K, V, q, pt, seq = _decode_setup(21, alpha)
    o, tau, pw, _ = orc.decode(q, K, V, pt, seq, 1, 8, alpha, want_p=True)
    for h in range(2):
        keys, vals, pos = [], [], []
        for p in range(pt.shape[1]):
            n = min(8, seq[0] - p * 8)
            keys.append(bf16_bits_to_f64(K[pt[0, p], 0, :n]))
            vals.append(bf16_bits_to_f64(V[pt[0, p], 0, :n]))
        keys, vals = np.concatenate(keys), np.concatenate(vals)
        s = keys @ bf16_bits_to_f64(q[0, h]) / 4.0
        z = (alpha - 1) * s
        t = orc.entmax15_tau(z) if alpha == 1.5 else (orc.sparsemax_tau(z) if alpha == 2.0 else _brute_tau_big(z, alpha))
        p = _p_from_tau(z, t, alpha)
        np.testing.assert_allclose(o[0, h], p @ vals, atol=1e-11)
        assert tau[0, h] == pytest.approx(t, abs=1e-11)


def _brute_tau_big(z, alpha):
    # bracketing root of the full sum (continuous, decreasing)
    r = 1.0 / (alpha - 1.0)
    f = lambda t: np.sum(np.maximum(z - t, 0.0) ** r) - 1.0
    return optimize.brentq(f, z.max() - 1.0 - 1e-12, z.max(), xtol=1e-15, rtol=1e-15)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
def test_sparse_equals_full_when_selection_holds_support(orc, alpha):
    """Section 2 / section 3: if the kept set contains the support, the sparse
    output is identical to the full-cache output."""
    K, V, q, pt, seq = _decode_setup(31, alpha)
    o_full, tau_full, pw, _ = orc.decode(q, K, V, pt, seq, 1, 8, alpha, want_p=True)
    npg = pt.shape[1]
    sel = np.full((1, 2, npg), -1, np.int32)
    cnt = np.zeros((1, 2), np.int32)
    rng = np.random.default_rng(5)
    for h in range(2):
        keep = set((np.nonzero(pw[0, h])[0] // 8).tolist())
        keep |= set(rng.choice(npg, 3, replace=False).tolist())
        ks = sorted(keep)
        sel[0, h, :len(ks)] = ks
        cnt[0, h] = len(ks)
    o_sp, tau_sp, _, _ = orc.decode(q, K, V, pt, seq, 1, 8, alpha, sel=sel, cnt=cnt)
    np.testing.assert_allclose(o_sp, o_full, atol=1e-12)
    np.testing.assert_allclose(tau_sp, tau_full, atol=1e-12)


@pytest.mark.parametrize("alpha", [1.25, 1.5, 2.0])
@pytest.mark.parametrize("seed", range(4))
def test_truncation_error_within_2_B_delta(orc, alpha, seed):
    """Section 3: |o - o~| <= 2 B delta, delta = full-cache mass of the dropped
    tokens, B = max value norm."""
    K, V, q, pt, seq = _decode_setup(41 + seed, alpha)
    o_full, _, pw, _ = orc.decode(q, K, V, pt, seq, 1, 8, alpha, want_p=True)
    npg = pt.shape[1]
    rng = np.random.default_rng(seed)
    sel = np.full((1, 2, npg), -1, np.int32)
    cnt = np.zeros((1, 2), np.int32)
    for h in range(2):
        ks = np.sort(rng.choice(npg, npg // 2, replace=False))
        sel[0, h, :len(ks)] = ks
        cnt[0, h] = len(ks)
    o_sp, _, _, _ = orc.decode(q, K, V, pt, seq, 1, 8, alpha, sel=sel, cnt=cnt)
    Bv = max(np.linalg.norm(bf16_bits_to_f64(V[pt[0, p], 0, :min(8, seq[0] - p * 8)]), axis=1).max()
             for p in range(npg))
    for h in range(2):
        kept = np.zeros(npg * 8, bool)
        for p in sel[0, h, :cnt[0, h]]:
            kept[p * 8:(p + 1) * 8] = True
        delta = pw[0, h][~kept].sum()
        err = np.linalg.norm(o_sp[0, h] - o_full[0, h])
        assert err <= 2 * Bv * delta + 1e-12


def test_softmax_closed_forms(orc):
    d, P = 8, 4
    rng = np.random.default_rng(3)
    # two tokens: p1 = 1/(1 + exp(s2 - s1))
    K = _random_pages(rng, 1, 1, P, d)
    V = _random_pages(rng, 1, 1, P, d)
    q = f32_to_bf16_bits(rng.normal(size=(1, 1, d)).astype(np.float32))
    pt = np.zeros((1, 1), np.int32)
    seq = np.array([2], np.int32)
    o, m, pw, _ = orc.decode(q, K, V, pt, seq, 1, P, 1.0, want_p=True)
    k = bf16_bits_to_f64(K[0, 0, :2])
    s = k @ bf16_bits_to_f64(q[0, 0]) / math.sqrt(d)
    p1 = 1.0 / (1.0 + math.exp(s[1] - s[0]))
    assert pw[0, 0, 0] == pytest.approx(p1, rel=1e-13)
    v = bf16_bits_to_f64(V[0, 0, :2])
    np.testing.assert_allclose(o[0, 0], p1 * v[0] + (1 - p1) * v[1], atol=1e-13)
    # identical keys: uniform weights, output = mean of the values
    Ku = np.tile(K[:, :, :1], (1, 1, P, 1))
    o, _, pw, _ = orc.decode(q, Ku, V, pt, np.array([P], np.int32), 1, P, 1.0, want_p=True)
    np.testing.assert_allclose(pw[0, 0, :P], 0.25, rtol=1e-14)
    np.testing.assert_allclose(o[0, 0], bf16_bits_to_f64(V[0, 0]).mean(0), atol=1e-13)


def test_needle_score_closed_form(orc):
    """A key planted as c*sqrt(d)*q/|q| scores c*|q| (up to bf16 rounding)."""
    d = 64
    rng = np.random.default_rng(4)
    qf = rng.normal(size=d).astype(np.float32)
    qb = f32_to_bf16_bits(qf)
    qd = bf16_bits_to_f64(qb)
    kn = 4.0 * math.sqrt(d) * qd / np.linalg.norm(qd)
    K = np.zeros((1, 1, 16, d), np.uint16)
    K[0, 0, 0] = f32_to_bf16_bits(kn.astype(np.float32))
    V = np.zeros_like(K)
    _, _, _, z = orc.decode(qb.reshape(1, 1, d), K, V, np.zeros((1, 1), np.int32),
                            np.array([1], np.int32), 1, 16, 2.0, want_z=True)
    assert z[0, 0, 0] == pytest.approx(4.0 * np.linalg.norm(qd), rel=1e-2)
