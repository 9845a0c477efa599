"""Pins of the fp64 oracle against facts that do not come from the oracle itself.

Operator ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
technical summary section 2.1): p_i = F((r_i - b)/t), F the Laplace CDF, with
b fixed by sum_i p_i = k, and an analytic VJP.  Each test below pins one part
of the oracle to a closed form, a library routine, brute force, an invariant or
a limit that the pages state (the zero-temperature limit of section 2.3).
"""
import math

import hypothesis.strategies as hyp
import numpy as np
import pytest
import scipy.stats as st
from hypothesis import given, settings

import workloads as W

RNG = np.random.default_rng(12345)


def icdf(q):
    return math.log(2 * q) if q < 0.5 else -math.log(2 * (1 - q))


# ---------------------------------------------------------------- closed forms
@pytest.mark.parametrize("k", [0.1, 0.5, 0.9])
def test_single_score_closed_form(orc, k):
    # n = 1: p = k, so (r - b)/t = F^{-1}(k)
    r, t = np.float32(0.75), 0.2
    b = orc.solve([r], k, t)
    assert abs(b - (float(r) - t * icdf(k))) <= 1e-13 * max(1.0, abs(b))
    assert abs(orc.p([r], b, t)[0] - k) <= 1e-13


@pytest.mark.parametrize("n,k", [(7, 3.0), (100, 1.0), (100, 99.5), (4096, 64.0)])
def test_all_equal_scores_closed_form(orc, n, k):
    r = np.full(n, 1.25, np.float32)
    t = 0.05
    b = orc.solve(r, k, t)
    assert abs(b - (1.25 - t * icdf(k / n))) <= 1e-13 * 1.25
    np.testing.assert_allclose(orc.p(r, b, t), k / n, rtol=1e-12)


@pytest.mark.parametrize("delta,t", [(0.5, 0.1), (0.03125, 0.01), (2.0, 0.7)])
def test_two_scores_closed_form(orc, delta, t):
    # r = (a, a - D), k = 1: by symmetry b = a - D/2, p = (1 - e^{-D/2t}/2, e^{-D/2t}/2)
    a = np.float32(0.5)
    r = np.array([a, a - np.float32(delta)], np.float32)
    b = orc.solve(r, 1.0, t)
    D = float(r[0]) - float(r[1])
    assert abs(b - (float(r[0]) - D / 2)) <= 1e-13
    e = 0.5 * math.exp(-D / (2 * t))
    np.testing.assert_allclose(orc.p(r, b, t), [1 - e, e], rtol=1e-13)


# ----------------------------------------------- library routine: Laplace CDF
def test_G_and_p_match_scipy_laplace(orc):
    r = RNG.standard_normal(3000).astype(np.float32)
    t = 0.3
    for b in (-1.0, 0.2, 2.5):
        x = (r.astype(np.float64) - b) / t
        ref = math.fsum(st.laplace.cdf(x))
        g, sf = orc.G(r, b, t)
        assert abs(g - ref) <= 1e-11 * len(r)
        assert abs(sf - math.fsum(st.laplace.pdf(x))) <= 1e-11 * len(r)
        np.testing.assert_allclose(orc.p(r, b, t), st.laplace.cdf(x), rtol=0, atol=1e-15)


# -------------------------------------------------------------- brute force
def brute_force_b(r, k, t):
    """Enumerate the n+1 intervals between sorted scores and solve, in each,
    1/2 S- u^2 + (k - m) u - 1/2 S+ = 0 with u = e^{b/t}, S- = sum_{above} e^{-r/t},
    S+ = sum_{below} e^{r/t}; keep the root that lies inside its interval.  The
    positive root (A >= 0 >= C) is taken in the form that subtracts nothing:
    (-B + sqrt(disc)) / 2A for B < 0, and -2C / (B + sqrt(disc)) for B >= 0 (the
    same number; the first form loses digits to cancellation when 4AC << B^2)."""
    c = sorted((float(v) for v in r), reverse=True)
    n = len(c)
    roots = []
    for m in range(n + 1):
        Sm = sum(math.exp(-v / t) for v in c[:m])
        Sp = sum(math.exp(v / t) for v in c[m:])
        A, B, Cc = 0.5 * Sm, (k - m), -0.5 * Sp
        if A == 0.0:
            u = -Cc / B if B != 0 else None
        else:
            disc = B * B - 4 * A * Cc
            u = (-B + math.sqrt(disc)) / (2 * A) if B < 0 else -2 * Cc / (B + math.sqrt(disc))
        if u is None or u <= 0:
            continue
        b = t * math.log(u)
        hi = c[m - 1] if m >= 1 else math.inf
        lo = c[m] if m < n else -math.inf
        if lo - 1e-9 <= b <= hi + 1e-9:
            roots.append(b)
    return roots


@pytest.mark.parametrize("seed", range(12))
def test_bisection_matches_interval_enumeration(orc, seed):
    rng = np.random.default_rng(seed)
    n = int(rng.integers(1, 13))
    r = (rng.standard_normal(n) * 0.7).astype(np.float32)
    if seed % 3 == 0 and n > 2:
        r[1] = r[0]                                       # a tie
    t = float(rng.uniform(0.05, 0.6))
    k = float(rng.uniform(0.05, n - 0.05)) if n > 1 else 0.4
    roots = brute_force_b(r, k, t)
    assert roots, "brute force found no root"
    b = orc.solve(r, k, t)
    assert min(abs(b - x) for x in roots) <= 1e-10 * t
    assert max(roots) - min(roots) <= 1e-9 * t             # unique root (ties repeat it)


@settings(max_examples=300, derandomize=True, deadline=None)
@given(data=hyp.data())
def test_bisection_matches_interval_enumeration_on_generated_rows(orc, data):
    # generated rows on a coarse grid (many ties, up to all equal), budgets from
    # near 0 to near n, temperatures across an order of magnitude
    n = data.draw(hyp.integers(1, 12))
    r = np.array(data.draw(hyp.lists(hyp.integers(-10, 10), min_size=n, max_size=n)), np.float32) * np.float32(0.1)
    t = data.draw(hyp.floats(0.05, 0.6))
    k = data.draw(hyp.floats(0.01, n - 0.01)) if n > 1 else data.draw(hyp.floats(0.01, 0.99))
    roots = brute_force_b(r, k, t)
    assert roots, "brute force found no root"
    b = orc.solve(r, k, t)
    assert min(abs(b - x) for x in roots) <= 1e-10 * t
    assert max(roots) - min(roots) <= 1e-9 * t


def test_newton_and_bisection_agree(orc):
    r = W.scores("n4096")[0]
    b0 = orc.solve(r, 64.0, 0.05, method=0)
    b1 = orc.solve(r, 64.0, 0.05, method=1)
    assert abs(b0 - b1) <= 1e-13 * max(1.0, abs(b0))


# --------------------------------------------------------------- invariants
def _row(n=2000, seed=1):
    return np.random.default_rng(seed).standard_normal(n).astype(np.float32)


@pytest.mark.parametrize("k,t", [(10.0, 0.05), (1000.0, 0.5), (1999.0, 0.01), (0.3, 2.0)])
def test_budget_and_monotonicity(orc, k, t):
    r = _row()
    b = orc.solve(r, k, t)
    p = orc.p(r, b, t)
    assert abs(p.sum() - k) <= 1e-9 * max(k, 1.0)
    o = np.argsort(r, kind="stable")
    ps, rs = p[o], r[o]
    assert np.all(np.diff(ps) >= 0)
    assert np.all((np.diff(ps) > 0) | (np.diff(rs) == 0) | (ps[1:] == 1.0) | (ps[:-1] == 0.0))


def test_translation_scale_permutation_reflection(orc):
    # scores on a 2^-12 grid in (-4, 4): r + 0.5 and 4 r are exact in fp32
    r = (np.round(_row(600) * 0.5 * 4096) / 4096).astype(np.float32)
    k, t = 37.0, 0.1
    b = orc.solve(r, k, t)
    p = orc.p(r, b, t)
    # translation by an exactly representable shift
    bt = orc.solve(r + np.float32(0.5), k, t)
    assert abs(bt - (b + 0.5)) <= 1e-12
    # scale by a power of two (exact in fp32): (s r, s t) -> s b
    bs = orc.solve(r * np.float32(4.0), k, 4 * t)
    assert abs(bs - 4 * b) <= 1e-12
    # permutation
    perm = np.random.default_rng(3).permutation(r.size)
    bp = orc.solve(r[perm], k, t)
    assert abs(bp - b) <= 1e-13
    np.testing.assert_allclose(orc.p(r[perm], bp, t), p[perm], atol=1e-14)
    # reflection: (-r, n - k) -> (-b, 1 - p)
    br = orc.solve(-r, r.size - k, t)
    assert abs(br + b) <= 1e-12
    np.testing.assert_allclose(orc.p(-r, br, t), 1 - p, atol=1e-12)


@settings(max_examples=100, derandomize=True, deadline=None)
@given(data=hyp.data())
def test_invariances_on_generated_rows(orc, data):
    # generated rows on a 2^-12 grid in (-3, 3) (r + 0.5, 4 r and -r stay exact in
    # fp32), any budget in (0, n), temperatures from 0.02 to 1
    n = data.draw(hyp.integers(2, 200))
    r = (np.array(data.draw(hyp.lists(hyp.integers(-3 * 4096, 3 * 4096), min_size=n, max_size=n)),
                  np.float64) / 4096).astype(np.float32)
    k = data.draw(hyp.floats(0.05, n - 0.05))
    t = data.draw(hyp.floats(0.02, 1.0))
    b = orc.solve(r, k, t)
    assert abs(orc.solve(r + np.float32(0.5), k, t) - (b + 0.5)) <= 1e-12 * max(1.0, abs(b))
    assert abs(orc.solve(r * np.float32(4.0), k, 4 * t) - 4 * b) <= 4e-12 * max(1.0, abs(b))
    assert abs(orc.solve(-r, n - k, t) + b) <= 1e-12 * max(1.0, abs(b))
    assert abs(orc.p(r, b, t).sum() - k) <= 1e-9 * max(k, 1.0)


# ------------------------------------------- zero-temperature (DFTopK) limit
@pytest.mark.parametrize("k", [1, 5, 40])
@pytest.mark.parametrize("ratio", [10.0, 20.0, 30.0])
def test_zero_temperature_limit(orc, k, ratio):
    # technical summary section 2.3: the t -> 0 limit puts the threshold at the
    # midpoint of order statistics k and k+1, i.e. p tends to the hard top-k mask.
    # With gap = c_k - c_{k+1} and no score crossing b, G(mid + d) = k - A e^{d/t} + Z e^{-d/t}
    # with A, Z in [e^{-gap/2t}/2, n e^{-gap/2t}/2], so |b - mid| <= (t/2) ln n and
    # |p - mask| <= (n/2) e^{-gap/2t}.  (gap/2t = ratio keeps G - k resolvable in fp64.)
    rng = np.random.default_rng(k)
    r = rng.permutation(np.arange(100, dtype=np.float32) * np.float32(0.125))
    c = np.sort(r.astype(np.float64))[::-1]
    gap = c[k - 1] - c[k]
    t = gap / (2 * ratio)
    b = orc.solve(r, float(k), t)
    mid = 0.5 * (c[k - 1] + c[k])
    n = r.size
    assert abs(b - mid) <= 0.5 * t * math.log(n) * (1 + 1e-6)
    mask = (r.astype(np.float64) >= c[k - 1]).astype(np.float64)
    assert np.max(np.abs(orc.p(r, b, t) - mask)) <= 0.5 * n * math.exp(-ratio)


# ---------------------------------------------------------------------- VJP
@pytest.mark.parametrize("seed", range(4))
def test_vjp_matches_finite_differences(orc, seed):
    rng = np.random.default_rng(100 + seed)
    n = 12
    # scores in [1, 2) on a 2^-12 grid, step h = 2^-20: r +- h stays exact in fp32
    r = (1.0 + rng.integers(0, 4096, n) / 4096.0).astype(np.float32)
    g = rng.standard_normal(n).astype(np.float32)
    k, t = float(rng.uniform(1, n - 1)), 0.125
    h = 2.0 ** -20

    def L(rr):
        bb = orc.solve(rr, k, t)
        return float(np.dot(g.astype(np.float64), orc.p(rr, bb, t)))

    b = orc.solve(r, k, t)
    grad, gf, sf = orc.vjp(r, g, b, t)
    fd = np.empty(n)
    for j in range(n):
        rp, rm = r.copy(), r.copy()
        rp[j] += np.float32(h)
        rm[j] -= np.float32(h)
        assert float(rp[j]) - float(r[j]) == h
        fd[j] = (L(rp) - L(rm)) / (2 * h)
    assert np.linalg.norm(grad - fd) <= 1e-6 * np.linalg.norm(fd)
    assert abs(grad.sum()) <= 1e-12 * np.abs(grad).sum()      # translation invariance
    gc, _, _ = orc.vjp(r, np.full(n, 0.7, np.float32), b, t)   # fixed budget
    assert np.max(np.abs(gc)) <= 1e-13


def test_vjp_survives_underflowing_density(orc):
    # two scores 2000 t apart: every f_i underflows in fp64, the shifted ratio does not
    r = np.array([0.0, 1000.0], np.float32)
    g = np.array([1.0, 3.0], np.float32)
    b = orc.solve(r, 1.0, 0.5)
    grad, _, _ = orc.vjp(r, g, b, 0.5)
    assert np.all(np.isfinite(grad))


# ------------------------------------------------ bracketing restatement pins
def test_philox_matches_numpy_bit_generator(orc):
    # numpy.random.Philox is Philox4x64-10 and advances its counter before each block
    for key in ([0, 0], [7, 9], [2**64 - 1, 12345]):
        key = np.array(key, dtype=np.uint64)            # numpy casts big Python ints through float
        for c0 in (0, 5, 2**40):
            bg = np.random.Philox(counter=np.array([c0, 0, 0, 0], np.uint64), key=key)
            assert np.array_equal(bg.random_raw(4).astype(np.uint64), orc.philox([c0 + 1, 0, 0, 0], key))
    bg = np.random.Philox(counter=np.array([2**64 - 1, 3, 0, 0], np.uint64), key=np.array([1, 2], np.uint64))
    assert np.array_equal(bg.random_raw(4).astype(np.uint64), orc.philox([0, 4, 0, 0], [1, 2]))


def test_own_log_is_within_two_ulp(orc):
    xs = np.concatenate([np.random.default_rng(5).random(20000),
                         np.logspace(-15.9, 0, 2000), [1.0, 0.5, 2.0 ** -53, 1 - 2.0 ** -53]])
    for x in xs:
        if x <= 0:
            continue
        got, ref = orc.ln(float(x)), math.log(float(x))
        assert abs(got - ref) <= 2 * math.ulp(ref) or got == ref


def test_sample_noise_is_laplace_and_hits_budget_quantile(orc):
    # P(y > b) = k/n for y = r_I + t L, L ~ Laplace(0,1) (the operator's own noise kernel)
    r = _row(5000, seed=9)
    k, t = 250.0, 0.2
    b = orc.solve(r, k, t)
    s = 200_000
    y, idx = orc.sample(r, t, seed=3, s=s)
    assert idx.min() >= 0 and idx.max() < r.size
    # indices are uniform: chi-square over 50 bins
    hist = np.bincount(idx * 50 // r.size, minlength=50)
    assert st.chisquare(hist).pvalue > 1e-4
    L = (y - r[idx].astype(np.float64)) / t
    assert st.kstest(L, st.laplace.cdf).pvalue > 1e-4
    frac = np.mean(y > b)
    pi = k / r.size
    assert abs(frac - pi) <= 5 * math.sqrt(pi * (1 - pi) / s)


@pytest.mark.parametrize("s,pi,delta", [(65536, 0.01, 1e-6), (16384, 210 / 1048576, 1e-6),
                                        (4096, 0.3, 0.5), (1000, 0.5, 1e-3), (50, 0.02, 0.1)])
def test_binomial_ranks_match_scipy(orc, s, pi, delta):
    jR, jL = orc.binom_ranks(s, pi, delta)
    d = st.binom(s, pi)
    # jR: largest j with P(X < j) <= delta/2
    assert jR == 0 or d.cdf(jR - 1) <= delta / 2
    assert d.cdf(jR) > delta / 2
    # jL: smallest j with P(X >= j) <= delta/2
    assert jL == s + 1 or d.sf(jL - 1) <= delta / 2
    assert jL == 0 or d.sf(jL - 2) > delta / 2
    assert jR < jL


def test_bracket_coverage_rate(orc):
    # over many seeds the bracket misses b with probability <= delta
    r = _row(3000, seed=21)
    k, t, s, delta = 60.0, 0.1, 512, 0.2
    b = orc.solve(r, k, t)
    misses = 0
    trials = 1500
    for seed in range(trials):
        br = orc.bracket(r, k, t, seed, s, delta)
        ok = float(br["a_L"]) <= b < float(br["a_R"])
        misses += not ok
        cert = orc.certify(r, k, t, br["a_L"], br["a_R"], band_cap=r.size)
        assert cert["verdict"] == int(ok)                    # certification == truth
        assert cert["c_L"] + cert["c_band"] + cert["c_R"] == r.size
    rate = misses / trials
    assert rate <= delta + 3 * math.sqrt(delta * (1 - delta) / trials)


def test_bracket_ends_are_outward_order_statistics(orc):
    r = _row(4000, seed=22)
    k, t, s, delta = 40.0, 0.05, 2048, 1e-3
    br = orc.bracket(r, k, t, 11, s, delta)
    y, _ = orc.sample(r, t, 11, s)
    ys = np.sort(y)[::-1]
    jR, jL = br["jR"], br["jL"]
    assert 0 < jR < jL <= s
    assert float(br["a_R"]) > ys[jR - 1] and np.float32(br["a_R"]) == np.nextafter(
        np.float32(np.nextafter(np.float32(ys[jR - 1]), np.float32(-np.inf))
                   if float(np.float32(ys[jR - 1])) > ys[jR - 1] else np.float32(ys[jR - 1])),
        np.float32(np.inf))
    assert float(br["a_L"]) <= ys[jL - 1] and float(np.nextafter(br["a_L"], np.float32(np.inf))) > ys[jL - 1]


def test_counts_partition(orc):
    r = _row(10000, seed=23)
    r[5] = np.nan
    cl, cb, cr = orc.counts(r, -0.5, 1.5)
    ok = r[np.isfinite(r)]
    assert (cl, cb, cr) == (int((ok < -0.5).sum()), int(((ok >= -0.5) & (ok < 1.5)).sum()),
                            int((ok >= 1.5).sum()))
    assert cl + cb + cr == r.size - 1


def _scipy_ranks(s, pi, delta):
    # jR: largest j with P(X < j) <= delta/2; jL: smallest j with P(X >= j) <= delta/2
    X = st.binom(s, pi)
    jR = max([j for j in range(0, s + 1) if X.cdf(j - 1) <= delta / 2] + [0])
    jL = min([j for j in range(0, s + 2) if X.sf(j - 1) <= delta / 2])
    return jR, jL


@pytest.mark.parametrize("s,pi,delta", [(256, 5000 / 2**20, 0.5), (64, 20000 / 2**20, 0.9),
                                        (4096, 0.01, 1e-3), (65536, 0.01, 1e-6), (512, 0.3, 0.2)])
def test_widen_ranks_pinned_to_binomial_tails(orc, s, pi, delta):
    # the widening round's ranks: at least as far out as the delta^2 tails
    # (scipy), at least one first-round spread beyond the first round, in [0, s+1]
    jR, jL = _scipy_ranks(s, pi, delta)
    r2, l2 = _scipy_ranks(s, pi, max(delta * delta, 1e-300))
    jR2, jL2 = orc.widen_ranks(s, pi, delta)
    spread = max(1, jL - jR)
    assert 0 <= jR2 <= min(r2, max(0, jR - spread)) and (jR2 == 0 or jR2 == min(r2, jR - spread))
    assert max(l2, min(s + 1, jL + spread)) <= jL2 <= s + 1 and (jL2 == s + 1 or jL2 == max(l2, jL + spread))
    assert jR2 < jR or jR == 0
    assert jL2 > jL or jL == s + 1


def test_widen_ranks_worked_cases(orc):
    # s = 256, pi = 5000/2^20, delta = 0.5: the first-round ranks are (0, 3) and the
    # delta^2 ranks are (0, 3) too, so only the one-spread rule moves jL: (0, 6)
    assert orc.binom_ranks(256, 5000 / 2**20, 0.5) == (0, 3)
    assert orc.binom_ranks(256, 5000 / 2**20, 0.25) == (0, 3)
    assert orc.widen_ranks(256, 5000 / 2**20, 0.5) == (0, 6)


def test_bracket_at_ranks_is_outward_order_statistics(orc):
    r = _row(4000, seed=24)
    t, s, seed = 0.05, 1024, 5
    y, _ = orc.sample(r, t, seed, s)
    ys = np.sort(y)[::-1]
    for jR, jL in [(0, 1), (3, 17), (100, 1025), (1024, 1024)]:
        br = orc.bracket_at_ranks(r, t, seed, s, jR, jL)
        if jR == 0:
            assert br["a_R"] == np.float32(np.inf)
        else:
            f = np.float32(ys[jR - 1])
            down = f if float(f) <= ys[jR - 1] else np.nextafter(f, np.float32(-np.inf))
            assert br["a_R"] == np.nextafter(down, np.float32(np.inf))
        if jL == s + 1:
            assert br["a_L"] == np.float32(-np.inf)
        else:
            assert float(br["a_L"]) <= ys[jL - 1] < float(np.nextafter(br["a_L"], np.float32(np.inf)))
    # at the first-round ranks it is the bracket itself
    k, delta = 40.0, 1e-3
    b1 = orc.bracket(r, k, t, seed, s, delta)
    b2 = orc.bracket_at_ranks(r, t, seed, s, b1["jR"], b1["jL"])
    assert (b1["a_L"], b1["a_R"]) == (b2["a_L"], b2["a_R"])


# ------------------------------------------------- sort and the tail sums
def test_sort_desc_matches_numpy_sort(orc):
    r = np.concatenate([RNG.standard_normal(5000), np.repeat([0.5, -0.0, 0.0, 3e-39], 100),
                        [np.float32(3.4e38), -np.float32(3.4e38)]]).astype(np.float32)
    RNG.shuffle(r)
    out = orc.sort_desc(r)
    ref = np.sort(r.astype(np.float64))[::-1]
    assert np.array_equal(out, ref)


@pytest.mark.parametrize("m,t", [(50, 0.1), (400, 0.1), (3000, 0.02)])
def test_tail_sums_geometric_closed_form(orc, m, t):
    # scores on a grid of step D below a_L (i = 1..m) and at or above a_R (i = 0..m-1):
    # the tail sums are geometric series in q = e^{-D/t}; the terms with z = iD/t > 16
    # form the tails of those series.  Band scores (a_L <= r < a_R) add nothing.
    D = 1.0 / 64
    aL, aR = np.float32(-1.0), np.float32(2.0)
    i = np.arange(1, m + 1)
    below = (np.float64(aL) - i * D).astype(np.float32)
    above = (np.float64(aR) + (i - 1) * D).astype(np.float32)
    band = np.array([aL, 0.0, np.nextafter(aR, np.float32(0))], np.float32)
    r = np.concatenate([below, above, band])
    RNG.shuffle(r)
    q = math.exp(-D / t)
    got = orc.tail_sums(r, aL, aR, t)
    geo = lambda a, b: (q ** a - q ** (b + 1)) / (1 - q)   # sum_{j=a}^{b} q^j
    far_from = math.floor(16 * t / D) + 1                    # first j with jD/t > 16
    assert abs(got["S_L"] - geo(1, m)) <= 1e-13 * geo(1, m)
    assert abs(got["S_R"] - geo(0, m - 1)) <= 1e-13 * geo(0, m - 1)
    want_far_L = geo(far_from, m) if m >= far_from else 0.0
    want_far_R = geo(far_from, m - 1) if m - 1 >= far_from else 0.0
    assert abs(got["S_L_far"] - want_far_L) <= 1e-13 * max(want_far_L, 1e-300)
    assert abs(got["S_R_far"] - want_far_R) <= 1e-13 * max(want_far_R, 1e-300)


def test_tail_sums_match_scipy_logsumexp(orc):
    from scipy.special import logsumexp
    r = RNG.laplace(0.0, 1.0, 200_000).astype(np.float32)
    t = 0.05
    for aL, aR in ((np.float32(1.5), np.float32(1.75)), (np.float32(-np.inf), np.float32(0.3)),
                   (np.float32(-0.2), np.float32(np.inf))):
        got = orc.tail_sums(r, aL, aR, t)
        lo = r[r < aL].astype(np.float64)
        hi = r[r >= aR].astype(np.float64)
        SL = math.exp(logsumexp((lo - float(aL)) / t)) if lo.size else 0.0
        SR = math.exp(logsumexp(-(hi - float(aR)) / t)) if hi.size else 0.0
        assert abs(got["S_L"] - SL) <= 1e-12 * max(SL, 1e-300)
        assert abs(got["S_R"] - SR) <= 1e-12 * max(SR, 1e-300)


# ------------------------------------------------------ stored expected values
def test_golden_forced_fallback_is_reproduced_by_the_oracle(orc):
    # tests/golden/forced_fallback.json holds values written by the oracle alone
    # (tests/golden/make_golden.py): running the script's computation again gives
    # every stored field exactly (seed, ranks, bracket ends, counts, G values, b)
    import importlib.util
    import json
    import os
    here = os.path.join(os.path.dirname(os.path.abspath(__file__)), "golden")
    spec = importlib.util.spec_from_file_location("make_golden", os.path.join(here, "make_golden.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    stored = json.load(open(os.path.join(here, "forced_fallback.json")))
    assert mod.forced_fallback() == stored
