"""GPU parity of the CUDA path against the fp64 oracle, through the C ABI.

Tolerances (the method's exact-budget operator, "Fast LapSum: Exact
Differentiable Top-k at Million Scale", technical summary section 2.1):
  |b_gpu - b_ref| <= 1e-4 t;  max |p_gpu - p_ref| <= 1e-5;  |sum p - k| <= 1e-3;
  VJP relative L2 <= 1e-4.
Integer results of the bracketing path (ranks, bracket ends, membership
counts, certification verdict) must equal the oracle's restatement exactly.
"""

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TOL_B = 1e-4        # times t
TOL_P = 1e-5
TOL_SUM = 1e-3
TOL_VJP = 1e-4


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_budget_soft_b200 as lib
    return lib


def run(L, r_np, k, t, opts=None, g_np=None):
    r = torch.from_numpy(np.ascontiguousarray(r_np)).cuda()
    p, b = L.forward(r, k, t, opts=opts)
    st = L.get_stats(check=False)
    grad = None
    if g_np is not None:
        g = torch.from_numpy(np.ascontiguousarray(g_np)).cuda()
        grad = L.backward(r, b, g, t).cpu().numpy()
    torch.cuda.synchronize()
    return p.cpu().numpy(), b.cpu().numpy(), st, grad


def check_row(orc, r, g, k, t, p, b, grad, exact_sum=True):
    bref = orc.solve(r, k, t, method=1)
    assert abs(b - bref) <= TOL_B * t, (b, bref)
    pref = orc.p(r, bref, t)
    assert np.max(np.abs(p.astype(np.float64) - pref)) <= TOL_P
    G, _ = orc.G(r, b, t)                  # exact mass at the GPU's threshold
    assert abs(G - k) <= TOL_SUM
    if exact_sum:
        assert abs(p.astype(np.float64).sum() - k) <= TOL_SUM
    if grad is not None:
        gref, _, _ = orc.vjp(r, g, bref, t)
        assert np.linalg.norm(grad - gref) <= TOL_VJP * np.linalg.norm(gref)


# ------------------------------------------------------------ full sort --
@pytest.mark.parametrize("n", [1, 2, 3, 31, 33, 100, 1000, 4095, 4096, 4097, 8191, 20000, 32767, 32768])
def test_full_sort_single_row_ragged(L, orc, n):
    r, g = W.small_case("normal", 1, n, seed=n)
    k = min(max(0.5, n / 64), n - 0.5)
    t = 0.05
    p, b, st, grad = run(L, r, k, t, g_np=g)
    assert st["rc"] == 0
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


def test_n4096_workload(L, orc):
    w = W.WORKLOADS["n4096"]
    r, g = W.scores(w), W.upstream_grad(w)
    p, b, st, grad = run(L, r, w.k, w.t, g_np=g)
    assert st["rc"] == 0 and st["path"] == 1
    check_row(orc, r[0], g[0], w.k, w.t, p[0], b[0], grad[0])


@pytest.mark.parametrize("dist,k,t", [("normal", 256.0, 0.1), ("laplace", 7.5, 0.02),
                                      ("levels256_desc", 300.0, 0.1), ("uniform", 16000.0, 1e-3)])
def test_rows_batched(L, orc, dist, k, t):
    r, g = W.small_case(dist, 24, 32768, seed=3)
    p, b, st, grad = run(L, r, k, t, g_np=g)
    for i in range(r.shape[0]):
        check_row(orc, r[i], g[i], k, t, p[i], b[i], grad[i])


def test_rows1024_workload(L, orc):
    w = W.WORKLOADS["rows1024"]
    r, g = W.scores(w), W.upstream_grad(w)
    p, b, st, grad = run(L, r, w.k, w.t, g_np=g)
    sums = p.astype(np.float64).sum(axis=1)
    assert np.max(np.abs(sums - w.k)) <= TOL_SUM
    for i in (0, 1, 511, 1023):
        check_row(orc, r[i], g[i], w.k, w.t, p[i], b[i], grad[i])


def test_all_equal_and_ties(L, orc):
    r = np.full((2, 5000), 0.75, np.float32)
    r[1, ::2] = -0.25
    p, b, st, _ = run(L, r, 17.0, 0.3)
    for i in range(2):
        check_row(orc, r[i], None, 17.0, 0.3, p[i], b[i], None)


# ----------------------------------------------- device-wide full sort --
@pytest.mark.parametrize("n,dist", [(32769, "normal"), (100_000, "laplace"), (300_001, "normal"),
                                    (500_000, "levels256_desc"), (1_100_003, "normal"),
                                    (300_007, "levels256_shuffled"), (2_000_000, "levels256_shuffled")])
def test_device_sort_path(L, orc, n, dist):
    # the shuffled levels (few mantissa bits, both signs) make the sort skip the
    # two low digits (decided by the sign) and still reorder the row
    r, g = W.small_case(dist, 1, n, seed=7)
    k, t = n / 100.0, 0.05
    p, b, st, grad = run(L, r, k, t, opts=L.options(force_path=L.PATH_FULLSORT), g_np=g)
    assert st["rc"] == 0 and st["path"] == 1
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


@pytest.mark.parametrize("rows,n", [(3, 40_001), (2, 65_538)])
def test_device_sort_path_rows_unaligned(L, orc, rows, n):
    # rows after the first start off a 16-byte boundary (odd n, or n = 2 mod 4):
    # the sort's first pass and the histogram take their element-wise paths there
    r, g = W.small_case("normal", rows, n, seed=11)
    k, t = n / 50.0, 0.05
    p, b, st, grad = run(L, r, k, t, opts=L.options(force_path=L.PATH_FULLSORT), g_np=g)
    assert st["rc"] == 0
    for i in range(rows):
        check_row(orc, r[i], g[i], k, t, p[i], b[i], grad[i])


# ----------------------------------------------------------- bracketing --
def check_bracket_integers(orc, r, k, t, st, seed, s, delta):
    br = orc.bracket(r, k, t, seed, s, delta)
    assert (st["jR"], st["jL"]) == (br["jR"], br["jL"])
    assert np.float32(st["a_L"]) == br["a_L"] and np.float32(st["a_R"]) == br["a_R"]
    cert = orc.certify(r, k, t, br["a_L"], br["a_R"], band_cap=10**12)
    assert (st["c_L"], st["c_band"], st["c_R"]) == (cert["c_L"], cert["c_band"], cert["c_R"])
    return cert


@pytest.mark.parametrize("certify", [0, 1])
@pytest.mark.parametrize("n,dist,k,t", [(1 << 20, "normal", 1000.0, 0.05), (1_500_001, "laplace", 150.0, 0.01),
                                        (1 << 20, "levels256_desc", 20000.0, 0.1)])
def test_bracketing_parity(L, orc, n, dist, k, t, certify):
    r, g = W.small_case(dist, 1, n, seed=11)
    p, b, st, grad = run(L, r, k, t, opts=L.options(certify=certify), g_np=g)
    assert st["rc"] == 0 and st["path"] == 2
    plan = L.bracket_plan(n, k)
    cert = check_bracket_integers(orc, r[0], k, t, st, 0, plan["s"], 1e-6)
    assert st["verdict"] == cert["verdict"] == 1
    assert abs(st["G_aL"] - cert["G_aL"]) <= 1e-6 * max(1.0, cert["G_aL"])
    assert abs(st["G_aR"] - cert["G_aR"]) <= 1e-6 * max(1.0, cert["G_aR"])
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0], exact_sum=(dist != "levels256_desc"))


def test_pixels1m_workload(L, orc):
    w = W.WORKLOADS["pixels1m"]
    r, g = W.scores(w), W.upstream_grad(w)
    p, b, st, grad = run(L, r, w.k, w.t, g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1
    plan = L.bracket_plan(w.n, w.k)
    check_bracket_integers(orc, r[0], w.k, w.t, st, 0, plan["s"], 1e-6)
    check_row(orc, r[0], g[0], w.k, w.t, p[0], b[0], grad[0])


@pytest.mark.parametrize("certify", [0, 1])
def test_bracketing_large_band(L, orc, certify):
    # a small sample leaves a wide bracket: the band (~1e5 scores, untied) takes
    # narrowing steps over the band buffer before its copy in shared memory
    n = (1 << 21) + 12345
    r, g = W.small_case("laplace", 1, n, seed=12)
    k, t, s = n / 10.0, 0.05, 4096
    p, b, st, grad = run(L, r, k, t, opts=L.options(sample_size=s, certify=certify), g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1 and st["fallback"] == 0
    assert st["c_band"] > 32768
    check_bracket_integers(orc, r[0], k, t, st, 0, s, 1e-6)
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


@pytest.mark.parametrize("certify", [0, 1])
def test_forced_fallback_by_band_capacity(L, orc, certify):
    r, g = W.small_case("normal", 1, 1 << 20, seed=5)
    k, t = 3000.0, 0.05
    p, b, st, grad = run(L, r, k, t, opts=L.options(band_cap=64, certify=certify), g_np=g)
    assert st["rc"] == 0 and st["verdict"] == 0 and st["fallback"] == 1
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


@pytest.mark.parametrize("certify", [0, 1])
def test_forced_fallback_by_missed_bracket(L, orc, certify):
    # a tiny sample with delta = 0.5 misses often; the oracle picks a seed that misses
    r, g = W.small_case("normal", 1, 1 << 20, seed=6)
    k, t, s, delta = 5000.0, 0.05, 256, 0.5
    bref = orc.solve(r[0], k, t, method=1)
    seed = next(sd for sd in range(200)
                if not (float(orc.bracket(r[0], k, t, sd, s, delta)["a_L"]) <= bref <
                        float(orc.bracket(r[0], k, t, sd, s, delta)["a_R"])))
    p, b, st, grad = run(L, r, k, t, opts=L.options(seed=seed, sample_size=s, delta=delta, certify=certify),
                         g_np=g)
    cert = check_bracket_integers(orc, r[0], k, t, st, seed, s, delta)
    assert st["verdict"] == cert["verdict"] == 0 and st["fallback"] == 1
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


def test_nonfinite_scores_reported(L):
    r = np.random.default_rng(0).standard_normal((1, 5000)).astype(np.float32)
    r[0, 77] = np.nan
    _, _, st, _ = run(L, r, 10.0, 0.1)
    assert st["rc"] == -2


def test_reproducible_bits(L):
    r, _ = W.small_case("laplace", 1, 1 << 20, seed=2)
    _, b1, _, _ = run(L, r, 500.0, 0.05)
    _, b2, _, _ = run(L, r, 500.0, 0.05)
    assert b1.tobytes() == b2.tobytes()


def test_autograd_function(L, orc):
    r, g = W.small_case("normal", 4, 4096, seed=9)
    x = torch.from_numpy(r).cuda().requires_grad_(True)
    p = L.soft_topk(x, 64.0, 0.05)
    p.backward(torch.from_numpy(g).cuda())
    b = L.forward(torch.from_numpy(r).cuda(), 64.0, 0.05)[1].cpu().numpy()
    for i in range(4):
        gref, _, _ = orc.vjp(r[i], g[i], orc.solve(r[i], 64.0, 0.05, 1), 0.05)
        assert np.linalg.norm(x.grad[i].cpu().numpy() - gref) <= TOL_VJP * np.linalg.norm(gref)


# ------------------------------------------------- full-size workloads --
@pytest.mark.slow
def test_laplace1e7_workload(L, orc):
    w = W.WORKLOADS["laplace1e7"]
    r, g = W.scores(w), W.upstream_grad(w)
    p, b, st, grad = run(L, r, w.k, w.t, g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1
    plan = L.bracket_plan(w.n, w.k)
    check_bracket_integers(orc, r[0], w.k, w.t, st, 0, plan["s"], 1e-6)
    check_row(orc, r[0], g[0], w.k, w.t, p[0], b[0], grad[0])


def check_large(orc, r, g, k, t, p, b, grad, rng):
    # b: G straddles k within +-1e-4 t of the GPU's b (G is decreasing)
    assert orc.G(r, b - TOL_B * t, t)[0] >= k >= orc.G(r, b + TOL_B * t, t)[0]
    G, _ = orc.G(r, b, t)
    assert abs(G - k) <= TOL_SUM
    bref = orc.solve(r, k, t, method=1)
    assert abs(b - bref) <= TOL_B * t
    idx = rng.integers(0, r.size, 200_000)
    assert np.max(np.abs(p[idx].astype(np.float64) - orc.p(r[idx], bref, t))) <= TOL_P
    if grad is not None:
        gref, _, _ = orc.vjp(r, g, bref, t)
        assert np.linalg.norm(grad - gref) <= TOL_VJP * np.linalg.norm(gref)


@pytest.mark.slow
def test_levels1e8_workload_and_forced_fallback(L, orc):
    w = W.WORKLOADS["levels1e8"]
    r, g = W.scores(w)[0], W.upstream_grad(w)[0]
    rng = np.random.default_rng(0)
    p, b, st, grad = run(L, r, w.k, w.t, g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1 and st["fallback"] == 0
    plan = L.bracket_plan(w.n, w.k)
    check_bracket_integers(orc, r, w.k, w.t, st, 0, plan["s"], 1e-6)
    check_large(orc, r, g, w.k, w.t, p, b[0], grad, rng)
    # the rounded-p sum is off by the shared rounding of ~4e5 tied scores; its bound:
    ps = p.astype(np.float64).sum()
    ulp_bound = np.sum(np.spacing(p.astype(np.float32)).astype(np.float64)) / 2
    assert abs(ps - w.k) <= ulp_bound + TOL_SUM
    del p, grad
    # forced fallback: a bracket that certification rejects
    import json, os
    gold = json.load(open(os.path.join(os.path.dirname(__file__), "golden", "forced_fallback.json")))
    o = L.options(seed=gold["seed"], sample_size=gold["sample_size"], delta=gold["delta"])
    p2, b2, st2, _ = run(L, r, w.k, w.t, opts=o)
    assert st2["verdict"] == 0 and st2["fallback"] == 1 and st2["rc"] == 0
    assert np.float32(st2["a_L"]) == np.float32(gold["a_L"]) and np.float32(st2["a_R"]) == np.float32(gold["a_R"])
    assert (st2["c_L"], st2["c_band"], st2["c_R"]) == (gold["c_L"], gold["c_band"], gold["c_R"])
    check_large(orc, r, None, w.k, w.t, p2, b2[0], None, rng)


@pytest.mark.slow
def test_levels1e8_in_random_order(L, orc):
    # the same 1e8 tied scores shuffled (the bench's random-order line): no warp
    # of the out-of-band passes sees one side of the bracket, a fifth of the
    # scores take the staged fp64 terms; bracket and counts exact, b, sampled p
    # and the VJP to tolerance
    w = W.WORKLOADS["levels1e8_shuffled"]
    r, g = W.scores(w)[0], W.upstream_grad(w)[0]
    rng = np.random.default_rng(1)
    p, b, st, grad = run(L, r, w.k, w.t, g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1 and st["fallback"] == 0
    plan = L.bracket_plan(w.n, w.k)
    cert = check_bracket_integers(orc, r, w.k, w.t, st, 0, plan["s"], 1e-6)
    assert abs(st["G_aL"] - cert["G_aL"]) <= 1e-6 * max(1.0, cert["G_aL"])
    assert abs(st["G_aR"] - cert["G_aR"]) <= 1e-6 * max(1.0, cert["G_aR"])
    check_large(orc, r, g, w.k, w.t, p, b[0], grad, rng)


@pytest.mark.slow
def test_batch64x1m_workload(L, orc):
    # the bench's batched-bracketing line: 64 rows of 2^20 N(0,1) scores, each
    # with its own bracket (Philox counter word = row), band and certification
    w = W.WORKLOADS["batch64x1m"]
    r, g = W.scores(w), W.upstream_grad(w)
    p, b, sts, grad = run_rows(L, r, w.k, w.t, g_np=g)
    plan = L.bracket_plan(w.n, w.k)
    for i in range(w.rows):
        st = sts[i]
        e = expected_row(orc, r[i], w.k, w.t, 0, plan["s"], 1e-6, i)
        assert st["rc"] == 0 and st["verdict"] == e["cert"]["verdict"] == 1
        assert np.float32(st["a_L"]) == e["br"]["a_L"] and np.float32(st["a_R"]) == e["br"]["a_R"]
        assert (st["c_L"], st["c_band"], st["c_R"]) == (e["cert"]["c_L"], e["cert"]["c_band"], e["cert"]["c_R"])
        check_row(orc, r[i], g[i], w.k, w.t, p[i], b[i], grad[i])


@pytest.mark.parametrize("certify", [0, 1])
@pytest.mark.parametrize("level", [0, 1, 2])
def test_bracketing_band_of_one_tied_level(L, orc, level, certify):
    # sorted, 32 tied levels of 65536 scores: the band holds one whole level (or
    # none); one level exceeds one CTA, so the histogram kernel solves it in closed form
    n = 1 << 21
    vals = (-1.0 + (np.arange(32) + 0.5) / 16).astype(np.float32)
    r = np.repeat(vals[::-1], n // 32)[None, :].copy()
    g = np.random.default_rng(level).standard_normal((1, n)).astype(np.float32)
    k = [n / 32 * 1.5, n / 32 * 3.25, n / 32 * 0.4][level]
    t = 0.05
    p, b, st, grad = run(L, r, k, t, opts=L.options(certify=certify), g_np=g)
    assert st["rc"] == 0 and st["path"] == 2
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0], exact_sum=False)


# ------------------------------------------------ bracket widening (NEXT-1) --
def widened_bracket(orc, r, k, t, seed, s, delta):
    """The oracle's prediction of the widening round: first-round bracket, the
    side it missed (from its certification), and the bracket of the second round
    (the missed side, up to the delta^2 order statistic of the same sample)."""
    br1 = orc.bracket(r, k, t, seed, s, delta)
    c1 = orc.certify(r, k, t, br1["a_L"], br1["a_R"], band_cap=10**12)
    if c1["verdict"] == 1:
        return br1, 0, None
    jR2, jL2 = orc.widen_ranks(s, k / r.size, delta)
    br2 = orc.bracket_at_ranks(r, t, seed, s, jR2, jL2)
    if c1["G_aR"] >= k:   # b at or above a_R
        return br1, 1, {"a_L": br1["a_R"], "a_R": br2["a_R"], "jL": br1["jR"], "jR": br2["jR"]}
    assert c1["G_aL"] < k
    return br1, -1, {"a_L": br2["a_L"], "a_R": br1["a_L"], "jL": br2["jL"], "jR": br1["jL"]}


def find_widen_seed(orc, r, k, t, s, delta, want_cover):
    for sd in range(400):
        _, d, br2 = widened_bracket(orc, r, k, t, sd, s, delta)
        if d == 0:
            continue
        c2 = orc.certify(r, k, t, br2["a_L"], br2["a_R"], band_cap=10**12)
        if (c2["verdict"] == 1) == want_cover:
            return sd, d, br2, c2
    raise AssertionError("no seed found")


@pytest.mark.parametrize("certify", [0, 1])
def test_widening_recovers_a_missed_bracket(L, orc, certify):
    r, g = W.small_case("normal", 1, 1 << 20, seed=6)
    k, t, s, delta = 5000.0, 0.05, 256, 0.5
    seed, d, br2, c2 = find_widen_seed(orc, r[0], k, t, s, delta, want_cover=True)
    p, b, st, grad = run(L, r, k, t, opts=L.options(seed=seed, sample_size=s, delta=delta, certify=certify,
                                                     widen=1), g_np=g)
    assert st["rc"] == 0 and st["widened"] == 1 and st["verdict"] == 1 and st["fallback"] == 0
    assert np.float32(st["a_L"]) == br2["a_L"] and np.float32(st["a_R"]) == br2["a_R"]
    assert (st["jR"], st["jL"]) == (br2["jR"], br2["jL"])
    assert (st["c_L"], st["c_band"], st["c_R"]) == (c2["c_L"], c2["c_band"], c2["c_R"])
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


@pytest.mark.parametrize("certify", [0, 1])
def test_widening_that_misses_again_falls_back(L, orc, certify):
    r, g = W.small_case("laplace", 1, 1 << 20, seed=8)
    k, t, s, delta = 20000.0, 0.05, 64, 0.9
    seed, d, br2, c2 = find_widen_seed(orc, r[0], k, t, s, delta, want_cover=False)
    p, b, st, grad = run(L, r, k, t, opts=L.options(seed=seed, sample_size=s, delta=delta, certify=certify,
                                                     widen=1), g_np=g)
    assert st["rc"] == 0 and st["widened"] == 1 and st["verdict"] == 0 and st["fallback"] == 1
    assert np.float32(st["a_L"]) == br2["a_L"] and np.float32(st["a_R"]) == br2["a_R"]
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


def test_widening_not_needed_changes_nothing(L, orc):
    r, g = W.small_case("normal", 1, 1 << 20, seed=9)
    k, t = 1000.0, 0.05
    p0, b0, st0, _ = run(L, r, k, t)
    p1, b1, st1, grad = run(L, r, k, t, opts=L.options(widen=1), g_np=g)
    assert st1["widened"] == 0 and st1["verdict"] == 1 and st1["fallback"] == 0
    assert b1[0] == b0[0] and np.array_equal(p1, p0)
    check_row(orc, r[0], g[0], k, t, p1[0], b1[0], grad[0])


def test_widening_skips_band_overflow(L, orc):
    # a bracket that holds b but whose band overflows is not widened: full sort
    r, g = W.small_case("normal", 1, 1 << 20, seed=5)
    k, t = 3000.0, 0.05
    p, b, st, grad = run(L, r, k, t, opts=L.options(band_cap=64, widen=1), g_np=g)
    assert st["widened"] == 0 and st["verdict"] == 0 and st["fallback"] == 1
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


# ------------------------------------------------ batched bracketing (NEXT-3) --
def run_rows(L, r_np, k, t, opts=None, g_np=None):
    r = torch.from_numpy(np.ascontiguousarray(r_np)).cuda()
    p, b = L.forward(r, k, t, opts=opts)
    sts = L.get_stats_rows(r.shape[0], check=False)
    grad = None
    if g_np is not None:
        g = torch.from_numpy(np.ascontiguousarray(g_np)).cuda()
        grad = L.backward(r, b, g, t).cpu().numpy()
    torch.cuda.synchronize()
    return p.cpu().numpy(), b.cpu().numpy(), sts, grad


def expected_row(orc, r, k, t, seed, s, delta, row, widen=False):
    """The oracle's bracket of one row of a batch (its own Philox counter word),
    the certification outcome, and -- with widening -- the second round."""
    br = orc.bracket(r, k, t, seed, s, delta, row=row)
    c = orc.certify(r, k, t, br["a_L"], br["a_R"], band_cap=10**12)
    out = {"br": br, "cert": c, "widened": 0}
    if widen and c["verdict"] == 0:
        jR2, jL2 = orc.widen_ranks(s, k / r.size, delta)
        b2 = orc.bracket_at_ranks(r, t, seed, s, jR2, jL2, row=row)
        if c["G_aR"] >= k:
            nb = {"a_L": br["a_R"], "a_R": b2["a_R"], "jL": br["jR"], "jR": jR2}
        else:
            nb = {"a_L": b2["a_L"], "a_R": br["a_L"], "jL": jL2, "jR": br["jL"]}
        out.update(br=nb, cert=orc.certify(r, k, t, nb["a_L"], nb["a_R"], band_cap=10**12), widened=1)
    return out


@pytest.mark.parametrize("certify", [0, 1])
def test_batched_bracketing_rows(L, orc, certify):
    # three rows of a ragged length (rows start off 16-byte boundaries): one
    # launch sequence, every row bracketed, certified and solved on its own
    rows, n = 3, (1 << 20) + 123
    r, g = W.small_case("laplace", rows, n, seed=13)
    k, t = 2000.0, 0.05
    p, b, sts, grad = run_rows(L, r, k, t, opts=L.options(certify=certify), g_np=g)
    plan = L.bracket_plan(n, k)
    assert len(sts) == rows
    for i in range(rows):
        st = sts[i]
        assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1 and st["fallback"] == 0
        e = expected_row(orc, r[i], k, t, 0, plan["s"], 1e-6, i)
        assert np.float32(st["a_L"]) == e["br"]["a_L"] and np.float32(st["a_R"]) == e["br"]["a_R"]
        assert (st["c_L"], st["c_band"], st["c_R"]) == (e["cert"]["c_L"], e["cert"]["c_band"], e["cert"]["c_R"])
        check_row(orc, r[i], g[i], k, t, p[i], b[i], grad[i])


@pytest.mark.parametrize("widen", [0, 1])
def test_batched_rows_with_misses(L, orc, widen):
    # a weak bracket (s = 256, delta = 0.5) misses on some rows: each row's
    # verdict, widening and fallback follow that row's own certification
    # (Philox seed 10: by the oracle, rows 0 and 4 miss; widening recovers row 0
    # and row 4 misses again)
    rows, n = 6, 1 << 20
    r, g = W.small_case("normal", rows, n, seed=14)
    k, t, s, delta, seed = 5000.0, 0.05, 256, 0.5, 10
    p, b, sts, grad = run_rows(L, r, k, t, opts=L.options(seed=seed, sample_size=s, delta=delta, widen=widen),
                               g_np=g)
    outcomes = set()
    for i in range(rows):
        st = sts[i]
        e = expected_row(orc, r[i], k, t, seed, s, delta, i, widen=bool(widen))
        assert st["rc"] == 0 and st["widened"] == e["widened"]
        assert np.float32(st["a_L"]) == e["br"]["a_L"] and np.float32(st["a_R"]) == e["br"]["a_R"]
        assert st["verdict"] == e["cert"]["verdict"] and st["fallback"] == 1 - e["cert"]["verdict"]
        outcomes.add((st["verdict"], st["widened"]))
        check_row(orc, r[i], g[i], k, t, p[i], b[i], grad[i])
    assert len(outcomes) > 1   # the batch mixes rows that pass and rows that do not


def test_batched_rows_all_fall_back(L, orc):
    # every row's band overflows: the cooperative sort walks all rows
    rows, n = 3, (1 << 20) + 5
    r, g = W.small_case("normal", rows, n, seed=15)
    k, t = 3000.0, 0.05
    p, b, sts, grad = run_rows(L, r, k, t, opts=L.options(band_cap=64), g_np=g)
    for i in range(rows):
        assert sts[i]["verdict"] == 0 and sts[i]["fallback"] == 1 and sts[i]["rc"] == 0
        check_row(orc, r[i], g[i], k, t, p[i], b[i], grad[i])


@pytest.mark.parametrize("s,lo,hi", [(65536, 0, 4096), (16384, 4096, 16384), (2048, 16384, 32768)])
def test_band_select_sizes(L, orc, s, lo, hi):
    # the sample size sets the band's size: a band of at most 4096 scores is
    # copied to shared memory before the first narrowing step, a longer one is
    # narrowed from the band buffer first
    n = 1 << 20
    r, g = W.small_case("normal", 1, n, seed=16)
    k, t = n / 100.0, 0.05
    br = orc.bracket(r[0], k, t, 0, s, 1e-6)
    cert = orc.certify(r[0], k, t, br["a_L"], br["a_R"], band_cap=10**12)
    assert lo < cert["c_band"] <= hi
    p, b, st, grad = run(L, r, k, t, opts=L.options(sample_size=s), g_np=g)
    assert st["rc"] == 0 and st["verdict"] == 1 and st["c_band"] == cert["c_band"]
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


@pytest.mark.parametrize("t", [0.02, 0.05])
def test_band_select_short_band_of_a_few_tied_levels(L, orc, t):
    # a short band (at most 4096 scores, copied to shared memory at once) of three
    # or four whole tied levels: the narrowing ends on one level or on the gap
    # between two
    n = 1 << 18
    r, g = W.small_case("levels256_desc", 1, n, seed=22)
    k = 1.5 * n / 256
    p, b, st, grad = run(L, r, k, t, opts=L.options(force_path=L.PATH_BRACKET), g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1
    band = r[0][(r[0] >= np.float32(st["a_L"])) & (r[0] < np.float32(st["a_R"]))]
    assert 0 < band.size <= 4096 and np.unique(band).size >= 3 and st["c_band"] == band.size
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0], exact_sum=False)


@pytest.mark.parametrize("certify", [0, 1])
def test_band_select_band_across_zero(L, orc, certify):
    # k = n/2 puts the band around 0: its keys span both signs (a 31-bit key
    # range), which takes the full four narrowing steps
    n = 1 << 20
    r, g = W.small_case("normal", 1, n, seed=19)
    k, t = n / 2.0, 0.05
    p, b, st, grad = run(L, r, k, t, opts=L.options(certify=certify), g_np=g)
    assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1
    plan = L.bracket_plan(n, k)
    cert = check_bracket_integers(orc, r[0], k, t, st, 0, plan["s"], 1e-6)
    band = r[0][(r[0] >= np.float32(st["a_L"])) & (r[0] < np.float32(st["a_R"]))]
    assert band.min() < 0.0 < band.max() and cert["c_band"] > 4096
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


def test_band_select_tied_runs_longer_than_the_copy(L, orc):
    # 256 tied levels of ~16k scores each; a small sample (4096) widens the
    # bracket so the band holds several whole levels, and the narrowing ends on
    # one level (more scores than the shared-memory copy holds) or on the gap
    # between two, both in closed form
    n = 1 << 22
    r, g = W.small_case("levels256_desc", 1, n, seed=20)
    for k in (2.5 * n / 256, 40.0 * n / 256):
        p, b, st, grad = run(L, r, k, 0.02, opts=L.options(sample_size=4096), g_np=g)
        assert st["rc"] == 0 and st["path"] == 2 and st["verdict"] == 1
        band = r[0][(r[0] >= np.float32(st["a_L"])) & (r[0] < np.float32(st["a_R"]))]
        assert np.unique(band).size >= 2 and band.size > 4096
        check_row(orc, r[0], g[0], k, 0.02, p[0], b[0], grad[0], exact_sum=False)


def test_band_select_root_above_the_band(L, orc):
    # 3000 scores in [1, 1.1] over a N(0, 0.1^2) bulk, k = 3010, t = 0.2: b lies
    # above every score of the cluster, and with some seeds the bracket's upper
    # end lies above b with no band score in [b, a_R) -- the root is in the
    # band's top interval, a regular case (no NO_ROOT)
    n = 1 << 20
    rng = np.random.default_rng(21)
    r = (0.1 * rng.standard_normal(n)).astype(np.float32)
    r[:3000] = rng.uniform(1.0, 1.1, 3000).astype(np.float32)
    rng.shuffle(r)
    g = rng.standard_normal(n).astype(np.float32)
    k, t = 3010.0, 0.2
    bref = orc.solve(r, k, t, method=1)
    plan = L.bracket_plan(n, k)

    def top_interval(seed):
        br = orc.bracket(r, k, t, seed, plan["s"], 1e-6)
        band = r[(r >= br["a_L"]) & (r < br["a_R"])]
        return br["a_L"] <= bref < br["a_R"] and band.size > 0 and float(band.max()) < bref

    seed = next(sd for sd in range(64) if top_interval(sd))
    p, b, st, grad = run(L, r[None, :], k, t, opts=L.options(seed=seed), g_np=g[None, :])
    assert st["rc"] == 0 and st["verdict"] == 1 and st["fallback"] == 0
    assert not (st["status"] & 8)
    check_row(orc, r, g, k, t, p[0], b[0], grad[0])


# ------------------------------------------------------- bracketing edges --
@pytest.mark.parametrize("k,t", [(1.5, 0.05), ((1 << 20) - 3.0, 0.05), (1000.0, 1e-4), (300000.0, 50.0)])
def test_bracketing_extreme_budgets_and_temperatures(L, orc, k, t):
    # k near 0 (a_R = +inf) and near n (a_L = -inf); a tiny t (nearly hard top-k)
    # and a large one (p nearly k/n everywhere)
    n = 1 << 20
    r, g = W.small_case("normal", 1, n, seed=17)
    p, b, st, grad = run(L, r, k, t, g_np=g)
    assert st["rc"] == 0 and st["path"] == 2
    plan = L.bracket_plan(n, k)
    check_bracket_integers(orc, r[0], k, t, st, 0, plan["s"], 1e-6)
    # with t large every p is mid-range (p ~ k/n): the plain sum of the returned
    # fp32 p keeps the budget too (no bias adds up over the 2^20 scores)
    check_row(orc, r[0], g[0], k, t, p[0], b[0], grad[0])


def test_batched_rows_report_a_nonfinite_row(L):
    rows, n = 3, 1 << 20
    r, _ = W.small_case("normal", rows, n, seed=18)
    r[1, 12345] = np.nan
    rt = torch.from_numpy(r).cuda()
    L.forward(rt, 1000.0, 0.05)
    sts = L.get_stats_rows(rows, check=False)
    assert sts[0]["rc"] == L.ERR_NONFINITE
    assert (sts[1]["status"] & 1) and not (sts[0]["status"] & 1) and not (sts[2]["status"] & 1)
