"""GPU parity on the rare routes of the CUDA path, through the C ABI, against the
fp64 oracle ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
technical summary sections 2.1-2.2; tolerances as in test_gpu_parity.py):

* the VJP when the threshold lies far from every score, so that the densities
  f_i are fp32 denormals or underflow altogether (the shifted ratio);
* the bracket select whose candidate buffer overflows (many sample keys under
  one 16-bit prefix: few tied score levels at a tiny temperature);
* the streaming pass's tail sums S_L, S_R and the certification values against
  their definitions, with an error bound derived from the tiered arithmetic;
* every row of the 1024 x 32768 workload;
* the plain lapsum_forward entry point on device buffers;
* a grid-barrier wait of the device-wide sort made to give up at once: the
  call reports the timeout and the next call is clean;
* calls on a non-blocking stream whose workspace is new (zeroed on that stream):
  bit-equal to the same calls on the default stream;
* the binding refusing output and input buffers of the wrong size before any
  launch.
"""
import ctypes as C
import math

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


def rel_l2(a, b):
    a, b = np.asarray(a, np.float64), np.asarray(b, np.float64)
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def two_clusters(n, half_gap, jitter, seed):
    """n scores in two equal clusters at +-half_gap (uniform jitter), shuffled, and g."""
    rng = np.random.default_rng(seed)
    r = np.empty(n, np.float64)
    r[: n // 2] = half_gap
    r[n // 2:] = -half_gap
    r += jitter * rng.uniform(-1.0, 1.0, n)
    rng.shuffle(r)
    g = rng.standard_normal(n).astype(np.float32)
    return r.astype(np.float32), g


# --------------------------------------------------- VJP far from every score --
@pytest.mark.parametrize("n", [4096, 1 << 17])
@pytest.mark.parametrize("half_gap,t", [(3.0, 0.05),        # nearest |x| ~ 60: fp32 densities, plain sums
                                        (4.5, 0.05),        # nearest |x| ~ 90: fp32 denormal densities
                                        (1.2e-28, 1e-30)])  # nearest |x| ~ 120: every f underflows,
def test_vjp_far_from_every_score(L, orc, n, half_gap, t):  # yet f/t is an fp32 number
    r, g = two_clusters(n, half_gap, 1e-3 * half_gap, seed=n)
    k = n / 2.0
    bref = 0.0   # the middle of the gap: the VJP at this b (any b defines one)
    xmin = np.min(np.abs((r.astype(np.float64) - bref) / t))
    assert 0.9 * half_gap / t < xmin < 1.1 * half_gap / t
    rd, gd = torch.from_numpy(r).cuda()[None, :], torch.from_numpy(g).cuda()[None, :]
    b = torch.tensor([bref], dtype=torch.float64, device="cuda")
    grad = L.backward(rd, b, gd, t).cpu().numpy()[0]
    gref, _, _ = orc.vjp(r, g, bref, t)
    assert np.all(np.isfinite(grad))
    assert rel_l2(grad, gref) <= TOL_VJP
    # and the forward on the same scores.  Every score lies >= 60 t from b, so G
    # is flat to fp64 across the gap (the oracle's bisection cannot place b
    # there; the method's closed form can): check the mass at the GPU's b, that b
    # lies in the gap, and p there
    p, bg = L.forward(rd, k, t)
    torch.cuda.synchronize()
    bg = float(bg[0])
    assert abs(orc.G(r, bg, t)[0] - k) <= TOL_SUM
    assert r[r < bg].max() < bg < r[r > bg].min()
    p = p.cpu().numpy()[0]
    assert np.max(np.abs(p.astype(np.float64) - orc.p(r, bg, t))) <= TOL_P
    assert abs(p.astype(np.float64).sum() - k) <= TOL_SUM


@pytest.mark.parametrize("rows", [1, 7281])
def test_noalloc_vjp_far_from_every_score(L, orc, rows):
    # the allocation-free backward on a row whose f all underflow (one block per
    # row at 7281 rows, the most its scratch holds; several blocks at one row)
    fn = L.lib.lapsum_backward_noalloc
    fn.argtypes = [C.c_void_p] * 3 + [C.c_int64, C.c_int64, C.c_double, C.c_void_p, C.c_void_p]
    fn.restype = C.c_int
    n, t = 512, 1e-30
    r1, g1 = two_clusters(n, 1.2e-28, 1.2e-31, seed=rows)
    r = np.tile(r1, (rows, 1))
    g = np.tile(g1, (rows, 1))
    bref = 0.0   # the middle of the gap: every |x| ~ 120
    rd, gd = torch.from_numpy(r).cuda(), torch.from_numpy(g).cuda()
    b = torch.full((rows,), bref, dtype=torch.float64, device="cuda")
    out = torch.empty_like(rd)
    assert fn(rd.data_ptr(), b.data_ptr(), gd.data_ptr(), rows, n, t, out.data_ptr(),
              torch.cuda.current_stream().cuda_stream) == 0
    ref = L.backward(rd, b, gd, t)
    torch.cuda.synchronize()
    gref, _, _ = orc.vjp(r1, g1, bref, t)
    o = out.cpu().numpy()
    assert rel_l2(o[0], gref) <= TOL_VJP and rel_l2(o[-1], gref) <= TOL_VJP
    assert rel_l2(o, ref.cpu().numpy()) <= TOL_VJP


# ------------------------------------------------ select candidate overflow --
@pytest.mark.parametrize("band_cap", [0, 1 << 20])
def test_select_walks_every_key_when_candidates_overflow(L, orc, band_cap):
    # 70% of the scores tie at 1.2345 (15% at 3.0, 15% at -0.5), t = 1e-6: the
    # noised samples of the big level all share one 16-bit key prefix (~11.5k of
    # 16384 > the 8192-key candidate buffer), and both bracket ranks fall in it
    n = 1 << 20
    rng = np.random.default_rng(31)
    r = np.full(n, 1.2345, np.float32)
    idx = rng.permutation(n)
    r[idx[: int(0.15 * n)]] = 3.0
    r[idx[int(0.15 * n): int(0.30 * n)]] = -0.5
    g = rng.standard_normal(n).astype(np.float32)
    k, t = n / 2.0 + 0.25, 1e-6
    rd = torch.from_numpy(r).cuda()[None, :]
    p, b = L.forward(rd, k, t, opts=L.options(band_cap=band_cap))
    st = L.get_stats()
    assert st["flags"] & L.FLAG_SELECT_ALL_KEYS
    plan = L.bracket_plan(n, k, L.options(band_cap=band_cap))
    br = orc.bracket(r, k, t, 0, plan["s"], 1e-6)
    assert (st["jR"], st["jL"]) == (br["jR"], br["jL"])
    assert np.float32(st["a_L"]) == br["a_L"] and np.float32(st["a_R"]) == br["a_R"]
    cert = orc.certify(r, k, t, br["a_L"], br["a_R"], band_cap=plan["band_cap"])
    assert (st["c_L"], st["c_band"], st["c_R"]) == (cert["c_L"], cert["c_band"], cert["c_R"])
    assert st["verdict"] == cert["verdict"] and st["fallback"] == 1 - cert["verdict"]
    bref = orc.solve(r, k, t, method=1)
    assert abs(float(b[0]) - bref) <= TOL_B * t
    pn = p.cpu().numpy()[0]
    assert np.max(np.abs(pn.astype(np.float64) - orc.p(r, bref, t))) <= TOL_P
    gd = torch.from_numpy(g).cuda()[None, :]
    grad = L.backward(rd, b, gd, t).cpu().numpy()[0]
    gref, _, _ = orc.vjp(r, g, bref, t)
    assert rel_l2(grad, gref) <= TOL_VJP


# ---------------------------------------------- tail sums vs the definition --
def tail_tolerance(r, a, t, S, S_far, n):
    """Bound on |S_gpu - S| for a tail sum of the streaming pass.  Terms with
    z = |r - a|/t <= 16 are fp64 (relative error ~1e-15, summed in fp64); terms
    with 16 < z <= 40 are fp32, 2^{-z2} with z2 = z log2(e) formed in fp32 from
    three roundings (r - a, the scale log2(e)/t, their product: |dz2| <= 3 z2 2^-24),
    so the term's relative error ln2 |dz2| is at most 3 z 2^-24 (z <= 40), plus
    ex2.approx (< 2^-21); each thread sums at most m of them in fp32 before one
    fp64 add (<= m 2^-24 relative); terms beyond z = 40 (< 4.3e-18 each) are
    dropped.  Scores within 0.01 t of z = 16 may fall in either tier."""
    m = math.ceil(n / (3 * 148 * 256)) + 8
    per_far = 3 * 40 * 2.0**-24 + 2.0**-21 + m * 2.0**-24
    z = np.abs(r.astype(np.float64) - float(a)) / t
    edge = np.count_nonzero(np.abs(z - 16.0) < 0.01) * math.exp(-15.99)
    return 1e-12 * S + per_far * (S_far + edge) + np.count_nonzero(z > 39.9) * 4.3e-18


@pytest.mark.parametrize("certify", [0, 1])
@pytest.mark.parametrize("n,dist,k,t", [(1 << 20, "normal", 1000.0, 0.05), (1_500_001, "laplace", 150.0, 0.01),
                                        (1 << 20, "levels256_desc", 20000.0, 0.1),
                                        (1 << 21, "pixel_mix", 420.0, 0.01)])
def test_tail_sums_and_certification_values(L, orc, n, dist, k, t, certify):
    r, _ = W.small_case(dist, 1, n, seed=23)
    rd = torch.from_numpy(r).cuda()
    L.forward(rd, k, t, opts=L.options(certify=certify))
    st = L.get_stats()
    assert st["path"] == 2 and st["verdict"] == 1
    aL, aR = np.float32(st["a_L"]), np.float32(st["a_R"])
    ts = orc.tail_sums(r[0], aL, aR, t)
    assert abs(st["S_L"] - ts["S_L"]) <= tail_tolerance(r[0], aL, t, ts["S_L"], ts["S_L_far"], n)
    assert abs(st["S_R"] - ts["S_R"]) <= tail_tolerance(r[0], aR, t, ts["S_R"], ts["S_R_far"], n)
    # G at each end, from the definition: the same tiers, now on both sides of the end
    cert = orc.certify(r[0], k, t, aL, aR, band_cap=10**12)
    for a, G_gpu, G_ref in ((aL, st["G_aL"], cert["G_aL"]), (aR, st["G_aR"], cert["G_aR"])):
        if not np.isfinite(a):
            continue
        both = orc.tail_sums(r[0], a, a, t)      # sums below a and at or above a
        tol = 0.5 * (tail_tolerance(r[0], a, t, both["S_L"], both["S_L_far"], n) +
                     tail_tolerance(r[0], a, t, both["S_R"], both["S_R_far"], n)) + 1e-12 * G_ref
        assert abs(G_gpu - G_ref) <= tol, (a, G_gpu, G_ref, tol)


# ------------------------------------------------------- every row, rows1024 --
@pytest.mark.slow
def test_rows1024_every_row(L, orc):
    w = W.WORKLOADS["rows1024"]
    r, g = W.scores(w), W.upstream_grad(w)
    rd, gd = torch.from_numpy(r).cuda(), torch.from_numpy(g).cuda()
    p, b = L.forward(rd, w.k, w.t)
    grad = L.backward(rd, b, gd, w.t).cpu().numpy()
    p, b = p.cpu().numpy(), b.cpu().numpy()
    bref = orc.solve_rows(r, w.k, w.t, method=1)
    assert np.max(np.abs(b - bref)) <= TOL_B * w.t
    worst_p = worst_v = 0.0
    for i in range(w.rows):
        worst_p = max(worst_p, np.max(np.abs(p[i].astype(np.float64) - orc.p(r[i], bref[i], w.t))))
        gref, _, _ = orc.vjp(r[i], g[i], bref[i], w.t)
        worst_v = max(worst_v, rel_l2(grad[i], gref))
    assert worst_p <= TOL_P and worst_v <= TOL_VJP
    assert np.max(np.abs(p.astype(np.float64).sum(axis=1) - w.k)) <= TOL_SUM


# ------------------------------------------------- the plain forward call --
@pytest.mark.parametrize("n", [4096, 100_000, 1 << 20])
def test_plain_forward_entry_point(L, orc, n):
    r, _ = W.small_case("normal", 1, n, seed=29)
    k, t = n / 128.0, 0.05
    rd = torch.from_numpy(r).cuda()
    p = torch.empty_like(rd)
    b = torch.empty(1, dtype=torch.float64, device="cuda")
    rc = L.lib.lapsum_forward(rd.data_ptr(), 1, n, k, t, p.data_ptr(), b.data_ptr(),
                              torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    torch.cuda.synchronize()
    bref = orc.solve(r[0], k, t, method=1)
    assert abs(float(b[0]) - bref) <= TOL_B * t
    assert np.max(np.abs(p.cpu().numpy()[0].astype(np.float64) - orc.p(r[0], bref, t))) <= TOL_P


# ------------------------------------------ a bounded wait made to give up --
def test_grid_barrier_timeout_is_reported_and_the_next_call_is_clean(L, orc):
    # spin_cap = -1: every grid-barrier wait of the device-wide sort gives up at
    # its first poll.  The CTAs that give up return at once; the others leave at
    # their next barrier.  The call reports the timeout; the sort's global
    # histograms (left with partial counts) are cleared by the next sort.
    n = 1 << 17
    r, g = W.small_case("normal", 1, n, seed=37)
    k, t = 300.0, 0.05
    rd = torch.from_numpy(r).cuda()
    full = L.options(force_path=L.PATH_FULLSORT)
    L.forward(rd, k, t, opts=L.options(force_path=L.PATH_FULLSORT, spin_cap=-1))
    st = L.get_stats(check=False)
    assert st["rc"] == L.ERR_DEVICE_TIMEOUT and (st["status"] & 2)
    for _ in range(2):
        p, b = L.forward(rd, k, t, opts=full)
        st = L.get_stats(check=False)
        assert st["rc"] == 0 and st["status"] == 0
        bref = orc.solve(r[0], k, t, method=1)
        assert abs(float(b[0]) - bref) <= TOL_B * t
        assert np.max(np.abs(p.cpu().numpy()[0].astype(np.float64) - orc.p(r[0], bref, t))) <= TOL_P


# ------------------------------------ a new workspace on a non-blocking stream --
def test_new_workspace_on_a_nonblocking_stream_matches_the_default_stream(L):
    # The workspace of a (device, stream) pair is allocated and zeroed on the
    # first call on that stream; the zeros (the sampler's select histograms, the
    # device sort's digit histograms, the tickets) must be ordered before the
    # call's kernels on a stream that does not wait for the legacy default stream.
    cases = [("normal", 4096, 64.0, 0.05, None),                                   # one-CTA row solve
             ("normal", 1 << 20, 1000.0, 0.05, None),                              # bracketing + streaming VJP
             ("laplace", 1 << 20, 3000.0, 0.02, L.options(force_path=L.PATH_FULLSORT))]   # device sort
    data = []
    for seed, (dist, n, k, t, opts) in enumerate(cases):
        r_np, g_np = W.small_case(dist, 1, n, seed=40 + seed)
        r, g = torch.from_numpy(r_np).cuda(), torch.from_numpy(g_np).cuda()
        p, b = L.forward(r, k, t, opts=opts)
        grad = L.backward(r, b, g, t)
        data.append((r, g, k, t, opts, p.clone(), b.clone(), grad.clone()))
    torch.cuda.synchronize()
    L.release()   # every workspace of this device: the calls below grow new ones
    s = torch.cuda.Stream()   # PyTorch's pool streams are non-blocking
    s.wait_stream(torch.cuda.current_stream())
    with torch.cuda.stream(s):
        outs = []
        for r, g, k, t, opts, _, _, _ in data:
            p, b = L.forward(r, k, t, opts=opts)
            outs.append((p, b, L.backward(r, b, g, t)))
    s.synchronize()
    for (_, _, _, _, _, p0, b0, g0), (p, b, grad) in zip(data, outs):
        assert torch.equal(b, b0) and torch.equal(p, p0) and torch.equal(grad, g0)
    torch.cuda.synchronize()


# ------------------------------------------------- buffers of the wrong size --
def test_binding_refuses_buffers_of_the_wrong_size(L):
    # the library writes and reads exactly rows x n values (rows thresholds): a
    # buffer of another size is refused by the binding, before anything runs
    rows, n = 2, 4096
    r = torch.randn(rows, n, device="cuda")
    g = torch.randn(rows, n, device="cuda")
    short = torch.empty(rows * n - 1, device="cuda")
    n0 = L.launch_count()
    with pytest.raises(ValueError):
        L.forward(r, 64.0, 0.1, p_out=short)
    with pytest.raises(ValueError):
        L.forward(r, 64.0, 0.1, b_out=torch.empty(rows - 1, dtype=torch.float64, device="cuda"))
    assert L.launch_count() == n0
    p, b = L.forward(r, 64.0, 0.1)
    n1 = L.launch_count()
    with pytest.raises(ValueError):
        L.backward(r, b, short, 0.1)
    with pytest.raises(ValueError):
        L.backward(r, b, g, 0.1, grad_out=short)
    with pytest.raises(ValueError):
        L.backward(r, b[:1], g, 0.1)
    assert L.launch_count() == n1
    grad = L.backward(r, b, g, 0.1)
    torch.cuda.synchronize()
    assert torch.isfinite(grad).all() and torch.isfinite(p).all()
