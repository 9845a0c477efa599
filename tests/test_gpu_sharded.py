"""The split-row kernels (lapsum_shard_*) on one GPU: R ranks emulated in one
process, each on its own stream (so each has its own workspace), the
collectives replaced by device tensor ops between the phases.  No kernel of one
rank waits on another's.  Checked against the one-GPU solve of the whole row
(same bracket, counts and verdict, bit for bit) and against the fp64 oracle (b,
p, VJP at the parity tolerances) -- "Fast LapSum: Exact Differentiable Top-k
at Million Scale", technical summary sections 2.1-2.2 and 4.1."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TOL_B, TOL_P, TOL_SUM, TOL_VJP = 1e-4, 1e-5, 1e-3, 1e-4


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_budget_soft_b200 as lib
    return lib


def emulate(L, r, g, k, t, R, opts=None):
    from exact_budget_soft_b200 import sharded as S
    n = r.size
    streams = [torch.cuda.Stream() for _ in range(R)]
    ops = [S.LibraryOps(stream=s) for s in streams]
    bounds = [S.slice_bounds(n, R, q) for q in range(R)]
    rd = torch.from_numpy(r).cuda()
    gd = torch.from_numpy(g).cuda()
    sl = [rd[o:o + m] for o, m in bounds]
    gl = [gd[o:o + m] for o, m in bounds]
    torch.cuda.synchronize()
    xwords, cap = ops[0].plan(n, k, opts)
    xb = [torch.empty(xwords, dtype=torch.int32, device="cuda") for _ in range(R)]
    for q in range(R):
        ops[q].sample(sl[q], bounds[q][0], n, k, t, opts, xb[q])
    torch.cuda.synchronize()
    xsum = torch.stack(xb).sum(0, dtype=torch.int64).to(torch.int32)   # the all-reduce
    parts = [torch.empty(S.SHARD_PART, dtype=torch.float64, device="cuda") for _ in range(R)]
    bands = [torch.empty(max(cap, 1), dtype=torch.float32, device="cuda") for _ in range(R)]
    for q in range(R):
        ops[q].stream_pass(sl[q], bounds[q][0], n, k, t, opts, xsum, parts[q], bands[q])
    torch.cuda.synchronize()
    P = torch.stack(parts)                                              # the all-gather, rank order
    counts = [int(c) for c in P[:, 2].tolist()]
    band_all = torch.cat([bands[q][: min(counts[q], cap)] for q in range(R)] + [bands[0][:1]])
    bs = [torch.empty(1, dtype=torch.float64, device="cuda") for _ in range(R)]
    vs = [torch.zeros(1, dtype=torch.int32, device="cuda") for _ in range(R)]
    for q in range(R):
        ops[q].solve(P, band_all, sum(counts), n, k, t, opts, bs[q], vs[q])
    torch.cuda.synchronize()
    stats = L.get_stats(stream=streams[0], check=False)
    verdict = int(vs[0].item())
    if verdict == 0:   # the full-sort fallback over the gathered row
        for q in range(R):
            with torch.cuda.stream(streams[q]):
                ops[q].full_solve(rd, k, t, bs[q])
        torch.cuda.synchronize()
    ps = [torch.empty_like(sl[q]) for q in range(R)]
    for q in range(R):
        ops[q].p(sl[q], t, bs[q], ps[q])
    torch.cuda.synchronize()
    vp = [torch.empty(3, dtype=torch.float64, device="cuda") for _ in range(R)]
    for q in range(R):
        ops[q].vjp_partial(sl[q], bs[q], gl[q], t, 0.0, vp[q])
    torch.cuda.synchronize()
    V = torch.stack(vp)
    shifted = float(V[:, 0].sum()) < S.TINY
    if shifted:
        shift = float(V[:, 2].min())
        for q in range(R):
            ops[q].vjp_partial(sl[q], bs[q], gl[q], t, shift, vp[q])
        torch.cuda.synchronize()
        V = torch.stack(vp)
    grads = [torch.empty_like(sl[q]) for q in range(R)]
    for q in range(R):
        ops[q].vjp_apply(sl[q], bs[q], gl[q], t, V, grads[q])
    torch.cuda.synchronize()
    return {"b": [float(x[0]) for x in bs], "verdict": verdict, "stats": stats, "shifted": shifted,
            "p": torch.cat(ps).cpu().numpy(), "grad": torch.cat(grads).cpu().numpy(), "band": sum(counts)}


@pytest.mark.parametrize("dist,n,k,t,R", [("normal", 1 << 20, 1000.0, 0.05, 2),
                                         ("normal", (1 << 20) + 7, 5000.0, 0.05, 3),
                                         ("laplace", 1_500_001, 150.0, 0.01, 4),
                                         ("levels256_desc", 1 << 21, 20000.0, 0.1, 3)])
def test_sharded_row_equals_the_one_gpu_row(L, orc, dist, n, k, t, R):
    r, g = W.small_case(dist, 1, n, seed=51)
    r, g = r[0], g[0]
    out = emulate(L, r, g, k, t, R)
    assert len(set(out["b"])) == 1                     # the same bits on every rank
    # the one-GPU fused-certification solve of the whole row: same bracket and counts
    rd = torch.from_numpy(r).cuda()[None, :]
    _, b1 = L.forward(rd, k, t, opts=L.options(certify=L.CERTIFY_FUSED))
    one = L.get_stats()
    st = out["stats"]
    for key in ("jR", "jL", "a_L", "a_R", "c_L", "c_band", "c_R", "verdict"):
        assert st[key] == one[key], key
    assert out["verdict"] == 1 and out["band"] == one["c_band"]
    b = out["b"][0]
    bref = orc.solve(r, k, t, method=1)
    assert abs(b - bref) <= TOL_B * t and abs(float(b1[0]) - bref) <= TOL_B * t
    assert np.max(np.abs(out["p"].astype(np.float64) - orc.p(r, bref, t))) <= TOL_P
    if dist != "levels256_desc":   # tied levels: the rounded-p sum has its own bound (X6)
        assert abs(out["p"].astype(np.float64).sum() - k) <= TOL_SUM
    gref, _, _ = orc.vjp(r, g, bref, t)
    assert np.linalg.norm(out["grad"] - gref) <= TOL_VJP * np.linalg.norm(gref)


def test_sharded_row_fallback(L, orc):
    r, g = W.small_case("normal", 1, 1 << 20, seed=53)
    r, g = r[0], g[0]
    k, t = 3000.0, 0.05
    out = emulate(L, r, g, k, t, 2, opts=L.options(band_cap=64))
    assert out["verdict"] == 0
    bref = orc.solve(r, k, t, method=1)
    assert all(abs(b - bref) <= TOL_B * t for b in out["b"])
    assert np.max(np.abs(out["p"].astype(np.float64) - orc.p(r, bref, t))) <= TOL_P
    gref, _, _ = orc.vjp(r, g, bref, t)
    assert np.linalg.norm(out["grad"] - gref) <= TOL_VJP * np.linalg.norm(gref)


def test_sharded_vjp_common_shift(L, orc):
    # two clusters ~120 t from the middle of the gap: every density underflows in
    # fp32, the second round shifts every slice by the smallest |x| of the row
    rng = np.random.default_rng(57)
    n = 1 << 20
    r = (np.where(np.arange(n) < n // 2, 1.2e-28, -1.2e-28) * (1 + 1e-3 * rng.uniform(-1, 1, n))).astype(np.float32)
    rng.shuffle(r)
    g = rng.standard_normal(n).astype(np.float32)
    k, t = n / 2.0, 1e-30
    out = emulate(L, r, g, k, t, 3)
    assert out["shifted"]
    b = out["b"][0]
    assert abs(orc.G(r, b, t)[0] - k) <= TOL_SUM and r[r < b].max() < b < r[r > b].min()
    gref, _, _ = orc.vjp(r, g, b, t)
    assert np.linalg.norm(out["grad"] - gref) <= TOL_VJP * np.linalg.norm(gref)
