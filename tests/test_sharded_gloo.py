"""The split-row exchange (exact_budget_soft_b200.sharded) on CPU: 2 and 3 gloo
ranks, each holding one slice of a row, run the sharded forward and VJP with a
stand-in for the slice kernels written from the oracle and numpy (the same
contract as the library's lapsum_shard_* calls).  What this checks is the
host-side logic around the kernels -- the sample all-reduce, the record and
band gathers in rank order, the replicated solve, the certification fallback
over the gathered row, the second VJP round with a common shift -- against the
oracle on the whole row: the bracket and counts exactly, b, p and the VJP to
the parity tolerances ("Fast LapSum: Exact Differentiable Top-k at Million
Scale", technical summary sections 2.1-2.2 and 4.1).  The kernels themselves
are checked on the GPU (test_gpu_sharded.py)."""
import math
import os
import socket

import numpy as np
import pytest
import torch
import torch.distributed as dist
import torch.multiprocessing as mp

TOL_B, TOL_P, TOL_VJP = 1e-4, 1e-5, 1e-4
HIST_WORDS = 65536 + 256
SAMPLE_TAG = 0x4C41505355534D50


def _free_port():
    with socket.socket() as s:
        s.bind(("127.0.0.1", 0))
        return s.getsockname()[1]


def _desc_key(f32):
    u = np.asarray(f32, np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, u, u ^ 0x7FFFFFFF).astype(np.uint32)


def _key_value(k):
    k = np.asarray(k, np.uint32).astype(np.uint64)
    return np.where(k & 0x80000000, k, k ^ 0x7FFFFFFF).astype(np.uint32).view(np.float32)


def _round_down_f32(y):
    f = y.astype(np.float32)
    return np.where(f.astype(np.float64) > y, np.nextafter(f, np.float32(-np.inf)), f)


class OracleOps:
    """Stand-in for the slice kernels (CPU, fp64): one rank's view of the row."""

    def __init__(self, orc, r_full, plan, rank):
        self.orc, self.r_full, self.plan_fn, self.rank = orc, r_full, plan, rank

    def plan(self, n_total, k, opts):
        p = self.plan_fn(n_total, k, opts)
        self.s, self.jR, self.jL, self.cap = p["s"], p["jR"], p["jL"], p["band_cap"]
        self.seed = opts.seed if opts is not None else 0
        return self.s + HIST_WORDS, self.cap

    def sample(self, r, offset, n_total, k, t, opts, xbuf):
        y, idx = self.orc.sample(self.r_full, t, self.seed, self.s)
        keys = _desc_key(_round_down_f32(y))
        mine = (idx >= offset) & (idx < offset + r.numel())
        kk = np.where(mine, keys, 0).astype(np.uint32)
        h16 = np.bincount(keys[mine] >> 16, minlength=65536)
        h8 = np.bincount(keys[mine] >> 24, minlength=256)
        out = np.concatenate([kk.view(np.int32), h16.astype(np.int32), h8.astype(np.int32)])
        xbuf.copy_(torch.from_numpy(out))

    def stream_pass(self, r, offset, n_total, k, t, opts, xbuf, part, band):
        keys = np.sort(xbuf[: self.s].numpy().view(np.uint32))         # ascending key = descending value
        h = xbuf[self.s:].numpy()
        assert np.array_equal(h[:65536], np.bincount(keys >> 16, minlength=65536))   # the summed histograms
        aR = np.nextafter(_key_value(keys[self.jR - 1]), np.float32(np.inf)) if self.jR >= 1 else np.float32(np.inf)
        aL = _key_value(keys[self.jL - 1]) if self.jL <= self.s else np.float32(-np.inf)
        self.aL, self.aR = np.float32(aL), np.float32(aR)
        x = r.numpy()
        cL, cb, cR = self.orc.counts(x, aL, aR)
        ts = self.orc.tail_sums(x, aL, aR, t)
        bsc = x[(x >= aL) & (x < aR)]
        hL = float(np.sum(np.exp(-(bsc.astype(np.float64) - float(aL)) / t))) if np.isfinite(aL) else 0.0
        lR = float(np.sum(np.exp(-(float(aR) - bsc.astype(np.float64)) / t))) if np.isfinite(aR) else 0.0
        kb = _desc_key(bsc)
        kmax = float(kb.max()) if kb.size else 0.0
        kinv = float((~kb).max()) if kb.size else 0.0
        part.copy_(torch.tensor([cL, cR, cb, ts["S_L"], ts["S_R"], hL, lR, kmax, kinv, 0.0], dtype=torch.float64))
        band[: min(cb, self.cap)] = torch.from_numpy(bsc[: self.cap])

    def solve(self, parts, band_all, band_total, n_total, k, t, opts, b, verdict):
        P = parts.numpy()
        cL, cR, cb = (int(v) for v in P[:, :3].sum(axis=0))
        SL, SR, hL, lR = (float(v) for v in P[:, 3:7].sum(axis=0))
        aL, aR = float(self.aL), float(self.aR)
        rho = 0.0 if not (np.isfinite(aL) and np.isfinite(aR)) else math.exp(-(aR - aL) / t)
        GaL = (cb + cR) - 0.5 * (rho * SR + hL) + 0.5 * SL
        GaR = cR - 0.5 * SR + 0.5 * (rho * SL + lR)
        ok = cb <= self.cap and cL + cb + cR == n_total and GaL >= k and GaR < k
        verdict.fill_(int(ok))
        if not ok:
            return
        band = band_all[:band_total].numpy().astype(np.float64)

        def G(bb):   # the row's mass at bb in [a_L, a_R], from the seeds and the band
            v = np.sum(np.where(band >= bb, 1 - 0.5 * np.exp(-(band - bb) / t), 0.5 * np.exp((band - bb) / t)))
            if np.isfinite(aR):
                v += cR - 0.5 * SR * math.exp(-(aR - bb) / t)
            if np.isfinite(aL):
                v += 0.5 * SL * math.exp((aL - bb) / t)
            return v

        lo = aL if np.isfinite(aL) else float(band.min(initial=aR)) - 50 * t
        hi = aR if np.isfinite(aR) else float(band.max(initial=aL)) + 50 * t
        for _ in range(200):
            mid = 0.5 * (lo + hi)
            if G(mid) > k:
                lo = mid
            else:
                hi = mid
        b.fill_(0.5 * (lo + hi))

    def full_solve(self, row, k, t, b):
        b.fill_(self.orc.solve(row.numpy(), k, t, method=1))

    def p(self, r, t, b, p_out):
        p_out.copy_(torch.from_numpy(self.orc.p(r.numpy(), float(b[0]), t).astype(np.float32)))

    def vjp_partial(self, r, b, g, t, shift, part):
        ax = np.abs((r.numpy().astype(np.float64) - float(b[0])) / t)
        e = np.exp(shift - ax)
        part.copy_(torch.tensor([e.sum(), (g.numpy() * e).sum(), ax.min()], dtype=torch.float64))

    def vjp_apply(self, r, b, g, t, parts, grad):
        P = parts.numpy()
        lam = P[:, 1].sum() / P[:, 0].sum()
        ax = np.abs((r.numpy().astype(np.float64) - float(b[0])) / t)
        grad.copy_(torch.from_numpy((0.5 * np.exp(-ax) / t * (g.numpy() - lam)).astype(np.float32)))


def _worker(rank, world, port, case, out):
    os.environ.update(MASTER_ADDR="127.0.0.1", MASTER_PORT=str(port), RANK=str(rank), WORLD_SIZE=str(world))
    import datetime
    dist.init_process_group("gloo", rank=rank, world_size=world, timeout=datetime.timedelta(seconds=120))
    try:
        import exact_budget_soft_b200 as L
        import oracle
        from exact_budget_soft_b200 import sharded as S
        r, g, k, t, opts = case()
        off, n = S.slice_bounds(r.size, world, rank)
        ops = OracleOps(oracle, r, L.bracket_plan, rank)
        rl, gl = torch.from_numpy(r[off:off + n].copy()), torch.from_numpy(g[off:off + n].copy())
        p, b, info = S.sharded_forward(rl, off, r.size, k, t, opts=opts, ops=ops)
        grad = S.sharded_backward(rl, b, gl, t, ops=ops)
        out.put((rank, off, float(b[0]), p.numpy(), grad.numpy(), info,
                 (float(ops.aL), float(ops.aR), ops.jR, ops.jL)))
        dist.barrier()
    finally:
        dist.destroy_process_group()


def _run(world, case):
    ctx = mp.get_context("spawn")
    q = ctx.Queue()
    port = _free_port()
    procs = [ctx.Process(target=_worker, args=(rk, world, port, case, q)) for rk in range(world)]
    for p in procs:
        p.start()
    res = sorted((q.get(timeout=300) for _ in range(world)), key=lambda x: x[0])
    for p in procs:
        p.join(timeout=120)
        assert p.exitcode == 0
    return res


def case_normal():
    import workloads as W
    r, g = W.small_case("normal", 1, 1 << 18, seed=41)
    return r[0], g[0], 300.0, 0.05, None


def case_fallback():
    import exact_budget_soft_b200 as L
    import workloads as W
    r, g = W.small_case("laplace", 1, 200_003, seed=43)
    return r[0], g[0], 2000.0, 0.05, L.options(band_cap=16)


def case_far():
    rng = np.random.default_rng(47)
    n = 60_000
    r = np.where(np.arange(n) < n // 2, 1.2e-28, -1.2e-28) * (1 + 1e-3 * rng.uniform(-1, 1, n))
    rng.shuffle(r)
    return r.astype(np.float32), rng.standard_normal(n).astype(np.float32), n / 2.0, 1e-30, None


def _check(orc, res, case, want_verdict, flat=False):
    r, g, k, t, opts = case()
    bs = [x[2] for x in res]
    assert all(v == bs[0] for v in bs)                      # one b on every rank
    if flat:   # every score ~100 t from b: G is flat to fp64 there, b is fixed by e^-100 terms
        bref = bs[0]
        assert abs(orc.G(r, bref, t)[0] - k) <= 1e-3 and r[r < bref].max() < bref < r[r > bref].min()
    else:
        bref = orc.solve(r, k, t, method=1)
        assert abs(bs[0] - bref) <= TOL_B * t
    p = np.concatenate([x[3] for x in res])
    grad = np.concatenate([x[4] for x in res])
    assert np.max(np.abs(p.astype(np.float64) - orc.p(r, bref, t))) <= TOL_P
    gref, _, _ = orc.vjp(r, g, bref, t)
    assert np.linalg.norm(grad - gref) <= TOL_VJP * np.linalg.norm(gref)
    assert all(x[5]["verdict"] == want_verdict for x in res)
    return r, k, t, opts, res[0][6]


@pytest.mark.parametrize("world", [2, 3, 4])
def test_sharded_row_matches_the_whole_row(orc, world):
    res = _run(world, case_normal)
    r, k, t, _, (aL, aR, jR, jL) = _check(orc, res, case_normal, 1)
    import exact_budget_soft_b200 as L
    plan = L.bracket_plan(r.size, k)
    br = orc.bracket(r, k, t, 0, plan["s"], 1e-6)             # the one-GPU bracket, bit for bit
    assert (jR, jL) == (br["jR"], br["jL"]) and np.float32(aL) == br["a_L"] and np.float32(aR) == br["a_R"]
    cert = orc.certify(r, k, t, br["a_L"], br["a_R"], band_cap=plan["band_cap"])
    assert res[0][5]["band"] == cert["c_band"]


@pytest.mark.parametrize("world", [2, 3])
def test_sharded_row_falls_back_over_the_gathered_row(orc, world):
    res = _run(world, case_fallback)
    _check(orc, res, case_fallback, 0)
    assert all(x[5]["fallback"] == 1 for x in res)


def test_sharded_vjp_takes_a_common_shift_when_every_density_underflows(orc):
    res = _run(2, case_far)
    _check(orc, res, case_far, 1, flat=True)
