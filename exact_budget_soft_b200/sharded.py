"""One row split across GPUs: the exact-budget soft top-k of a row too long for
one GPU ("Fast LapSum: Exact Differentiable Top-k at Million Scale", technical
summary section 4.1: rows of 1e8 scores and beyond).

One process per GPU (torch.distributed, NCCL); rank q holds the contiguous
slice [offset_q, offset_q + n_q) of a row of n_total scores.  Every step of the
bracketing path runs in the library's kernels on the slices (``lapsum_shard_*``
of include/lapsum.h); this module only moves the small exchange buffers between
the steps:

    sample    all-reduce (sum) of the sample buffer: every rank gets the one-GPU
              sample of the whole row, hence the one-GPU bracket
    stream    all-gather of the per-slice records (counts, tail sums, band-term
              sums, band key range) and of the band scores (gather-v, rank order)
    solve     replicated on every rank from the same data: the same b and verdict
    fallback  (verdict 0) all-gather of the whole row, full sort on every rank
    VJP       all-gather of {sum e, sum g e, min |x|}; a second round with a
              common shift when every density underflows

    p_local, b = sharded_forward(scores_local, offset, n_total, k, t)
    grad_local = sharded_backward(scores_local, b, g_local, t)

``ops`` (default: the library) is the set of slice steps; a test can pass a
stand-in with the same contract to exercise this exchange logic without GPUs.
"""
from __future__ import annotations

import ctypes as C

import torch
import torch.distributed as dist

SHARD_PART = 10
VJP_PART = 3
TINY = 2.0 ** -96   # below this, the plain sum of e^{-|x|} may have lost its precision


class LibraryOps:
    """The slice steps, run by the CUDA library on this rank's GPU."""

    def __init__(self, stream=None):
        import exact_budget_soft_b200 as L
        self.L = L
        self.stream = stream

    def _st(self):
        s = self.stream or torch.cuda.current_stream()
        return s.cuda_stream

    def _check(self, rc, where):
        if rc != 0:
            raise self.L.LapSumError(rc, where)

    def plan(self, n_total, k, opts):
        xw, cap = C.c_int64(), C.c_int64()
        self._check(self.L.lib.lapsum_shard_plan(int(n_total), float(k), C.byref(opts) if opts else None,
                                                 C.byref(xw), C.byref(cap)), "lapsum_shard_plan")
        return xw.value, cap.value

    def sample(self, r, offset, n_total, k, t, opts, xbuf):
        self._check(self.L.lib.lapsum_shard_sample(r.data_ptr(), r.numel(), int(offset), int(n_total), float(k),
                                                   float(t), C.byref(opts) if opts else None, xbuf.data_ptr(),
                                                   self._st()), "lapsum_shard_sample")

    def stream_pass(self, r, offset, n_total, k, t, opts, xbuf, part, band):
        self._check(self.L.lib.lapsum_shard_stream(r.data_ptr(), r.numel(), int(offset), int(n_total), float(k),
                                                   float(t), C.byref(opts) if opts else None, xbuf.data_ptr(),
                                                   part.data_ptr(), band.data_ptr(), self._st()),
                    "lapsum_shard_stream")

    def solve(self, parts, band_all, band_total, n_total, k, t, opts, b, verdict):
        self._check(self.L.lib.lapsum_shard_solve(parts.data_ptr(), parts.shape[0], band_all.data_ptr(),
                                                  int(band_total), int(n_total), float(k), float(t),
                                                  C.byref(opts) if opts else None, b.data_ptr(),
                                                  verdict.data_ptr(), self._st()), "lapsum_shard_solve")

    def full_solve(self, row, k, t, b):
        opts = self.L.options(force_path=self.L.PATH_FULLSORT)
        p = torch.empty_like(row)
        self.L.forward(row[None, :], k, t, p_out=p[None, :], b_out=b, opts=opts)

    def p(self, r, t, b, p_out):
        self._check(self.L.lib.lapsum_shard_p(r.data_ptr(), r.numel(), float(t), b.data_ptr(), p_out.data_ptr(),
                                              self._st()), "lapsum_shard_p")

    def vjp_partial(self, r, b, g, t, shift, part):
        self._check(self.L.lib.lapsum_shard_vjp_partial(r.data_ptr(), b.data_ptr(), g.data_ptr(), r.numel(),
                                                        float(t), float(shift), part.data_ptr(), self._st()),
                    "lapsum_shard_vjp_partial")

    def vjp_apply(self, r, b, g, t, parts, grad):
        self._check(self.L.lib.lapsum_shard_vjp_apply(r.data_ptr(), b.data_ptr(), g.data_ptr(), r.numel(),
                                                      float(t), parts.data_ptr(), parts.shape[0],
                                                      grad.data_ptr(), self._st()), "lapsum_shard_vjp_apply")


def _gather(x: torch.Tensor, group) -> torch.Tensor:
    """All-gather of equal-size tensors, stacked in rank order."""
    world = dist.get_world_size(group)
    out = [torch.empty_like(x) for _ in range(world)]
    dist.all_gather(out, x, group=group)
    return torch.stack(out)


def _gather_v(x: torch.Tensor, counts: list[int], group) -> torch.Tensor:
    """All-gather of rank-dependent lengths (counts[q] from rank q), concatenated in rank order."""
    m = max(max(counts), 1)
    pad = torch.zeros(m, dtype=x.dtype, device=x.device)
    pad[: counts[dist.get_rank(group)]] = x[: counts[dist.get_rank(group)]]
    parts = _gather(pad, group)
    return torch.cat([parts[q, : counts[q]] for q in range(len(counts))])


def slice_bounds(n_total: int, world: int, rank: int) -> tuple[int, int]:
    """The contiguous slice [offset, offset + n) of rank `rank` when n_total scores
    are split as evenly as possible over `world` ranks."""
    base, extra = divmod(n_total, world)
    offset = rank * base + min(rank, extra)
    return offset, base + (1 if rank < extra else 0)


def sharded_forward(scores_local: torch.Tensor, offset: int, n_total: int, k: float, t: float,
                    group=None, opts=None, ops=None) -> tuple[torch.Tensor, torch.Tensor, dict]:
    """p of this rank's slice, b (fp64 [1], the same on every rank) and a small
    record of the exchange (band size, verdict, whether the fallback ran)."""
    ops = ops or LibraryOps()
    dev = scores_local.device
    xwords, band_cap = ops.plan(n_total, k, opts)
    xbuf = torch.empty(xwords, dtype=torch.int32, device=dev)
    ops.sample(scores_local, offset, n_total, k, t, opts, xbuf)
    dist.all_reduce(xbuf, op=dist.ReduceOp.SUM, group=group)   # every draw filled by exactly one rank
    part = torch.empty(SHARD_PART, dtype=torch.float64, device=dev)
    band = torch.empty(max(band_cap, 1), dtype=torch.float32, device=dev)
    ops.stream_pass(scores_local, offset, n_total, k, t, opts, xbuf, part, band)
    parts = _gather(part, group)
    counts = [int(c) for c in parts[:, 2].tolist()]          # the ranks' band sizes (one host read)
    kept = [min(c, band_cap) for c in counts]
    band_all = _gather_v(band, kept, group) if sum(kept) else band[:1]
    b = torch.empty(1, dtype=torch.float64, device=dev)
    verdict = torch.zeros(1, dtype=torch.int32, device=dev)
    ops.solve(parts, band_all, sum(counts), n_total, k, t, opts, b, verdict)
    certified = int(verdict.item()) == 1
    if not certified:   # the bracket failed certification: full sort of the gathered row
        sizes = _gather(torch.tensor([scores_local.numel()], dtype=torch.int64, device=dev), group)
        row = _gather_v(scores_local, [int(v) for v in sizes[:, 0].tolist()], group)
        ops.full_solve(row, k, t, b)
    p_local = torch.empty_like(scores_local)
    ops.p(scores_local, t, b, p_local)
    return p_local, b, {"band": sum(counts), "verdict": int(certified), "fallback": int(not certified)}


def sharded_backward(scores_local: torch.Tensor, b: torch.Tensor, g_local: torch.Tensor, t: float,
                     group=None, ops=None) -> torch.Tensor:
    """grad of this rank's slice: (f/t)(g - <g,f>/sum f) with both sums over the whole row."""
    ops = ops or LibraryOps()
    dev = scores_local.device
    part = torch.empty(VJP_PART, dtype=torch.float64, device=dev)
    ops.vjp_partial(scores_local, b, g_local, t, 0.0, part)
    parts = _gather(part, group)
    if float(parts[:, 0].sum()) < TINY:   # every density tiny: one common shift, gathered again
        shift = float(parts[:, 2].min())
        ops.vjp_partial(scores_local, b, g_local, t, shift, part)
        parts = _gather(part, group)
    grad = torch.empty_like(scores_local)
    ops.vjp_apply(scores_local, b, g_local, t, parts, grad)
    return grad
