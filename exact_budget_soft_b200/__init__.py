"""Fast LapSum exact-budget soft top-k on B200 (sm_100a).

Thin ctypes binding over the C ABI in ``include/lapsum.h`` (the library
``liblapsum.so`` built in-tree by ``build.py``).  This module only marshals
arguments: every step of the solver runs in the library's CUDA kernels, and
there is no CPU fallback -- importing fails loudly when the library is missing.

    p, b = forward(scores, k, t)          # scores: cuda float32 [rows, n] or [n]
    grad = backward(scores, b, g, t)
    p = soft_topk(scores, k, t)           # autograd-aware (analytic VJP)

Operator ("Fast LapSum: Exact Differentiable Top-k at Million Scale",
technical summary section 2.1): p_i = F((r_i - b)/t), F the Laplace CDF, b the
unique threshold with sum_i p_i = k; grad = (f/t)(g - <g,f>/sum f).
"""
from __future__ import annotations

import contextlib
import ctypes as C
import os

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
# LAPSUM_CHECKED=1 loads the checked build (bounds tests on computed indices,
# guard words around the workspace; slower, for debugging)
CHECKED = os.environ.get("LAPSUM_CHECKED") == "1"
LIB_PATH = os.path.join(_HERE, "liblapsum_checked.so" if CHECKED else "liblapsum.so")

PATH_AUTO, PATH_FULLSORT, PATH_BRACKET = 0, 1, 2
CERTIFY_PASS, CERTIFY_FUSED = 0, 1
# lapsum_stats.flags bits (rare routes a solve took)
FLAG_SELECT_ALL_KEYS = 1
# error codes (LAPSUM_ERR_* of the C header)
ERR_ARG, ERR_NONFINITE, ERR_ALLOC, ERR_DEVICE_TIMEOUT, ERR_CUDA, ERR_NO_ROOT = -1, -2, -3, -4, -5, -6
ERR_BOUNDS = -7
ERRORS = {0: "ok", -1: "invalid argument", -2: "non-finite score", -3: "workspace allocation failed",
          -4: "device wait timeout", -5: "CUDA runtime error", -6: "no crossing found",
          -7: "index or guard word out of bounds (checked build)"}


class LapSumError(RuntimeError):
    def __init__(self, code: int, where: str):
        super().__init__(f"{where}: {ERRORS.get(code, 'error')} ({code})")
        self.code = code


class Options(C.Structure):
    _fields_ = [("seed", C.c_uint64), ("sample_size", C.c_int64), ("delta", C.c_double),
                ("band_cap", C.c_int64), ("spin_cap", C.c_int32), ("force_path", C.c_int32),
                ("certify", C.c_int32), ("widen", C.c_int32), ("reserved", C.c_int32 * 2)]


class Stats(C.Structure):
    _fields_ = [("path", C.c_int32), ("verdict", C.c_int32), ("status", C.c_int32),
                ("fallback", C.c_int32), ("s", C.c_int64), ("jR", C.c_int64), ("jL", C.c_int64),
                ("c_L", C.c_int64), ("c_band", C.c_int64), ("c_R", C.c_int64),
                ("a_L", C.c_float), ("a_R", C.c_float), ("S_L", C.c_double), ("S_R", C.c_double),
                ("G_aL", C.c_double), ("G_aR", C.c_double), ("b", C.c_double),
                ("sum_p", C.c_double), ("j_star", C.c_int64), ("widened", C.c_int64),
                ("flags", C.c_int64), ("reserved", C.c_int64 * 2)]

    def as_dict(self) -> dict:
        return {f: getattr(self, f) for f, _ in self._fields_ if f != "reserved"}


EXPORTS = ["lapsum_forward", "lapsum_forward_ex", "lapsum_backward", "lapsum_get_stats", "lapsum_get_stats_rows",
           "lapsum_strerror", "lapsum_release", "lapsum_profile_enable", "lapsum_profile_read",
           "lapsum_bracket_plan", "lapsum_profile_filter", "lapsum_selftest_math", "lapsum_launch_count",
           "lapsum_backward_noalloc", "lapsum_shard_plan", "lapsum_shard_sample", "lapsum_shard_stream",
           "lapsum_shard_solve", "lapsum_shard_p", "lapsum_shard_vjp_partial", "lapsum_shard_vjp_apply",
           "lapsum_step_host"]
SHARD_PART = 10   # doubles in a slice's streaming-pass record (LAPSUM_SHARD_PART)


def _load() -> C.CDLL:
    if not os.path.exists(LIB_PATH):
        raise ImportError(f"{LIB_PATH} is missing: build it with `python -m exact_budget_soft_b200.build`"
                          " (--checked for the checked build)"
                          " (there is no CPU fallback)")
    lib = C.CDLL(LIB_PATH)
    vp, i64, dbl = C.c_void_p, C.c_int64, C.c_double
    lib.lapsum_forward.argtypes = [vp, i64, i64, dbl, dbl, vp, vp, vp]
    lib.lapsum_forward_ex.argtypes = [vp, i64, i64, dbl, dbl, vp, vp, C.POINTER(Options), vp]
    lib.lapsum_backward.argtypes = [vp, vp, vp, i64, i64, dbl, vp, vp]
    lib.lapsum_step_host.argtypes = [vp, vp, i64, i64, dbl, dbl, vp, vp, vp, C.POINTER(Options),
                                     vp, vp, vp, vp, vp, vp]
    lib.lapsum_get_stats.argtypes = [C.POINTER(Stats), vp]
    lib.lapsum_get_stats_rows.argtypes = [C.POINTER(Stats), i64, C.POINTER(i64), vp]
    lib.lapsum_strerror.restype = C.c_char_p
    lib.lapsum_strerror.argtypes = [C.c_int]
    lib.lapsum_profile_enable.argtypes = [C.c_int]
    lib.lapsum_profile_read.argtypes = [C.POINTER(C.c_char_p), C.POINTER(C.c_int64),
                                        C.POINTER(C.c_double), C.c_int]
    lib.lapsum_launch_count.restype = C.c_int64
    lib.lapsum_bracket_plan.argtypes = [i64, dbl, C.POINTER(Options), C.POINTER(i64), C.POINTER(i64),
                                        C.POINTER(i64), C.POINTER(i64)]
    lib.lapsum_bracket_plan.restype = C.c_int
    lib.lapsum_profile_filter.argtypes = [C.c_char_p]
    lib.lapsum_profile_filter.restype = C.c_int
    lib.lapsum_selftest_math.argtypes = [C.c_int, vp, vp, vp, i64, vp]
    lib.lapsum_selftest_math.restype = C.c_int
    op = C.POINTER(Options)
    lib.lapsum_shard_plan.argtypes = [i64, dbl, op, C.POINTER(i64), C.POINTER(i64)]
    lib.lapsum_shard_sample.argtypes = [vp, i64, i64, i64, dbl, dbl, op, vp, vp]
    lib.lapsum_shard_stream.argtypes = [vp, i64, i64, i64, dbl, dbl, op, vp, vp, vp, vp]
    lib.lapsum_shard_solve.argtypes = [vp, i64, vp, i64, i64, dbl, dbl, op, vp, vp, vp]
    lib.lapsum_shard_p.argtypes = [vp, i64, dbl, vp, vp, vp]
    lib.lapsum_shard_vjp_partial.argtypes = [vp, vp, vp, i64, dbl, dbl, vp, vp]
    lib.lapsum_shard_vjp_apply.argtypes = [vp, vp, vp, i64, dbl, vp, i64, vp, vp]
    for name in ("lapsum_shard_plan", "lapsum_shard_sample", "lapsum_shard_stream", "lapsum_shard_solve",
                 "lapsum_shard_p", "lapsum_shard_vjp_partial", "lapsum_shard_vjp_apply"):
        getattr(lib, name).restype = C.c_int
    for name in ("lapsum_forward", "lapsum_forward_ex", "lapsum_backward", "lapsum_step_host", "lapsum_get_stats",
                 "lapsum_release", "lapsum_profile_enable", "lapsum_profile_read"):
        getattr(lib, name).restype = C.c_int
    return lib


lib = _load()


def _stream(stream) -> int:
    if stream is None:
        stream = torch.cuda.current_stream()
    return stream.cuda_stream


def _on(dev: torch.device):
    """The library works on the current device: make it the tensors' device for
    the call (no switch, and no cost beyond one query, when it already is)."""
    if dev.index is None or dev.index == torch.cuda.current_device():
        return contextlib.nullcontext()
    return torch.cuda.device(dev)


def _check(rc: int, where: str):
    if rc != 0:
        raise LapSumError(rc, where)


def _as_rows(x: torch.Tensor) -> tuple[int, int]:
    if x.dim() == 1:
        return 1, x.shape[0]
    if x.dim() == 2:
        return x.shape[0], x.shape[1]
    raise ValueError("scores must be [n] or [rows, n]")


def _need(x: torch.Tensor, name: str, dtype=torch.float32, numel: int | None = None,
          device: torch.device | None = None):
    """A contiguous CUDA tensor of `dtype` (of `numel` values and on `device` when
    given): the library writes and reads exactly that many, so a short buffer is
    refused here rather than overrun on the device."""
    if not x.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor (there is no CPU path)")
    if x.dtype != dtype or not x.is_contiguous():
        raise ValueError(f"{name} must be contiguous {dtype}")
    if numel is not None and x.numel() != numel:
        raise ValueError(f"{name} must hold {numel} values, not {x.numel()}")
    if device is not None and x.device != device:
        raise ValueError(f"{name} is on {x.device}, the scores on {device}")


def options(seed: int = 0, sample_size: int = 0, delta: float = 0.0, band_cap: int = 0,
            spin_cap: int = 0, force_path: int = PATH_AUTO, certify: int = CERTIFY_PASS,
            widen: int = 0) -> Options:
    o = Options()
    o.seed, o.sample_size, o.delta, o.band_cap = seed, sample_size, delta, band_cap
    o.spin_cap, o.force_path, o.certify, o.widen = spin_cap, force_path, certify, widen
    return o


def forward(scores: torch.Tensor, k: float, t: float, p_out: torch.Tensor | None = None,
            b_out: torch.Tensor | None = None, opts: Options | None = None,
            stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """p (float32, like scores) and b (float64 [rows]) of lapsum_forward_ex."""
    _need(scores, "scores")
    rows, n = _as_rows(scores)
    dev = scores.device
    if p_out is None:
        p_out = torch.empty_like(scores)
    if b_out is None:
        b_out = torch.empty(rows, dtype=torch.float64, device=dev)
    _need(p_out, "p_out", numel=rows * n, device=dev)
    _need(b_out, "b_out", torch.float64, numel=rows, device=dev)
    with _on(dev):
        rc = lib.lapsum_forward_ex(scores.data_ptr(), rows, n, float(k), float(t), p_out.data_ptr(),
                                   b_out.data_ptr(), C.byref(opts) if opts is not None else None,
                                   _stream(stream))
        _check(rc, "lapsum_forward")
        if CHECKED:   # the checked build reports an out-of-bounds index through the device status
            st = Stats()
            if lib.lapsum_get_stats(C.byref(st), _stream(stream)) == ERR_BOUNDS:
                raise LapSumError(ERR_BOUNDS, "lapsum_forward")
    return p_out, b_out


def backward(scores: torch.Tensor, b: torch.Tensor, g: torch.Tensor, t: float,
             grad_out: torch.Tensor | None = None, stream=None) -> torch.Tensor:
    _need(scores, "scores")
    rows, n = _as_rows(scores)
    dev = scores.device
    _need(g, "g", numel=rows * n, device=dev)
    _need(b, "b", torch.float64, numel=rows, device=dev)
    if grad_out is None:
        grad_out = torch.empty_like(scores)
    _need(grad_out, "grad_out", numel=rows * n, device=dev)
    with _on(dev):
        rc = lib.lapsum_backward(scores.data_ptr(), b.data_ptr(), g.data_ptr(), rows, n, float(t),
                                 grad_out.data_ptr(), _stream(stream))
    _check(rc, "lapsum_backward")
    return grad_out


def get_stats(stream=None, check: bool = True) -> dict:
    """Diagnostics of the last forward on `stream` (synchronises it)."""
    st = Stats()
    rc = lib.lapsum_get_stats(C.byref(st), _stream(stream))
    if check:
        _check(rc, "lapsum_get_stats")
    d = st.as_dict()
    d["rc"] = rc
    return d


def get_stats_rows(max_rows: int, stream=None, check: bool = True) -> list[dict]:
    """Per-row diagnostics of the last forward on `stream` (synchronises it)."""
    arr = (Stats * max(1, int(max_rows)))()
    got = C.c_int64()
    rc = lib.lapsum_get_stats_rows(arr, max(1, int(max_rows)), C.byref(got), _stream(stream))
    if check:
        _check(rc, "lapsum_get_stats_rows")
    out = []
    for i in range(got.value):
        d = arr[i].as_dict()
        d["rc"] = rc
        out.append(d)
    return out


def bracket_plan(n: int, k: float, opts: Options | None = None) -> dict:
    """Sample size, ranks and band capacity the bracketing path would use (host only)."""
    s, jr, jl, cap = C.c_int64(), C.c_int64(), C.c_int64(), C.c_int64()
    rc = lib.lapsum_bracket_plan(int(n), float(k), C.byref(opts) if opts is not None else None,
                                 C.byref(s), C.byref(jr), C.byref(jl), C.byref(cap))
    _check(rc, "lapsum_bracket_plan")
    return {"s": s.value, "jR": jr.value, "jL": jl.value, "band_cap": cap.value}


def release():
    _check(lib.lapsum_release(), "lapsum_release")


def launch_count() -> int:
    return int(lib.lapsum_launch_count())


def profile_enable(mode: int = 1):
    lib.lapsum_profile_enable(int(mode))


def profile_filter(substring: str | None = None):
    lib.lapsum_profile_filter(substring.encode() if substring else None)


def selftest_math(which: int, x: torch.Tensor) -> tuple[torch.Tensor, torch.Tensor]:
    """(ours, CUDA library) for which = 0: 2^{-x} near-tier exp; 1: the sampler's ln."""
    _need(x, "x", torch.float64)
    out, ref = torch.empty_like(x), torch.empty_like(x)
    _check(lib.lapsum_selftest_math(int(which), x.data_ptr(), out.data_ptr(), ref.data_ptr(), x.numel(),
                                    _stream(None)), "lapsum_selftest_math")
    return out, ref


def profile_read() -> dict:
    """{kernel: (launches, total_ms)} of the launches recorded since profile_enable (syncs)."""
    cap = 64
    names = (C.c_char_p * cap)()
    launches = (C.c_int64 * cap)()
    ms = (C.c_double * cap)()
    m = lib.lapsum_profile_read(names, launches, ms, cap)
    return {names[i].decode(): (int(launches[i]), float(ms[i])) for i in range(min(m, cap))}


def forward_host(scores_host: torch.Tensor, k: float, t: float, device="cuda", opts=None,
                 stream=None) -> tuple[torch.Tensor, torch.Tensor]:
    """End-to-end call on host tensors: copy in, solve on the GPU, copy p and b back
    (the copies and the solve all on `stream`, default the current stream)."""
    with torch.cuda.stream(stream) if stream is not None else contextlib.nullcontext():
        d = scores_host.to(device, non_blocking=True)
        p, b = forward(d, k, t, opts=opts)
        return p.to("cpu", non_blocking=False), b.to("cpu", non_blocking=False)


def step_host(scores_h: torch.Tensor, g_h: torch.Tensor, k: float, t: float, p_h: torch.Tensor,
              b_h: torch.Tensor, grad_h: torch.Tensor, scores_d: torch.Tensor, g_d: torch.Tensor,
              p_d: torch.Tensor, b_d: torch.Tensor, grad_d: torch.Tensor, opts: Options | None = None,
              stream=None) -> None:
    """One forward + VJP step on host tensors (lapsum_step_host): scores_h and g_h
    in, p_h, b_h and grad_h out, through the caller's device buffers; the copies
    overlap the work where the data allow.  Asynchronous on `stream`: the host
    results are there once it has been synchronised.  Pinned host tensors let the
    copies run asynchronously."""
    rows, n = _as_rows(scores_h)
    for x, name, dt in ((scores_h, "scores_h", torch.float32), (g_h, "g_h", torch.float32),
                        (p_h, "p_h", torch.float32), (b_h, "b_h", torch.float64),
                        (grad_h, "grad_h", torch.float32)):
        if x.is_cuda or x.dtype != dt or not x.is_contiguous():
            raise ValueError(f"{name} must be a contiguous host tensor of {dt}")
    for x, name, dt in ((scores_d, "scores_d", torch.float32), (g_d, "g_d", torch.float32),
                        (p_d, "p_d", torch.float32), (b_d, "b_d", torch.float64),
                        (grad_d, "grad_d", torch.float32)):
        _need(x, name, dt, device=scores_d.device)
    for x, name in ((g_h, "g_h"), (p_h, "p_h"), (grad_h, "grad_h"), (scores_d, "scores_d"), (g_d, "g_d"),
                    (p_d, "p_d"), (grad_d, "grad_d")):
        if x.numel() != rows * n:
            raise ValueError(f"{name} must hold rows x n = {rows} x {n} values")
    if b_h.numel() != rows or b_d.numel() != rows:
        raise ValueError("b_h and b_d must hold one threshold per row")
    with _on(scores_d.device):
        rc = lib.lapsum_step_host(scores_h.data_ptr(), g_h.data_ptr(), rows, n, float(k), float(t),
                                  p_h.data_ptr(), b_h.data_ptr(), grad_h.data_ptr(),
                                  C.byref(opts) if opts is not None else None, scores_d.data_ptr(),
                                  g_d.data_ptr(), p_d.data_ptr(), b_d.data_ptr(), grad_d.data_ptr(),
                                  _stream(stream))
    _check(rc, "lapsum_step_host")


class _SoftTopK(torch.autograd.Function):
    @staticmethod
    def forward(ctx, scores, k, t, opts):
        p, b = forward(scores.contiguous(), k, t, opts=opts)
        ctx.save_for_backward(scores, b)
        ctx.t = t
        return p

    @staticmethod
    def backward(ctx, g):
        scores, b = ctx.saved_tensors
        grad = backward(scores.contiguous(), b, g.contiguous().float(), ctx.t)
        return grad, None, None, None


def soft_topk(scores: torch.Tensor, k: float, t: float, opts: Options | None = None) -> torch.Tensor:
    """Exact-budget soft top-k mask p (sum p = k per row), differentiable in scores."""
    return _SoftTopK.apply(scores, k, t, opts)
