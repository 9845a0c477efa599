"""fp64 CPU oracle for the Fast LapSum exact-budget soft top-k (TEST INFRASTRUCTURE).

Only the tests, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import this package.  It shares no code with the CUDA path.

The arithmetic lives in ``lapsum_oracle.c`` (plain C, fp64, OpenMP over fixed
chunks); this module builds it with gcc on first use and wraps it with ctypes.
Every function cites the passage it follows in the C source:

* ``solve``      -- the unique b with sum_i F((r_i-b)/t) = k, by bisection on the
                    definition (or safeguarded Newton, ``method=1``).
* ``p``          -- p_i = F((r_i-b)/t).
* ``vjp``        -- grad = (f/t)(g - <g,f>/sum f).
* ``G``          -- the budget function itself (and sum f).
* ``sort_desc``  -- the scores in descending order (fp64).
* ``tail_sums``  -- the streaming pass's tail sums S_L, S_R from their definition.
* ``philox``, ``ln``, ``sample``, ``binom_ranks``, ``bracket``, ``counts``,
  ``certify`` -- an independent restatement of the probabilistic bracket, for
  exact comparison of the integer results with the GPU path.
"""
from __future__ import annotations

import ctypes as C
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "lapsum_oracle.c")
_LIB = os.path.join(_HERE, "liblapsum_oracle.so")
_lock = threading.Lock()
_lib = None

CFLAGS = ["-O2", "-std=c11", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
          "-shared", "-fPIC", "-Wall", "-Wextra"]


def build(force: bool = False) -> str:
    """Compile the oracle with gcc (idempotent)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        tmp = _LIB + f".tmp{os.getpid()}"
        subprocess.check_call(["gcc", *CFLAGS, "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _LIB)
    return _LIB


def _load():
    global _lib
    with _lock:
        if _lib is None:
            lib = C.CDLL(build())
            f32p = np.ctypeslib.ndpointer(np.float32, flags="C_CONTIGUOUS")
            f64p = np.ctypeslib.ndpointer(np.float64, flags="C_CONTIGUOUS")
            i64p = np.ctypeslib.ndpointer(np.int64, flags="C_CONTIGUOUS")
            u64p = np.ctypeslib.ndpointer(np.uint64, flags="C_CONTIGUOUS")
            dp, ip, lp = C.POINTER(C.c_double), C.POINTER(C.c_int), C.POINTER(C.c_int64)
            fp = C.POINTER(C.c_float)
            sig = {
                "orc_laplace_cdf": (C.c_double, [C.c_double]),
                "orc_laplace_icdf": (C.c_double, [C.c_double]),
                "orc_G": (C.c_int, [f32p, C.c_int64, C.c_double, C.c_double, dp, dp]),
                "orc_solve": (C.c_int, [f32p, C.c_int64, C.c_double, C.c_double, C.c_int, dp, ip]),
                "orc_p": (None, [f32p, C.c_int64, C.c_double, C.c_double, f64p]),
                "orc_vjp": (None, [f32p, f32p, C.c_int64, C.c_double, C.c_double, f64p, dp, dp]),
                "orc_sort_desc": (None, [f32p, C.c_int64, f64p]),
                "orc_tail_sums": (None, [f32p, C.c_int64, C.c_float, C.c_float, C.c_double, dp, dp, dp, dp]),
                "orc_philox4x64_10": (None, [u64p, u64p, u64p]),
                "orc_ln": (C.c_double, [C.c_double]),
                "orc_sample": (None, [f32p, C.c_int64, C.c_double, C.c_uint64, C.c_int64,
                                      C.c_int64, f64p, i64p]),
                "orc_binom_ranks": (C.c_int, [C.c_int64, C.c_double, C.c_double, lp, lp]),
                "orc_widen_ranks": (C.c_int, [C.c_int64, C.c_double, C.c_double, lp, lp]),
                "orc_bracket_at_ranks": (C.c_int, [f32p, C.c_int64, C.c_double, C.c_uint64, C.c_int64,
                                                   C.c_int64, C.c_int64, C.c_int64, fp, fp]),
                "orc_bracket": (C.c_int, [f32p, C.c_int64, C.c_double, C.c_double, C.c_uint64,
                                          C.c_int64, C.c_int64, C.c_double, fp, fp, lp, lp]),
                "orc_counts": (None, [f32p, C.c_int64, C.c_float, C.c_float, lp, lp, lp]),
                "orc_certify": (C.c_int, [f32p, C.c_int64, C.c_double, C.c_double, C.c_float,
                                          C.c_float, C.c_int64, dp, dp, lp, lp, lp]),
                "orc_num_threads": (C.c_int, []),
            }
            for name, (res, args) in sig.items():
                fn = getattr(lib, name)
                fn.restype = res
                fn.argtypes = args
            _lib = lib
    return _lib


def _f32(a) -> np.ndarray:
    return np.ascontiguousarray(np.asarray(a, dtype=np.float32).ravel())


def num_threads() -> int:
    return int(_load().orc_num_threads())


def laplace_cdf(x: float) -> float:
    return float(_load().orc_laplace_cdf(float(x)))


def G(r, b: float, t: float) -> tuple[float, float]:
    """(G(b), sum f) over all scores of one row."""
    r = _f32(r)
    g, sf = C.c_double(), C.c_double()
    rc = _load().orc_G(r, r.size, float(b), float(t), C.byref(g), C.byref(sf))
    if rc != 0:
        raise ValueError("non-finite score")
    return g.value, sf.value


def solve(r, k: float, t: float, method: int = 0) -> float:
    """b of one row (fp64)."""
    r = _f32(r)
    b, ev = C.c_double(), C.c_int()
    rc = _load().orc_solve(r, r.size, float(k), float(t), int(method), C.byref(b), C.byref(ev))
    if rc != 0:
        raise ValueError(f"orc_solve failed ({rc})")
    return b.value


def solve_rows(r2d, k: float, t: float, method: int = 0) -> np.ndarray:
    r2d = np.asarray(r2d, dtype=np.float32)
    return np.array([solve(row, k, t, method) for row in r2d], dtype=np.float64)


def p(r, b: float, t: float) -> np.ndarray:
    r = _f32(r)
    out = np.empty(r.size, dtype=np.float64)
    _load().orc_p(r, r.size, float(b), float(t), out)
    return out


def vjp(r, g, b: float, t: float) -> tuple[np.ndarray, float, float]:
    """(grad, <g,f>, sum f) of one row."""
    r, g = _f32(r), _f32(g)
    out = np.empty(r.size, dtype=np.float64)
    gf, sf = C.c_double(), C.c_double()
    _load().orc_vjp(r, g, r.size, float(b), float(t), out, C.byref(gf), C.byref(sf))
    return out, gf.value, sf.value


def sort_desc(r) -> np.ndarray:
    r = _f32(r)
    out = np.empty(r.size, dtype=np.float64)
    _load().orc_sort_desc(r, r.size, out)
    return out


def tail_sums(r, a_L: float, a_R: float, t: float) -> dict:
    """Streaming-pass tail sums S_L, S_R from their definition, and the parts of
    each made of terms with |r - a|/t > 16."""
    r = _f32(r)
    v = [C.c_double() for _ in range(4)]
    _load().orc_tail_sums(r, r.size, float(a_L), float(a_R), float(t), *[C.byref(x) for x in v])
    return {"S_L": v[0].value, "S_R": v[1].value, "S_L_far": v[2].value, "S_R_far": v[3].value}


def philox(counter, key) -> np.ndarray:
    c = np.ascontiguousarray(np.asarray(counter, dtype=np.uint64))
    k = np.ascontiguousarray(np.asarray(key, dtype=np.uint64))
    out = np.empty(4, dtype=np.uint64)
    _load().orc_philox4x64_10(c, k, out)
    return out


def ln(x: float) -> float:
    return float(_load().orc_ln(float(x)))


def sample(r, t: float, seed: int, s: int, row: int = 0) -> tuple[np.ndarray, np.ndarray]:
    r = _f32(r)
    y = np.empty(s, dtype=np.float64)
    idx = np.empty(s, dtype=np.int64)
    _load().orc_sample(r, r.size, float(t), int(seed), int(row), int(s), y, idx)
    return y, idx


def binom_ranks(s: int, pi: float, delta: float) -> tuple[int, int]:
    jr, jl = C.c_int64(), C.c_int64()
    rc = _load().orc_binom_ranks(int(s), float(pi), float(delta), C.byref(jr), C.byref(jl))
    if rc != 0:
        raise ValueError("bad binomial arguments")
    return jr.value, jl.value


def bracket(r, k: float, t: float, seed: int, s: int, delta: float, row: int = 0) -> dict:
    r = _f32(r)
    aL, aR = C.c_float(), C.c_float()
    jr, jl = C.c_int64(), C.c_int64()
    rc = _load().orc_bracket(r, r.size, float(k), float(t), int(seed), int(row), int(s),
                             float(delta), C.byref(aL), C.byref(aR), C.byref(jr), C.byref(jl))
    if rc != 0:
        raise ValueError("bad bracket arguments")
    return {"a_L": np.float32(aL.value), "a_R": np.float32(aR.value), "jR": jr.value, "jL": jl.value}


def widen_ranks(s: int, pi: float, delta: float) -> tuple[int, int]:
    """Ranks (jR2, jL2) of the widening round (delta^2 ranks, moved at least one
    first-round spread beyond the first round's ranks)."""
    jr, jl = C.c_int64(), C.c_int64()
    rc = _load().orc_widen_ranks(int(s), float(pi), float(delta), C.byref(jr), C.byref(jl))
    if rc != 0:
        raise ValueError("bad binomial arguments")
    return jr.value, jl.value


def bracket_at_ranks(r, t: float, seed: int, s: int, jR: int, jL: int, row: int = 0) -> dict:
    r = _f32(r)
    aL, aR = C.c_float(), C.c_float()
    rc = _load().orc_bracket_at_ranks(r, r.size, float(t), int(seed), int(row), int(s), int(jR), int(jL),
                                      C.byref(aL), C.byref(aR))
    if rc != 0:
        raise ValueError("bad rank arguments")
    return {"a_L": np.float32(aL.value), "a_R": np.float32(aR.value), "jR": jR, "jL": jL}


def counts(r, a_L: float, a_R: float) -> tuple[int, int, int]:
    r = _f32(r)
    cl, cb, cr = C.c_int64(), C.c_int64(), C.c_int64()
    _load().orc_counts(r, r.size, float(a_L), float(a_R), C.byref(cl), C.byref(cb), C.byref(cr))
    return cl.value, cb.value, cr.value


def certify(r, k: float, t: float, a_L: float, a_R: float, band_cap: int) -> dict:
    r = _f32(r)
    gl, gr = C.c_double(), C.c_double()
    cl, cb, cr = C.c_int64(), C.c_int64(), C.c_int64()
    v = _load().orc_certify(r, r.size, float(k), float(t), float(a_L), float(a_R), int(band_cap),
                            C.byref(gl), C.byref(gr), C.byref(cl), C.byref(cb), C.byref(cr))
    return {"verdict": int(v), "G_aL": gl.value, "G_aR": gr.value,
            "c_L": cl.value, "c_band": cb.value, "c_R": cr.value}
