"""Host-side checks of the C ABI that need no GPU: the library builds for
sm_100a, loads, exports every entry point include/lapsum.h declares, rejects
bad arguments before touching a device, and plans the bracket (sample size,
binomial ranks, band capacity) exactly as the oracle's restatement does."""
import ctypes as C
import os
import re
import subprocess

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "lapsum.h")


def _lib_path():
    import importlib.util
    spec = importlib.util.spec_from_file_location("lapsum_build",
                                                  os.path.join(ROOT, "exact_budget_soft_b200", "build.py"))
    mod = importlib.util.module_from_spec(spec)
    spec.loader.exec_module(mod)
    return mod.build()


@pytest.fixture(scope="module")
def lib():
    return C.CDLL(_lib_path())


def declared_symbols():
    text = open(HEADER).read()
    return sorted(set(re.findall(r"LAPSUM_API\s+[\w\s\*]+?\b(lapsum_\w+)\s*\(", text)))


def test_header_declares_the_entry_points():
    names = declared_symbols()
    for must in ("lapsum_forward", "lapsum_backward", "lapsum_forward_ex", "lapsum_get_stats"):
        assert must in names


def test_library_exports_every_declared_symbol(lib):
    out = subprocess.check_output(["nm", "-D", "--defined-only", _lib_path()]).decode()
    exported = set(re.findall(r"\sT\s(lapsum_\w+)", out))
    missing = [s for s in declared_symbols() if s not in exported]
    assert not missing, missing
    for s in declared_symbols():
        assert getattr(lib, s)


def test_strerror(lib):
    lib.lapsum_strerror.restype = C.c_char_p
    assert lib.lapsum_strerror(0) == b"ok"
    assert b"argument" in lib.lapsum_strerror(-1)


@pytest.mark.parametrize("rows,n,k,t", [(0, 10, 1.0, 1.0), (1, 0, 1.0, 1.0), (1, 10, 0.0, 1.0),
                                        (1, 10, 10.0, 1.0), (1, 10, 2.0, 0.0), (1, 10, 2.0, -1.0),
                                        (1, 10, float("nan"), 1.0), (1, 10, 2.0, float("inf")),
                                        (1, 10, 2.0, 1e-37), (1, 10, 2.0, 1e37)])
def test_bad_arguments_rejected_on_host(lib, rows, n, k, t):
    lib.lapsum_forward.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_double, C.c_double,
                                   C.c_void_p, C.c_void_p, C.c_void_p]
    fake = C.c_void_p(0x1000)   # never dereferenced: the check comes first
    assert lib.lapsum_forward(fake, rows, n, k, t, fake, fake, None) == -1
    lib.lapsum_backward.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64,
                                    C.c_double, C.c_void_p, C.c_void_p]
    if rows < 1 or n < 1 or not (1e-36 <= t <= 1e36):
        assert lib.lapsum_backward(fake, fake, fake, rows, n, t, fake, None) == -1
        lib.lapsum_backward_noalloc.argtypes = lib.lapsum_backward.argtypes
        assert lib.lapsum_backward_noalloc(fake, fake, fake, rows, n, t, fake, None) == -1


def test_null_pointers_rejected(lib):
    lib.lapsum_forward.argtypes = [C.c_void_p, C.c_int64, C.c_int64, C.c_double, C.c_double,
                                   C.c_void_p, C.c_void_p, C.c_void_p]
    assert lib.lapsum_forward(None, 1, 10, 2.0, 1.0, None, None, None) == -1


STEP_HOST_ARGS = [C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_double, C.c_double, C.c_void_p, C.c_void_p,
                  C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]


@pytest.mark.parametrize("null_at", range(10))
def test_step_host_rejects_a_null_buffer(lib, null_at):
    # lapsum_step_host: any null host or device buffer is refused before anything is enqueued
    lib.lapsum_step_host.argtypes = STEP_HOST_ARGS
    bufs = [C.c_void_p(0x1000 + 0x100 * i) for i in range(10)]   # never dereferenced
    bufs[null_at] = None
    sh, gh, ph, bh, grh, sd, gd, pd, bd, grd = bufs
    assert lib.lapsum_step_host(sh, gh, 1, 10, 2.0, 1.0, ph, bh, grh, None, sd, gd, pd, bd, grd, None) == -1


@pytest.mark.parametrize("rows,n,k,t", [(0, 10, 1.0, 1.0), (1, 10, 10.0, 1.0), (1, 10, 2.0, 0.0),
                                        (1, 10, float("nan"), 1.0), (1, 10, 2.0, 1e37)])
def test_step_host_rejects_bad_sizes(lib, rows, n, k, t):
    lib.lapsum_step_host.argtypes = STEP_HOST_ARGS
    f = C.c_void_p(0x1000)
    assert lib.lapsum_step_host(f, f, rows, n, k, t, f, f, f, None, f, f, f, f, f, None) == -1


class Options(C.Structure):
    _fields_ = [("seed", C.c_uint64), ("sample_size", C.c_int64), ("delta", C.c_double),
                ("band_cap", C.c_int64), ("spin_cap", C.c_int32), ("force_path", C.c_int32),
                ("certify", C.c_int32), ("widen", C.c_int32), ("reserved", C.c_int32 * 2)]


@pytest.mark.parametrize("field,value", [("force_path", 7), ("certify", 2), ("widen", 2), ("delta", 1.5),
                                         ("sample_size", -1), ("band_cap", -5), ("spin_cap", -2)])
def test_step_host_rejects_bad_options_before_enqueueing(lib, field, value):
    # an invalid option is refused before any copy is queued (the pointers are
    # never dereferenced, and no device is needed to get the answer)
    lib.lapsum_step_host.argtypes = STEP_HOST_ARGS
    f = C.c_void_p(0x1000)
    o = Options()
    setattr(o, field, value)
    assert lib.lapsum_step_host(f, f, 1, 10, 2.0, 1.0, f, f, f, C.byref(o), f, f, f, f, f, None) == -1


def test_step_host_rejects_a_batch_too_tall_for_the_bracketing_grid(lib):
    lib.lapsum_step_host.argtypes = STEP_HOST_ARGS
    f = C.c_void_p(0x1000)
    o = Options()
    o.force_path = 2   # bracketing: one grid slice per row, at most 65535 rows
    assert lib.lapsum_step_host(f, f, 65536, 16, 2.0, 1.0, f, f, f, C.byref(o), f, f, f, f, f, None) == -1



def _plan(lib, n, k, s=0, delta=0.0):
    lib.lapsum_bracket_plan.argtypes = [C.c_int64, C.c_double, C.POINTER(Options)] + [C.POINTER(C.c_int64)] * 4
    o = Options()
    o.sample_size, o.delta = s, delta
    out = [C.c_int64() for _ in range(4)]
    rc = lib.lapsum_bracket_plan(n, k, C.byref(o), *[C.byref(x) for x in out])
    assert rc == 0
    return [x.value for x in out]


@pytest.mark.parametrize("n,k,s,delta", [(1_048_576, 210, 0, 0.0), (10_000_000, 1e5, 0, 0.0),
                                         (100_000_000, 1e6, 0, 0.0), (100_000_000, 1e6, 4096, 0.5),
                                         (5000, 60, 512, 0.2), (3000, 60.0, 512, 0.2),
                                         (2_000_000, 1.5, 0, 1e-3), (2_000_000, 1999999.0, 0, 1e-9)])
def test_bracket_plan_matches_oracle_ranks(lib, orc, n, k, s, delta):
    s_, jR, jL, cap = _plan(lib, n, k, s, delta)
    if s == 0:
        pw = 1
        while pw * 2 <= n // 64:
            pw *= 2
        assert s_ == min(65536, max(4096, pw))
    assert (jR, jL) == orc.binom_ranks(s_, k / n, delta or 1e-6)
    assert 0 < cap <= n


def test_bracket_plan_ranks_fuzz(lib, orc):
    # the library's log-free ratio recurrence and the oracle's lgamma sums pick the same ranks
    import numpy as np
    rng = np.random.default_rng(0)
    for _ in range(400):
        s = int(rng.choice([50, 512, 1000, 4096, 16384, 65536]))
        pi = float(10 ** rng.uniform(-6, -0.01))
        delta = float(10 ** rng.uniform(-9, -0.3))
        n = 10 ** 9
        _, jR, jL, _ = _plan(lib, n, pi * n, s, delta)
        assert (jR, jL) == orc.binom_ranks(s, pi, delta)
    # budgets near n and far below one sample's worth, confidence down to 1e-12
    for i in range(300):
        s = int(rng.choice([50, 333, 4096, 5000, 65536]))
        pi = float(1 - 10 ** rng.uniform(-6, -0.31)) if i % 2 else float(10 ** rng.uniform(-8, -6))
        delta = float(10 ** rng.uniform(-12, -0.3))
        n = 10 ** 9
        _, jR, jL, _ = _plan(lib, n, pi * n, s, delta)
        assert (jR, jL) == orc.binom_ranks(s, pi * n / n, delta)


FWD_EX_ARGS = [C.c_void_p, C.c_int64, C.c_int64, C.c_double, C.c_double, C.c_void_p, C.c_void_p, C.c_void_p,
               C.c_void_p]


@pytest.mark.parametrize("field,value", [("force_path", 3), ("certify", 2), ("widen", 2), ("delta", 1.0),
                                         ("delta", -0.1), ("sample_size", -1), ("band_cap", -1),
                                         ("spin_cap", -2)])
def test_forward_rejects_bad_options_on_host(lib, field, value):
    lib.lapsum_forward_ex.argtypes = FWD_EX_ARGS
    f = C.c_void_p(0x1000)   # never dereferenced: the options are checked first
    o = Options()
    setattr(o, field, value)
    assert lib.lapsum_forward_ex(f, 1, 10, 2.0, 1.0, f, f, C.byref(o), None) == -1


def test_forward_rejects_a_batch_too_tall_for_the_bracketing_grid(lib):
    lib.lapsum_forward_ex.argtypes = FWD_EX_ARGS
    f = C.c_void_p(0x1000)
    assert lib.lapsum_forward_ex(f, 65536, 1 << 20, 1000.0, 0.1, f, f, None, None) == -1   # auto: bracketing


SHARD_SAMPLE_ARGS = [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_double, C.c_double, C.c_void_p,
                     C.c_void_p, C.c_void_p]
SHARD_STREAM_ARGS = [C.c_void_p, C.c_int64, C.c_int64, C.c_int64, C.c_double, C.c_double, C.c_void_p,
                     C.c_void_p, C.c_void_p, C.c_void_p, C.c_void_p]


@pytest.mark.parametrize("n_local,offset,n_total,field,value",
                         [(10, -1, 100, None, 0),           # a slice before the row
                          (60, 50, 100, None, 0),           # a slice past the row's end
                          (0, 0, 100, None, 0),             # an empty slice
                          (1, 0, 1, None, 0),               # a row of one score
                          (10, 0, 100, "widen", 1),         # no widening round on a split row
                          (10, 0, 100, "force_path", 1)])   # nor the full-sort path
def test_split_row_calls_reject_bad_slices_on_host(lib, n_local, offset, n_total, field, value):
    lib.lapsum_shard_sample.argtypes = SHARD_SAMPLE_ARGS
    lib.lapsum_shard_stream.argtypes = SHARD_STREAM_ARGS
    f = C.c_void_p(0x1000)
    o = Options()
    if field:
        setattr(o, field, value)
    assert lib.lapsum_shard_sample(f, n_local, offset, n_total, 2.0 if n_total > 2 else 0.5, 1.0, C.byref(o),
                                   f, None) == -1
    assert lib.lapsum_shard_stream(f, n_local, offset, n_total, 2.0 if n_total > 2 else 0.5, 1.0, C.byref(o),
                                   f, f, f, None) == -1


@pytest.mark.parametrize("n_total,k", [(1 << 20, 1000.0), (100_000_000, 1e6), (3_000_000, 0.5)])
def test_split_row_plan_sizes_the_exchange_buffers(lib, n_total, k):
    # the sample exchange buffer holds the s sample keys and the select's
    # histograms (65536 top-16-bit bins + 256 top-8-bit bins); the band capacity
    # is the one-GPU plan's
    lib.lapsum_shard_plan.argtypes = [C.c_int64, C.c_double, C.POINTER(Options), C.POINTER(C.c_int64),
                                      C.POINTER(C.c_int64)]
    words, cap = C.c_int64(), C.c_int64()
    assert lib.lapsum_shard_plan(n_total, k, None, C.byref(words), C.byref(cap)) == 0
    s, _, _, band_cap = _plan(lib, n_total, k)
    assert words.value == s + 65536 + 256
    assert cap.value == band_cap


C_CONSUMER = r"""
#include <stdio.h>
#include <string.h>
#include "lapsum.h"

int main(void) {
    lapsum_options o;
    memset(&o, 0, sizeof o);
    int64_t s = 0, jR = 0, jL = 0, cap = 0;
    if (strcmp(lapsum_strerror(LAPSUM_OK), "ok") != 0) return 1;
    if (lapsum_bracket_plan(100000000, 1e6, &o, &s, &jR, &jL, &cap) != LAPSUM_OK) return 2;
    if (!(s == 65536 && 0 < jR && jR < jL && jL <= s && cap > 0)) return 3;
    /* argument errors come back before any device work */
    if (lapsum_forward(NULL, 1, 10, 2.0, 1.0, NULL, NULL, NULL) != LAPSUM_ERR_ARG) return 4;
    if (lapsum_backward(NULL, NULL, NULL, 1, 10, 1.0, NULL, NULL) != LAPSUM_ERR_ARG) return 5;
    printf("%lld %lld %lld %lld\n", (long long)s, (long long)jR, (long long)jL, (long long)cap);
    return 0;
}
"""


def test_header_serves_a_plain_c_program(lib, tmp_path):
    # the boundary is a C ABI: a C11 program compiles against include/lapsum.h
    # with warnings as errors, links to the library and calls its host-side entry
    # points; its bracket plan equals the one ctypes sees
    src = tmp_path / "consumer.c"
    src.write_text(C_CONSUMER)
    exe = tmp_path / "consumer"
    libdir = os.path.dirname(_lib_path())
    subprocess.check_call(["gcc", "-std=c11", "-Wall", "-Wextra", "-Werror", "-I", os.path.join(ROOT, "include"),
                           str(src), "-o", str(exe), "-L", libdir, "-llapsum", f"-Wl,-rpath,{libdir}"])
    out = subprocess.check_output([str(exe)]).decode().split()
    s, jR, jL, cap = (int(x) for x in out)
    assert [s, jR, jL, cap] == _plan(lib, 100_000_000, 1e6)
