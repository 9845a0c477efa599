"""The allocation-free backward entry point (lapsum_backward_noalloc).

It serves callers that may not call cudaMalloc while they run -- plugins inside
a framework that owns all device memory, processes held to a fixed memory
budget -- by keeping its scratch in an array compiled into the library.  These tests call it through
the C ABI and compare it with lapsum_backward on the same inputs, two calls in a
row (the second call must not see the first call's leftovers), and check that a
call too large for the array is refused.  The file is named to be collected
last, and it also passes when run on its own.
"""
import ctypes as C

import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu

TOL_VJP = 1e-4       # relative L2, as in the parity tests


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_budget_soft_b200 as lib
    fn = lib.lib.lapsum_backward_noalloc
    fn.argtypes = [C.c_void_p, C.c_void_p, C.c_void_p, C.c_int64, C.c_int64, C.c_double, C.c_void_p,
                   C.c_void_p]
    fn.restype = C.c_int
    return lib


def noalloc(L, r, b, g, t):
    rows, n = r.shape
    out = torch.empty_like(r)
    rc = L.lib.lapsum_backward_noalloc(r.data_ptr(), b.data_ptr(), g.data_ptr(), rows, n, float(t),
                                       out.data_ptr(), torch.cuda.current_stream().cuda_stream)
    assert rc == 0
    return out


def case(L, dist, rows, n, k, t, seed):
    r_np, g_np = W.small_case(dist, rows, n, seed=seed)
    r, g = torch.from_numpy(r_np).cuda(), torch.from_numpy(g_np).cuda()
    _, b = L.forward(r, k, t)
    return r, b, g


def rel_l2(a, b):
    a, b = a.double().cpu().numpy(), b.double().cpu().numpy()
    return np.linalg.norm(a - b) / np.linalg.norm(b)


def test_matches_backward_two_calls_in_a_row(L):
    cases = [("normal", 1, 1 << 20, 1000.0, 0.05, 1), ("laplace", 64, 4096, 40.0, 0.02, 2),
             ("levels256_desc", 3, 100_003, 900.0, 0.1, 3), ("normal", 1, 1 << 20, 500.0, 0.2, 4)]
    for dist, rows, n, k, t, seed in cases:
        r, b, g = case(L, dist, rows, n, k, t, seed)
        ref = L.backward(r, b, g, t)
        first = noalloc(L, r, b, g, t)
        second = noalloc(L, r, b, g, t)
        torch.cuda.synchronize()
        assert rel_l2(first, ref) <= TOL_VJP, (dist, rows, n)
        assert rel_l2(second, ref) <= TOL_VJP, (dist, rows, n)
        assert torch.equal(first, second)


def test_refuses_calls_that_do_not_fit(L):
    fake = C.c_void_p(0x1000)   # never dereferenced: the size check comes first
    rc = L.lib.lapsum_backward_noalloc(fake, fake, fake, 7282, 16, 0.1, fake, None)
    assert rc == -1
    rc = L.lib.lapsum_backward_noalloc(fake, fake, fake, 1, 16, 0.0, fake, None)
    assert rc == -1
