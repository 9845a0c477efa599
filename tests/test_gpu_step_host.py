"""lapsum_step_host: one forward + VJP step on host buffers, the copies on the
library's side streams overlapping the work ("Fast LapSum: Exact Differentiable
Top-k at Million Scale", technical summary sections 2.1-2.2).  The results must
equal, bit for bit, those of lapsum_forward_ex + lapsum_backward on device
buffers of the same inputs (the same kernels run on the same data)."""
import numpy as np
import pytest
import torch

import workloads as W

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_budget_soft_b200 as lib
    return lib


def host(x, pinned):
    t = torch.from_numpy(np.ascontiguousarray(x))
    return t.pin_memory() if pinned else t


@pytest.mark.parametrize("pinned", [True, False])
@pytest.mark.parametrize("rows,n,dist,k,t", [(1, 1 << 20, "normal", 1000.0, 0.05),
                                            (1, 1_500_001, "laplace", 150.0, 0.01),
                                            (64, 4096, "normal", 64.0, 0.05)])
def test_step_host_equals_the_device_calls(L, rows, n, dist, k, t, pinned):
    r, g = W.small_case(dist, rows, n, seed=61)
    rh, gh = host(r, pinned), host(g, pinned)
    ph, grh = host(np.zeros_like(r), pinned), host(np.zeros_like(r), pinned)
    bh = host(np.zeros(rows, np.float64), pinned)
    rd, gd, pd, grd = (torch.empty(rows, n, dtype=torch.float32, device="cuda") for _ in range(4))
    bd = torch.empty(rows, dtype=torch.float64, device="cuda")
    for _ in range(2):   # twice with the same buffers: the second call's copies follow the first's work
        L.step_host(rh, gh, k, t, ph, bh, grh, rd, gd, pd, bd, grd)
    torch.cuda.current_stream().synchronize()
    r2, g2 = torch.from_numpy(r).cuda(), torch.from_numpy(g).cuda()
    p2, b2 = L.forward(r2, k, t)
    grad2 = L.backward(r2, b2, g2, t)
    torch.cuda.synchronize()
    assert torch.equal(bh, b2.cpu())
    assert torch.equal(ph.reshape(rows, n), p2.cpu().reshape(rows, n))
    assert torch.equal(grh.reshape(rows, n), grad2.cpu().reshape(rows, n))
    assert L.get_stats()["rc"] == 0


def test_step_host_grad_may_overwrite_g_on_the_device(L):
    r, g = W.small_case("normal", 1, 1 << 20, seed=62)
    k, t = 500.0, 0.05
    rh, gh = host(r, True), host(g, True)
    ph, grh, bh = host(np.zeros_like(r), True), host(np.zeros_like(r), True), host(np.zeros(1, np.float64), True)
    rd, gd, pd = (torch.empty(1, r.shape[1], dtype=torch.float32, device="cuda") for _ in range(3))
    bd = torch.empty(1, dtype=torch.float64, device="cuda")
    L.step_host(rh, gh, k, t, ph, bh, grh, rd, gd, pd, bd, gd)   # grad written over g's device copy
    torch.cuda.current_stream().synchronize()
    r2, g2 = torch.from_numpy(r).cuda(), torch.from_numpy(g).cuda()
    p2, b2 = L.forward(r2, k, t)
    assert torch.equal(grh, L.backward(r2, b2, g2, t).cpu())


@pytest.mark.parametrize("on_side_stream", [False, True])
def test_forward_host_equals_the_device_call(L, on_side_stream):
    # forward_host: the copy in, the solve and the copies out all on one stream
    r, _ = W.small_case("normal", 1, 1 << 20, seed=67)
    p0, b0 = L.forward(torch.from_numpy(r).cuda(), 1000.0, 0.05)
    torch.cuda.synchronize()
    s = torch.cuda.Stream() if on_side_stream else None
    if s is not None:
        s.wait_stream(torch.cuda.current_stream())
    p, b = L.forward_host(host(r, True), 1000.0, 0.05, stream=s)
    assert not p.is_cuda and not b.is_cuda
    assert torch.equal(p, p0.cpu()) and torch.equal(b, b0.cpu())
