"""Device math helpers against the CUDA math library (through the C ABI).

* The near-tier exponential of the tail sums (table-driven 2^{-w}, after Tang,
  ACM TOMS 1989) must stay within 8 ulp of exp2 on [0, 1000].
* The sampler's own ln (2 atanh((m-1)/(m+1)) series) must stay within 2 ulp of
  log on (0, 1] -- and its bits must equal the oracle's restatement, which is
  what makes the bracket ends bit-exact between GPU and CPU.
"""
import numpy as np
import pytest
import torch

pytestmark = pytest.mark.gpu


@pytest.fixture(scope="module")
def L():
    if not torch.cuda.is_available():
        pytest.skip("no CUDA device")
    import exact_budget_soft_b200 as lib
    return lib


def test_near_tier_exp2_vs_library(L):
    rng = np.random.default_rng(0)
    w = np.concatenate([np.linspace(0, 24, 200001), rng.uniform(0, 1000, 100000),
                        np.arange(0, 1000, 1 / 32), [0.0, 1 / 64, 1 / 64 + 1e-12, 23.0831206]])
    x = torch.from_numpy(w).cuda()
    ours, ref = L.selftest_math(0, x)
    ours, ref = ours.cpu().numpy(), ref.cpu().numpy()
    ok = ref > 1e-300                       # stay clear of the subnormal range
    ulp = np.spacing(ref[ok])
    assert np.max(np.abs(ours[ok] - ref[ok]) / ulp) <= 8


def test_sampler_ln_vs_library_and_oracle(L, orc):
    rng = np.random.default_rng(1)
    u = np.concatenate([(np.arange(1, 200001, dtype=np.float64)) * 2.0 ** -53 * 2 ** 30,
                        rng.random(200000), [1.0, 0.5, 2.0 ** -53, 1 - 2.0 ** -53]])
    u = u[(u > 0) & (u <= 1)]
    x = torch.from_numpy(u).cuda()
    ours, ref = L.selftest_math(1, x)
    ours, ref = ours.cpu().numpy(), ref.cpu().numpy()
    nz = ref != 0
    assert np.all(ours[~nz] == 0)
    assert np.max(np.abs(ours[nz] - ref[nz]) / np.spacing(np.abs(ref[nz]))) <= 2
    sub = u[:: max(1, u.size // 3000)]
    gpu_sub = ours[:: max(1, u.size // 3000)]
    assert all(orc.ln(float(v)) == float(gv) for v, gv in zip(sub, gpu_sub))
