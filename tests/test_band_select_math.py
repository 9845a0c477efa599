"""The band select's bin arithmetic against the definition of G (CPU, fp64).

The band solve of the bracketing path ("Fast LapSum: Exact Differentiable
Top-k at Million Scale", technical summary section 2.2 step 3) narrows the band
by bins of its descending-order key range instead of sorting it.  Its claims:
  * with A_j = sum_{r in bin j} e^{(r - e_j)/t}, B_j = sum_{r in bin j} e^{(e_{j+1} - r)/t}
    and d_j = e^{(e_{j+1} - e_j)/t}, the recurrences U_{j+1} = B_j + d_j U_j (from
    U_0 = sum_{r >= a_R} e^{(a_R - r)/t}) and V_j = A_j + d_j V_{j+1} (from
    V_J = sum_{r < a_L} e^{(r - a_L)/t}) give G(e_j) = C_j - U_j/2 + V_j/2 at every edge;
  * with every term of a bin at its largest (1) or smallest (d_j) value the same
    recurrences bound G from the bin counts alone.
This module restates that arithmetic in numpy and checks it against the
oracle's G evaluated from the definition at the same edges.  Host logic only:
it imports neither the CUDA path nor its sources.
"""
import numpy as np
import pytest

import workloads as W


def desc_key(x: np.ndarray) -> np.ndarray:
    u = np.asarray(x, dtype=np.float32).view(np.uint32).astype(np.uint64)
    return np.where(u & 0x80000000, u, u ^ 0x7FFFFFFF).astype(np.uint64)


def key_value(k: int) -> float:
    k = int(k) & 0xFFFFFFFF
    u = k if k & 0x80000000 else k ^ 0x7FFFFFFF
    return float(np.array([u], dtype=np.uint32).view(np.float32)[0])


def bins_and_edges(band, top, bot, bits=10):
    keys = desc_key(band)
    klo, khi = int(keys.min()), int(keys.max())
    w = khi - klo
    nb = w.bit_length()
    s = max(0, nb - bits)
    J = (w >> s) + 1
    edges = [top] + [key_value(klo + (j << s) - 1) for j in range(1, J)] + [bot]
    j_of = ((keys - klo) >> s).astype(np.int64)
    return j_of, np.array(edges, dtype=np.float64), J


def edge_G(r_all, band, a_L, a_R, t):
    """G at every bin edge from the bin recurrences, and the count-only bounds."""
    above = r_all[r_all >= a_R].astype(np.float64)
    below = r_all[r_all < a_L].astype(np.float64)
    S_R = np.sum(np.exp(-(above - a_R) / t))
    S_L = np.sum(np.exp((below - a_L) / t))
    j_of, e, J = bins_and_edges(band, float(a_R), float(a_L))
    x = band.astype(np.float64)
    A = np.zeros(J)
    B = np.zeros(J)
    cnt = np.zeros(J)
    np.add.at(A, j_of, np.exp((x - e[j_of]) / t))
    np.add.at(B, j_of, np.exp((e[j_of + 1] - x) / t))
    np.add.at(cnt, j_of, 1.0)
    assert np.all(x <= e[j_of]) and np.all(x >= e[j_of + 1])   # e_{j+1} <= r < e_j (up to ties at +-0)
    d = np.exp((e[1:] - e[:-1]) / t)
    U = np.zeros(J + 1); Umax = np.zeros(J + 1); Umin = np.zeros(J + 1)
    V = np.zeros(J + 1); Vmax = np.zeros(J + 1); Vmin = np.zeros(J + 1)
    U[0] = Umax[0] = Umin[0] = S_R
    V[J] = Vmax[J] = Vmin[J] = S_L
    for j in range(J):
        U[j + 1] = B[j] + d[j] * U[j]
        Umax[j + 1] = cnt[j] + d[j] * Umax[j]
        Umin[j + 1] = cnt[j] * d[j] + d[j] * Umin[j]
    for j in range(J - 1, -1, -1):
        V[j] = A[j] + d[j] * V[j + 1]
        Vmax[j] = cnt[j] + d[j] * Vmax[j + 1]
        Vmin[j] = cnt[j] * d[j] + d[j] * Vmin[j + 1]
    C = above.size + np.concatenate([[0.0], np.cumsum(cnt)])
    G = C - 0.5 * U + 0.5 * V
    Ghi = C - 0.5 * Umin + 0.5 * Vmax
    Glo = C - 0.5 * Umax + 0.5 * Vmin
    return e, G, Glo, Ghi


@pytest.mark.parametrize("dist,n,k,t,lo_q,hi_q", [
    ("normal", 200_000, 2000.0, 0.05, 0.985, 0.995),
    ("laplace", 300_000, 3000.0, 0.02, 0.985, 0.994),
    ("normal", 100_000, 50_000.0, 0.05, 0.45, 0.55),      # a band across zero: both signs
])
def test_bin_recurrences_give_G_at_every_edge(orc, dist, n, k, t, lo_q, hi_q):
    r, _ = W.small_case(dist, 1, n, seed=31)
    r = r[0]
    a_L = np.float32(np.quantile(r, lo_q))
    a_R = np.float32(np.quantile(r, hi_q))
    band = r[(r >= a_L) & (r < a_R)]
    e, G, Glo, Ghi = edge_G(r, band, a_L, a_R, t)
    for j in np.linspace(0, e.size - 1, 40).astype(int):
        Gdef, _ = orc.G(r, float(e[j]), t)
        assert abs(G[j] - Gdef) <= 1e-9 * max(1.0, abs(Gdef)), (j, G[j], Gdef)
        assert Glo[j] - 1e-9 * max(1.0, Gdef) <= Gdef <= Ghi[j] + 1e-9 * max(1.0, Gdef)
    # G at the edges rises with the edge index (falls as b rises)
    assert np.all(np.diff(G) >= -1e-9 * np.maximum(1.0, G[1:]))


def test_count_bounds_leave_a_narrow_window(orc):
    # bins much narrower than t: the bounds differ by a factor e^{width/t} ~ 1,
    # so the window that must hold b spans only a few bins
    r, _ = W.small_case("laplace", 1, 400_000, seed=32)
    r = r[0]
    k, t = 4000.0, 0.05
    b = orc.solve(r, k, t, method=1)
    a_L = np.float32(np.quantile(r, 0.985))
    a_R = np.float32(np.quantile(r, 0.995))
    band = r[(r >= a_L) & (r < a_R)]
    e, G, Glo, Ghi = edge_G(r, band, a_L, a_R, t)
    jlo = int(np.max(np.nonzero(Ghi < k)[0]))     # edges above b
    jhi = int(np.min(np.nonzero(Glo >= k)[0]))    # edges at or below b
    assert e[jhi] <= b < e[jlo]
    assert 1 <= jhi - jlo <= 8, (jlo, jhi, e.size)
