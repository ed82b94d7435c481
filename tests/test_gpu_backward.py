"""GPU parity of laplex_backward (L = <g, K x>): dx = K g and
da_i = -g_i D(x)_i - x_i D(g)_i with D(v)_i = sum_j sign(a_i - a_j) K_ij v_j,
sign(0) = 0, against the fp64 oracle.  Normalisers: K0|g| for dx and
|g| K0|x| + |x| K0|g| for da."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host, rows_local

pytestmark = pytest.mark.gpu


def run_bwd(a, x, g, use_perm=True):
    s, perm = O.stable_sort(a)
    s = s.astype(a.dtype)
    if use_perm:
        dx, da = X.backward(dev(s), dev(x), dev(g), dev(perm.astype(np.int32)))
        return host(dx), host(da)
    dxs, das = X.backward(dev(s), dev(x[perm]), dev(g[perm]))
    dx, da = np.empty_like(host(dxs)), np.empty_like(host(das))
    dx[perm] = host(dxs)
    da[perm] = host(das)
    return dx, da


def check(a, x, g, dtype, what):
    rdx, rda = O.backward(a, x, g)
    ndx, nda = O.norm_backward(a, x, g)
    mx, mg = O.far_mass(a, x), O.far_mass(a, g)
    sda = np.abs(g) * mx + np.abs(x) * mg
    for use_perm in (True, False):
        dx, da = run_bwd(a, x, g, use_perm)
        assert_close(dx, rdx, ndx, dtype, f"{what} dx perm={use_perm}", mg)
        assert_close(da, rda, nda, dtype, f"{what} da perm={use_perm}", sda)


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 2, 3, 17, 2047, 2048, 2049, 4097, 100003])
def test_sizes(n, dtype):
    a, x, g = synth.sym_uniform(n, 0.0, float(n), seed=n, dtype=dtype, with_g=True)
    check(a, x, g, dtype, f"n={n}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_ties(dtype):
    rng = np.random.default_rng(2)
    n = 60000
    x = rng.normal(size=n).astype(dtype)
    g = rng.normal(size=n).astype(dtype)
    check(np.round(rng.uniform(0, 300, n)).astype(dtype), x, g, dtype, "coarse grid")
    check((64.0 * np.round(rng.uniform(0, 2000, n))).astype(dtype), x, g, dtype, "64-apart groups")
    check(np.full(n, 2.0, dtype=dtype), x, g, dtype, "all equal")
    check(rng.uniform(0, 1, n).astype(dtype), x, g, dtype, "dense")
    check((np.arange(n) * 200.0).astype(dtype), x, g, dtype, "far apart")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_deep_dependencies(dtype):
    """Ties and decays spanning far more tiles than the look-ahead waits for."""
    rng = np.random.default_rng(4)
    n = 700001
    x = rng.normal(size=n).astype(dtype)
    g = rng.normal(size=n).astype(dtype)
    a = np.concatenate([np.full(n // 2, -1.0), rng.uniform(0, 0.5, n - n // 2)]).astype(dtype)
    check(a, x, g, dtype, "long tie run + dense")


def test_c5_full_size_sampled():
    """n = 2^30, a ~ U(0, 2^30) ascending (fp32 rounding: runs of up to 64 equal
    anchors), x, g ~ N(0,1): 10^4 sampled rows of dx and da against the dense
    definition, plus the first and last 4096 rows."""
    n = 1 << 30
    s, x, g = synth.sym_uniform(n, 0.0, float(1 << 30), seed=0, presorted=True, with_g=True)
    dx, da = X.backward(dev(s), dev(x), dev(g))
    dx, da = host(dx), host(da)
    idx = np.concatenate([synth.randint(10000, n, seed=1, stream="misc"),
                          np.arange(4096), np.arange(n - 4096, n)])
    kx, sx, nx = rows_local(s, x, idx)
    kg, sg, ng = rows_local(s, g, idx)
    assert_close(dx[idx], kg, ng, np.float32, "C5 dx")
    da_ref = -(g[idx] * sx + x[idx] * sg)
    assert_close(da[idx], da_ref, np.abs(g[idx]) * nx + np.abs(x[idx]) * ng, np.float32, "C5 da")


@pytest.mark.parametrize("case", ["spacing_0.46", "spacing_0.47", "spacing_1.0", "mixed_ties", "short_right",
                                  "runs_of_64"])
def test_halo_carries(case):
    """Tiles whose carries come from the halos of 192 elements, next to tiles
    that fall back to the carry kernels and the redo pass: spacing 0.46 spans
    87.9 < 88 (fall back), 0.47 spans 89.8 (halo carries); runs of equal
    anchors inside the halos (and runs of 64 equal anchors 64 apart, the fp32
    grid of a ~ U(0, 2^30) above 2^29); a last-but-one tile without room for
    a right halo."""
    rng = np.random.default_rng(21)
    tile = 256 * 8
    n = 11 * tile + 77
    if case.startswith("spacing_"):
        a = np.arange(n) * float(case.split("_")[1])
    elif case == "runs_of_64":
        a = 2.0 ** 29 + 64.0 * (np.arange(n) // 64)
    elif case == "mixed_ties":
        # groups of equal anchors 3 apart, a dense stretch, then unit spacing
        k = n // 3
        a = np.concatenate([3.0 * np.repeat(np.arange(k // 8 + 1), 8)[:k],
                            3.0 * (k // 8 + 2) + np.sort(rng.uniform(0, 5, k)),
                            3.0 * (k // 8 + 2) + 10 + np.arange(n - 2 * k)])
    else:
        n = 9 * tile + 100
        a = rng.uniform(0, n, n)
    a = a.astype(np.float32)
    x = rng.normal(size=n).astype(np.float32)
    g = rng.normal(size=n).astype(np.float32)
    check(a, x, g, np.float32, case)


@pytest.mark.parametrize("L", [2, 5, 12, 13, 37, 64, 100, 191, 193, 385, 3072, 5000])
@pytest.mark.parametrize("n", [7 * 3072 + 1234, 7 * 3072 + 100])
def test_runs_across_chunks_and_tiles(L, n):
    """Runs of L equal anchors, L apart (about one unit per element, so the
    halos of the exp channels span the cut for short runs), shifted so that
    run boundaries fall at several offsets from the chunk (12 elements) and
    tile (3072) boundaries: the run sums of the sorted-order pass cross
    neighbouring chunks, the tile edges and the halos; runs longer than 32
    chunks or than a halo list their tiles for the four-channel redo pass.
    n = 7 * 3072 + 100 leaves the last full tile without room for a right halo."""
    rng = np.random.default_rng(L)
    for off in (0, 7):
        a = (float(L) * ((np.arange(n) + off) // L)).astype(np.float32)
        x = rng.normal(size=n).astype(np.float32)
        g = rng.normal(size=n).astype(np.float32)
        check(a, x, g, np.float32, f"L={L} off={off}")
