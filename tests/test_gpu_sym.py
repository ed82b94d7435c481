"""GPU parity of laplex_matvec_sym against the fp64 oracle (same seeded inputs).

Criterion: max_i |y_i - y_ref_i| / (K0|x|)_i <= 1e-4 (fp32), 1e-10 (fp64).
The sorted anchors and the permutation fed to the kernel come from the oracle's
stable sort, never from the CUDA path."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host, rows_local

pytestmark = pytest.mark.gpu


def run_sym(a, x, use_perm=True):
    s, perm = O.stable_sort(a)
    s = s.astype(a.dtype)
    if use_perm:
        y = X.matvec_sym(dev(s), dev(x), dev(perm.astype(np.int32)))
        return host(y)
    xs = x[perm]
    ys = host(X.matvec_sym(dev(s), dev(xs)))
    y = np.empty_like(ys)
    y[perm] = ys
    return y


def test_c1_n4096_dense_oracle():
    """n = 4096, a ~ U(0, 64), x ~ N(0, 1), seed 0: checked against the dense fp64
    definition and the sequential oracle."""
    a, x = synth.sym_uniform(4096, 0.0, 64.0, seed=0)
    y_dense = O.dense_matvec(a, x)
    y_seq = O.sym(a, x)
    norm = O.norm_sym(a, x)
    assert O.max_norm_err(y_seq, y_dense, norm) < 1e-13
    for use_perm in (True, False):
        y = run_sym(a, x, use_perm)
        assert_close(y, y_dense, norm, np.float32, f"C1 perm={use_perm}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 2, 3, 5, 31, 33, 4095, 4096, 4097, 65537, 300001])
def test_ragged_sizes(n, dtype):
    a, x = synth.sym_uniform(n, -50.0, 50.0, seed=n, dtype=dtype)
    y_ref = O.sym(a, x)
    norm = O.norm_sym(a, x)
    for use_perm in (True, False):
        assert_close(run_sym(a, x, use_perm), y_ref, norm, dtype, f"n={n} perm={use_perm}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("B", [2, 3, 4, 5, 8, 11, 16])
def test_columns(B, dtype):
    n = 20011
    a, x = synth.sym_uniform(n, 0.0, 300.0, B=B, seed=B, dtype=dtype)
    y_ref = O.sym(a, x)
    norm = O.norm_sym(a, x)
    for use_perm in (True, False):
        assert_close(run_sym(a, x, use_perm), y_ref, norm, dtype, f"B={B} perm={use_perm}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_ties_and_degenerate(dtype):
    rng = np.random.default_rng(7)
    n = 50000
    # heavy ties: anchors on a coarse grid
    a = np.round(rng.uniform(0, 200, n)).astype(dtype)
    x = rng.normal(size=n).astype(dtype)
    assert_close(run_sym(a, x), O.sym(a, x), O.norm_sym(a, x), dtype, "ties")
    # all anchors equal: y_i = sum(x)
    a = np.full(n, 3.5, dtype=dtype)
    assert_close(run_sym(a, x), O.sym(a, x), O.norm_sym(a, x), dtype, "all equal")
    # anchors far apart: y = x
    a = (np.arange(n) * 200.0).astype(dtype)
    assert_close(run_sym(a, x), x.astype(np.float64), np.abs(x) + 1e-300, dtype, "far apart")
    # very dense: 50000 anchors within one unit
    a = rng.uniform(0, 1, n).astype(dtype)
    assert_close(run_sym(a, x), O.sym(a, x), O.norm_sym(a, x), dtype, "dense")


def test_c2_full_size_b1_b8():
    """Symmetric matvec, n = 2^24, a ~ N(0, 2000^2) unsorted, x ~ N(0,1) of shape
    (n, B), B in {1, 8}: every output against the sequential fp64 oracle."""
    n = 1 << 24
    for B in (1, 8):
        a, x = synth.sym_normal(n, 2000.0, B=B, seed=0)
        y_ref = O.sym(a, x)
        norm = O.norm_sym(a, x)
        assert_close(run_sym(a, x, True), y_ref, norm, np.float32, f"C2 B={B}")


def test_c5_full_size_presorted_sampled():
    """n = 2^30, a ~ U(0, 2^30) generated ascending (the pre-sorted launch the
    benchmark times), x ~ N(0,1): 10^4 sampled rows against the dense definition
    evaluated row by row over the window where fp64 terms are non-zero."""
    n = 1 << 30
    s, x = synth.sym_uniform(n, 0.0, float(1 << 30), seed=0, presorted=True)
    assert np.all(s[1:] >= s[:-1])
    y = host(X.matvec_sym(dev(s), dev(x)))
    idx = synth.randint(10000, n, seed=0, stream="misc")
    out, _, absn = rows_local(s, x, idx)
    assert_close(y[idx], out, absn, np.float32, "C5 sampled rows")
    # the first and last 4096 rows (the tile edges of the array) in full
    for lo, hi in ((0, 4096), (n - 4096, n)):
        sub = np.arange(lo, hi)
        out, _, absn = rows_local(s, x, sub)
        assert_close(y[sub], out, absn, np.float32, f"C5 rows {lo}..{hi}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_deep_lookahead_fixup(dtype):
    """Dependencies that span more tiles than the look-ahead may wait for: all
    anchors equal (every output is sum(x)) and 10^6 anchors inside one unit.
    Exercises the deferred suffix-carry fix-up."""
    n = 1_000_003
    rng = np.random.default_rng(11)
    x = rng.normal(size=n).astype(dtype)
    a = np.full(n, -7.0, dtype=dtype)
    assert_close(run_sym(a, x, False), O.sym(a, x), O.norm_sym(a, x), dtype, "all equal")
    a = rng.uniform(0, 1, n).astype(dtype)
    assert_close(run_sym(a, x, True), O.sym(a, x), O.norm_sym(a, x), dtype, "dense")
    xb = rng.normal(size=(n, 3)).astype(dtype)
    assert_close(run_sym(a, xb, True), O.sym(a, xb), O.norm_sym(a, xb), dtype, "dense B=3")


TILE_F32 = 256 * 12  # elements per tile of the single-column fp32 product
HALO_SPACINGS = [0.30, 0.345, 0.35, 0.46, 0.47, 0.69, 0.70, 1.0]


def _spaced(n, spacing, seed, jitter=0.0):
    rng = np.random.default_rng(seed)
    a = np.arange(n) * spacing + rng.uniform(0, jitter, n) if jitter else np.arange(n) * spacing
    return np.sort(a).astype(np.float32), rng.normal(size=n).astype(np.float32)


@pytest.mark.parametrize("use_perm", [False, True])
@pytest.mark.parametrize("spacing", HALO_SPACINGS)
def test_halo_span_boundary(spacing, use_perm):
    """Constant anchor spacing around the points where a halo spans the cut of
    88: with 192 elements 191 x 0.46 = 87.9 falls back to the carry kernels
    and the redo pass, 191 x 0.47 = 89.8 takes the halo carries (0.69 / 0.70
    for halos of 128, 0.345 / 0.35 for halos of 256)."""
    n = 9 * TILE_F32 + 1234
    a, x = _spaced(n, spacing, seed=int(spacing * 1000))
    assert_close(run_sym(a, x, use_perm), O.sym(a, x), O.norm_sym(a, x), np.float32,
                 f"spacing {spacing} perm={use_perm}")


@pytest.mark.parametrize("use_perm", [False, True])
@pytest.mark.parametrize("case", ["unit", "mixed", "far", "aligned", "short_right", "runs_of_64"])
def test_halo_carries(case, use_perm):
    """Tiles whose carries come from the halos (sparse anchors) and tiles that
    fall back to the carry kernels and the redo pass (denser), side by side."""
    n = 7 * TILE_F32 + 1234
    if case == "unit":
        a, x = synth.sym_uniform(n, 0.0, float(n), seed=3)
    elif case == "mixed":
        # alternating sparse and dense stretches, with jumps between them
        rng = np.random.default_rng(6)
        parts, lo = [], 0.0
        for k in range(9):
            m = 3000 + 1500 * k
            dens = (0.05, 1.0, 2.5, 0.3)[k % 4]
            parts.append(lo + np.sort(rng.uniform(0, m * dens, m)))
            lo += m * dens + (0.0 if k % 3 else 50.0)
        a = np.concatenate(parts).astype(np.float32)
        n = a.size
        x = rng.normal(size=n).astype(np.float32)
    elif case == "far":
        a, x = _spaced(n, 150.0, seed=7)
    elif case == "runs_of_64":
        # the fp32 grid of a ~ U(0, 2^30) above 2^29: runs of 64 equal anchors
        a = (2.0 ** 29 + 64.0 * (np.arange(n) // 64)).astype(np.float32)
        x = np.random.default_rng(10).normal(size=n).astype(np.float32)
    elif case == "aligned":
        n = 5 * TILE_F32
        a, x = synth.sym_uniform(n, 0.0, float(n), seed=8)
    else:  # the tile before the ragged last one has no room for a right halo
        n = 6 * TILE_F32 + 100
        a, x = synth.sym_uniform(n, 0.0, float(n), seed=9)
    y_ref = O.sym(a, x)
    norm = O.norm_sym(a, x)
    assert_close(run_sym(a, x, use_perm), y_ref, norm, np.float32, f"{case} perm={use_perm}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("B", [2, 4, 8])
def test_columns_dense_and_tied(B, dtype):
    """Several columns (the column-parallel kernels), in sorted order and
    through perm: carries that cross every tile (10^5 anchors in one unit; all
    anchors equal) and a size that leaves a ragged last tile."""
    rng = np.random.default_rng(B)
    for n, a in ((100_003, rng.uniform(0.0, 1.0, 100_003)), (5_003, np.full(5_003, 2.5)),
                 (70_001, np.round(rng.uniform(0.0, 400.0, 70_001)))):
        a = a.astype(dtype)
        x = synth.normal(n * B, seed=n, stream="x", dtype=dtype).reshape(n, B)
        y_ref = O.sym(a, x)
        for use_perm in (False, True):  # through perm: rows gathered once, the same kernels, rows scattered
            assert_close(run_sym(a, x, use_perm=use_perm), y_ref, O.norm_sym(a, x), dtype,
                         f"n={n} B={B} perm={use_perm}", slack=O.far_mass(a, x))
