"""GPU parity of laplex_matvec_general (a != b), y = K x and z = K^T w, against
the fp64 oracle's u/v interval aggregation; sorted anchors and permutations fed
to the kernels come from the oracle's stable sort."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


def run_general(a, b, x, transpose=False, use_perm=True):
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    sa, sb = sa.astype(a.dtype), sb.astype(b.dtype)
    if use_perm:
        y = X.matvec_general(dev(sa), dev(sb), dev(x), dev(pa.astype(np.int32)),
                             dev(pb.astype(np.int32)), transpose=transpose)
        return host(y)
    pin, pout = (pa, pb) if transpose else (pb, pa)
    ys = host(X.matvec_general(dev(sa), dev(sb), dev(x[pin]), transpose=transpose))
    y = np.empty_like(ys)
    y[pout] = ys
    return y


def check(a, b, x, w, dtype, what):
    y_ref = O.general(a, b, x)
    my = O.far_mass(a, x, b)
    assert_close(run_general(a, b, x), y_ref, O.norm_general(a, b, x), dtype, what + " Kx", my)
    assert_close(run_general(a, b, x, use_perm=False), y_ref, O.norm_general(a, b, x), dtype,
                 what + " Kx sorted", my)
    z_ref = O.general_T(a, b, w)
    assert_close(run_general(a, b, w, transpose=True), z_ref, O.norm_general(b, a, w), dtype,
                 what + " K^T w", O.far_mass(b, w, a))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n,k", [(1, 1), (1, 5), (5, 1), (3, 2), (100, 37), (2047, 2049),
                                 (2048, 2048), (4097, 100), (100, 4097), (30011, 50021)])
def test_sizes(n, k, dtype):
    a, b, x, w = synth.general_ties(n, k, -50.0, 50.0, seed=n + k, dtype=dtype)
    check(a, b, x, w, dtype, f"n={n} k={k}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("B", [2, 3, 8, 9])
def test_columns(B, dtype):
    n, k = 9001, 7003
    a, b, _, _ = synth.general_ties(n, k, 0.0, 400.0, seed=B, dtype=dtype)
    rng = np.random.default_rng(B)
    x = rng.normal(size=(k, B)).astype(dtype)
    w = rng.normal(size=(n, B)).astype(dtype)
    check(a, b, x, w, dtype, f"B={B}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_edge_cases(dtype):
    rng = np.random.default_rng(5)
    x = rng.normal(size=3000).astype(dtype)
    w = rng.normal(size=2000).astype(dtype)
    # disjoint ranges (b entirely to the right, then to the left)
    a = rng.uniform(0, 10, 2000).astype(dtype)
    check(a, (a[:1500] + 100).astype(dtype)[np.arange(3000) % 1500], x, w, dtype, "b right")
    check(a, (rng.uniform(-50, -40, 3000)).astype(dtype), x, w, dtype, "b left")
    # every anchor tied: b = a repeated
    check(np.full(2000, 1.5, dtype=dtype), np.full(3000, 1.5, dtype=dtype), x, w, dtype, "all tied")
    # b is a exactly (the general product equals the symmetric one)
    a2 = rng.uniform(-3, 3, 3000).astype(dtype)
    y = run_general(a2, a2, x)
    assert_close(y, O.sym(a2, x), O.norm_sym(a2, x), dtype, "b == a")
    # dense: 200000 anchors in one unit (deep carries -> deferred tiles)
    a3 = rng.uniform(0, 1, 200000).astype(dtype)
    b3 = rng.uniform(0, 1, 150000).astype(dtype)
    x3 = rng.normal(size=150000).astype(dtype)
    w3 = rng.normal(size=200000).astype(dtype)
    check(a3, b3, x3, w3, dtype, "dense")


def test_k_zero_gives_zeros():
    a = np.linspace(0, 1, 100).astype(np.float32)
    y = X.matvec_general(dev(a), dev(np.zeros(0, np.float32)), dev(np.zeros(0, np.float32)))
    assert np.array_equal(host(y), np.zeros(100, np.float32))


def test_c3_full_size():
    """a in R^(2^22) ~ U(-1000, 1000), b in R^(2^20) with 1 % of b equal to entries
    of a, x ~ N(0,1)^(2^20), w ~ N(0,1)^(2^22): every output of y = K x and
    z = K^T w against the oracle."""
    a, b, x, w = synth.general_ties(1 << 22, 1 << 20, -1000.0, 1000.0, seed=0)
    assert np.isin(b, a).mean() > 0.009
    check(a, b, x, w, np.float32, "C3")


@pytest.mark.parametrize("case", ["sparse", "b_spacing_0.46", "b_spacing_0.47", "b_sparse_a_dense",
                                  "runs_of_64"])
def test_halo_carries(case):
    """Merged tiles whose carries come from halos of 192 b-points (exact when
    they span the cut of 88 or reach the end of b), next to tiles that fall
    back to the carry kernels and the redo pass."""
    rng = np.random.default_rng(29)
    if case == "sparse":
        a = rng.uniform(0, 60000, 40000)
        b = rng.uniform(0, 60000, 30000)
    elif case.startswith("b_spacing_"):
        sp = float(case.split("_")[-1])
        b = np.arange(30000) * sp
        a = rng.uniform(0, b[-1], 20000)
    elif case == "b_sparse_a_dense":
        b = rng.uniform(0, 30000, 20000)
        a = rng.uniform(1000, 1010, 50000)
    else:
        b = 2.0 ** 29 + 64.0 * (np.arange(30000) // 64)
        a = 2.0 ** 29 + 64.0 * (np.arange(25000) // 50) + 7.0
    a, b = a.astype(np.float32), b.astype(np.float32)
    x = rng.normal(size=b.size).astype(np.float32)
    w = rng.normal(size=a.size).astype(np.float32)
    check(a, b, x, w, np.float32, case)
