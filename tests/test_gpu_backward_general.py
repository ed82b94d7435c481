"""GPU parity of laplex_backward_general (L = <g, K x>, K_ij = exp(-|a_i - b_j|)):
dx = K^T g, da_i = -g_i S(a <- b, x)_i, db_j = -x_j S(b <- a, g)_j with
S(p <- q, v)_i = sum_j sign(p_i - q_j) exp(-|p_i - q_j|) v_j, sign(0) = 0, against
the fp64 oracle.  Normalisers: K^T|g| for dx, |g| K|x| for da, |x| K^T|g| for db;
fp32 slack: the oracle's mass of the terms below FLT_MIN (oracle.far_mass)."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


def run(a, b, x, g, use_perm=True):
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    sa, sb = sa.astype(a.dtype), sb.astype(b.dtype)
    if use_perm:
        dx, da, db = X.backward_general(dev(sa), dev(sb), dev(x), dev(g), dev(pa.astype(np.int32)),
                                        dev(pb.astype(np.int32)))
        return host(dx), host(da), host(db)
    dxs, das, dbs = X.backward_general(dev(sa), dev(sb), dev(x[pb]), dev(g[pa]))
    dx, da, db = np.empty_like(host(dxs)), np.empty_like(host(das)), np.empty_like(host(dbs))
    dx[pb], da[pa], db[pb] = host(dxs), host(das), host(dbs)
    return dx, da, db


def check(a, b, x, g, dtype, what):
    rdx, rda, rdb = O.backward_general(a, b, x, g)
    ndx, nda, ndb = O.norm_backward_general(a, b, x, g)
    mg_b, mx_a = O.far_mass(b, g, a), O.far_mass(a, x, b)
    for use_perm in (True, False):
        dx, da, db = run(a, b, x, g, use_perm)
        assert_close(dx, rdx, ndx, dtype, f"{what} dx perm={use_perm}", mg_b)
        assert_close(da, rda, nda, dtype, f"{what} da perm={use_perm}", np.abs(g) * mx_a)
        assert_close(db, rdb, ndb, dtype, f"{what} db perm={use_perm}", np.abs(x) * mg_b)


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n,k", [(1, 1), (1, 5), (5, 1), (3, 2), (100, 37), (3071, 3073),
                                 (4097, 100), (100, 4097), (30011, 50021)])
def test_sizes(n, k, dtype):
    """a, b ~ U(-50, 50) with 1 % of b equal to entries of a (ties, sign 0)."""
    a, b, x, _ = synth.general_ties(n, k, -50.0, 50.0, seed=n + k, dtype=dtype)
    g = np.random.default_rng(n * 7 + k).normal(size=n).astype(dtype)
    check(a, b, x, g, dtype, f"n={n} k={k}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_edge_cases(dtype):
    rng = np.random.default_rng(23)
    x = rng.normal(size=3000).astype(dtype)
    g = rng.normal(size=2000).astype(dtype)
    a = rng.uniform(0, 10, 2000).astype(dtype)
    check(a, (rng.uniform(40, 60, 3000)).astype(dtype), x, g, dtype, "b right")
    check(a, (rng.uniform(-30, -20, 3000)).astype(dtype), x, g, dtype, "b left")
    check(np.full(2000, 1.5, dtype=dtype), np.full(3000, 1.5, dtype=dtype), x, g, dtype, "all tied")
    # sparse, spacing ~1: the scans' halos carry (n, k spanning many tiles)
    a2 = rng.uniform(0, 60000, 40000).astype(dtype)
    b2 = rng.uniform(0, 60000, 50000).astype(dtype)
    check(a2, b2, rng.normal(size=50000).astype(dtype), rng.normal(size=40000).astype(dtype), dtype,
          "sparse")


def test_empty_sides():
    """n = 0 or k = 0: the outputs on the other side are zero."""
    b = np.linspace(0, 5, 7).astype(np.float32)
    x = np.ones(7, dtype=np.float32)
    dx, da, db = X.backward_general(dev(np.zeros(0, np.float32)), dev(b), dev(x), dev(np.zeros(0, np.float32)))
    assert np.all(host(dx) == 0) and np.all(host(db) == 0) and host(da).size == 0


def test_c3_full_size():
    """The general workload: a in R^(2^22), b in R^(2^20) ~ U(-1000, 1000), 1 % ties;
    x ~ N(0, 1) on b, g ~ N(0, 1) on a."""
    a, b, x, w = synth.general_ties(1 << 22, 1 << 20, -1000.0, 1000.0, seed=0)
    check(a, b, x, w, np.float32, "C3")
