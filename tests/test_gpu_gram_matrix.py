"""GPU parity of laplex_gram_matrix, M = A diag(D) A^T with A_ij = exp(-|a_i - b_j|),
against the oracle's dense definition.  Normaliser: A diag(|D|) A^T entry by
entry; fp32 slack: every term whose kernel product exp(-|a_i - b| - |a_j - b|) is
below FLT_MIN may be flushed, at most FLT_MIN sum_b |D_b| per entry."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


def run(a, b, D, use_perm=True):
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    sa, sb = sa.astype(a.dtype), sb.astype(b.dtype)
    Dd = None if D is None else dev(D)
    if use_perm:
        return host(X.gram_matrix(dev(sa), dev(sb), Dd, dev(pa.astype(np.int32)), dev(pb.astype(np.int32))))
    Ms = host(X.gram_matrix(dev(sa), dev(sb), None if D is None else dev(D[pb])))
    M = np.empty_like(Ms)
    M[np.ix_(pa, pa)] = Ms
    return M


def check(a, b, D, dtype, what):
    ref = O.gram_matrix(a, b, D)
    norm = O.gram_matrix(a, b, None if D is None else np.abs(D))
    slack = np.finfo(np.float32).tiny * (b.size if D is None else np.abs(D).sum())
    for use_perm in (True, False):
        M = run(a, b, D, use_perm)
        assert_close(M.ravel(), ref.ravel(), norm.ravel(), dtype, f"{what} perm={use_perm}",
                     np.full(M.size, slack))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n,k", [(1, 1), (1, 7), (7, 1), (5, 3), (300, 37), (1000, 5000), (2500, 777)])
def test_sizes(n, k, dtype):
    rng = np.random.default_rng(n * 3 + k)
    a = rng.uniform(-40, 40, n).astype(dtype)
    b = rng.uniform(-50, 50, k).astype(dtype)
    m = min(k // 50, n)
    b[:m] = a[:m]  # some ties between a and b
    D = rng.uniform(0.1, 2.0, k).astype(dtype)
    check(a, b, D, dtype, f"n={n} k={k}")
    check(a, b, None, dtype, f"n={n} k={k} D=1")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_edge_cases(dtype):
    rng = np.random.default_rng(31)
    a = rng.uniform(0, 10, 800).astype(dtype)
    check(a, rng.uniform(40, 60, 900).astype(dtype), rng.normal(size=900).astype(dtype), dtype, "b right, D signed")
    check(np.full(600, 2.0, dtype=dtype), np.full(700, 2.0, dtype=dtype), None, dtype, "all tied")
    check(np.round(rng.uniform(0, 20, 900)).astype(dtype), np.round(rng.uniform(0, 20, 5000)).astype(dtype),
          rng.uniform(0, 1, 5000).astype(dtype), dtype, "integer grid ties")
    # dense b: 100000 points in 3 units (the fp64 prefix sums keep the middle sums exact)
    check(rng.uniform(0, 3, 500).astype(dtype), rng.uniform(0, 3, 100000).astype(dtype),
          rng.uniform(0.5, 1.5, 100000).astype(dtype), dtype, "dense b")
    # k = 0: M = 0
    M = host(X.gram_matrix(dev(np.sort(a)), dev(np.zeros(0, dtype))))
    assert np.all(M == 0)
