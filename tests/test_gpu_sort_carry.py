"""GPU parity of the sort that carries a value per anchor and of the one-call
product on anchors in the caller's order:

- laplex_sort_anchors_carry: perm and sorted bit for bit against the oracle's
  stable sort (as for laplex_sort_anchors), and xs == x[perm] bit for bit, with
  x drawn as arbitrary bit patterns (NaN payloads included: the values are moved,
  never computed on);
- laplex_matvec_sym_unsorted: y against the fp64 oracle of the symmetric
  product (criterion max_i |y_i - y_ref_i| / (K0|x|)_i within 1e-4 in fp32,
  terms below FLT_MIN allowed to vanish, 1e-10 in fp64), and its sorted / perm
  outputs against the oracle's sort;
- n = 2^30, a ~ U(0, 2^30) in caller order: the properties that define the
  stable sort (perm a permutation, a[perm] == sorted non-decreasing, ties in
  ascending index order), xs == x[perm], and sampled rows of y against the
  oracle's rows on windows of the sorted anchors."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host, rows_local

pytestmark = pytest.mark.gpu

UINT = {np.dtype(np.float32): np.uint32, np.dtype(np.float64): np.uint64}


def bits(n, dtype, seed):
    """n arbitrary bit patterns viewed as dtype."""
    u = UINT[np.dtype(dtype)]
    return np.random.default_rng(seed).integers(0, np.iinfo(u).max, size=n, dtype=u, endpoint=True).view(dtype)


def check_carry(a, x):
    s, p, xs = X.sort_anchors_carry(dev(a), dev(x))
    X.device_status()
    s, p, xs = host(s), host(p), host(xs)
    _, ref = O.stable_sort(a)
    assert np.array_equal(p, ref.astype(np.int32))
    u = UINT[a.dtype]
    assert np.array_equal(s.view(u), (a[ref] + a.dtype.type(0)).view(u))  # -0.0 stored as +0.0
    assert np.array_equal(xs.view(u), x[ref].view(u))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 2, 3, 100, 4095, 4096, 4097, 8193, 65536, (1 << 20) + 7])
def test_carry_sizes(n, dtype):
    check_carry(synth.normal(n, 0.0, 100.0, seed=n, stream="a", dtype=dtype), bits(n, dtype, n + 1))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_carry_special_values_and_ties(dtype):
    rng = np.random.default_rng(3)
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-40, -1e-40, 1.0, -1.0, 3.4e38, -3.4e38,
                         2.0 ** -126, -(2.0 ** -126)], dtype=np.float64)
    for n in (37, 5000, 300000):
        check_carry(rng.choice(specials, size=n).astype(dtype), bits(n, dtype, n))
    n = 200000
    check_carry(np.round(rng.normal(size=n) * 3).astype(dtype), bits(n, dtype, 1))   # heavy ties
    check_carry(np.full(n, -2.5, dtype=dtype), bits(n, dtype, 2))                     # one value
    check_carry(np.arange(n, 0, -1).astype(dtype), bits(n, dtype, 3))                 # reversed


def test_carry_c2_full_size_exact():
    """n = 2^24, a ~ N(0, 2000^2)."""
    n = 1 << 24
    check_carry(synth.normal(n, 0.0, 2000.0, seed=0, stream="a"), synth.normal(n, seed=0, stream="x"))


def test_carry_non_finite_reported():
    a = np.linspace(0, 1, 10000).astype(np.float32)
    a[777] = np.nan
    X.sort_anchors_carry(dev(a), dev(a))
    with pytest.raises(X.LaplexError) as e:
        X.device_status()
    assert e.value.status == X.ENONFINITE
    X.device_status()


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 5, 4097, 300001])
def test_unsorted_against_oracle(n, dtype):
    a, x = synth.sym_uniform(n, -50.0, 50.0, seed=n, dtype=dtype)
    y, s, p = X.matvec_sym_unsorted(dev(a), dev(x))
    X.device_status()
    _, ref = O.stable_sort(a)
    assert np.array_equal(host(p), ref.astype(np.int32))
    assert_close(host(y), O.sym(a, x), O.norm_sym(a, x), dtype, f"n={n}", slack=O.far_mass(a, x))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_unsorted_c1_against_dense(dtype):
    a, x = synth.sym_uniform(4096, 0.0, 64.0, seed=0, dtype=dtype)
    y, _, _ = X.matvec_sym_unsorted(dev(a), dev(x))
    assert_close(host(y), O.dense_matvec(a, x), O.norm_sym(a, x), dtype, "C1 unsorted")


def test_unsorted_c2_full_size():
    """n = 2^24, a ~ N(0, 2000^2) in caller order, x ~ N(0, 1)."""
    a, x = synth.sym_normal(1 << 24, 2000.0, B=1, seed=0)
    y, _, _ = X.matvec_sym_unsorted(dev(a), dev(x))
    X.device_status()
    assert_close(host(y), O.sym(a, x), O.norm_sym(a, x), np.float32, "C2 unsorted", slack=O.far_mass(a, x))


def test_c5_full_size():
    """n = 2^30, a ~ U(0, 2^30) and x ~ N(0, 1) in caller order.  The sort
    carrying x: the properties that define the stable sort (perm a permutation,
    a[perm] == sorted non-decreasing, ties in ascending index order) and
    xs == x[perm] bit for bit.  The one-call product: the same sorted and perm,
    and 4096 sampled rows plus the first and last 64 rows of sorted order
    against the oracle's rows."""
    n = 1 << 30
    a = synth.uniform(n, 0.0, float(1 << 30), seed=0, stream="a")
    x = synth.normal(n, seed=0, stream="x")
    a_d, x_d = dev(a), dev(x)
    s_d, p_d, xs_d = X.sort_anchors_carry(a_d, x_d)
    X.device_status()
    s, p, xs_gpu = host(s_d), host(p_d), host(xs_d)
    del s_d, xs_d
    seen = np.zeros(n, dtype=np.bool_)
    seen[p] = True
    assert seen.all()
    del seen
    ap = a[p]
    assert np.array_equal(ap.view(np.uint32), s.view(np.uint32))
    d = np.diff(ap)
    assert (d >= 0).all()
    assert (np.diff(p)[d == 0] > 0).all()
    del ap, d
    xs = x[p]
    assert np.array_equal(xs_gpu.view(np.uint32), xs.view(np.uint32))
    del xs_gpu
    y_d, s2_d, p2_d = X.matvec_sym_unsorted(a_d, x_d)
    X.device_status()
    assert bool((p2_d == p_d).all())
    del p_d, p2_d, s2_d, a_d, x_d
    y = host(y_d)
    r = np.concatenate([np.arange(64), n - 64 + np.arange(64), synth.randint(4096, n, seed=1, stream="misc")])
    out, _, absn = rows_local(s, xs, r)
    assert_close(y[p[r]], out, absn, np.float32, "C5 unsorted sampled rows")


def test_carry_expired_wait_reports_timeout():
    """The carrying sort's copy waits are bounded like the plain sort's: with
    every block's first copy left unissued and a bound of 16 polls, the call
    returns, the status is LAPLEX_ETIMEOUT (cleared once read), and the next
    call is exact."""
    n = 100_000
    a = synth.normal(n, 0.0, 100.0, seed=5, stream="a")
    x = bits(n, np.float32, 6)
    X.test_set_sort_wait(16, True)
    try:
        X.sort_anchors_carry(dev(a), dev(x))
    finally:
        X.test_set_sort_wait(0, False)
    with pytest.raises(X.LaplexError) as e:
        X.device_status()
    assert e.value.status == X.ETIMEOUT
    X.device_status()
    check_carry(a, x)
