"""GPU parity of laplex_sort_anchors: the permutation must equal, bit for bit,
the oracle's stable sort (ascending, ties by index, -0.0 equal to +0.0), and the
sorted values must equal a[perm] with -0.0 stored as +0.0."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import dev, host

pytestmark = pytest.mark.gpu


def gpu_sort(a):
    s, p = X.sort_anchors(dev(a))
    X.device_status()
    return host(s), host(p)


def check_exact(a):
    s, p = gpu_sort(a)
    _, ref = O.stable_sort(a)
    assert np.array_equal(p, ref.astype(np.int32))
    expect = a[ref] + a.dtype.type(0)  # -0.0 + 0.0 = +0.0
    ui = np.uint32 if a.dtype == np.float32 else np.uint64
    assert np.array_equal(s.view(ui), expect.view(ui))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 2, 3, 100, 2047, 2048, 4095, 4096, 4097, 65536, (1 << 20) + 7])
def test_sizes(n, dtype):
    check_exact(synth.normal(n, 0.0, 100.0, seed=n, stream="a", dtype=dtype))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_special_values_and_ties(dtype):
    rng = np.random.default_rng(3)
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-40, -1e-40, 1.0, -1.0, 3.4e38, -3.4e38,
                         2.0 ** -126, -(2.0 ** -126)], dtype=np.float64)
    for n in (37, 5000, 300000):
        a = rng.choice(specials, size=n).astype(dtype)
        check_exact(a)
    check_exact(np.round(rng.normal(size=200000) * 3).astype(dtype))   # heavy ties
    check_exact(np.full(100000, -2.5, dtype=dtype))                      # one value
    check_exact(np.arange(100000, 0, -1).astype(dtype))                  # reversed
    check_exact(np.arange(100000).astype(dtype))                         # already sorted


def test_non_finite_reported():
    for bad in (np.nan, np.inf, -np.inf):
        a = np.linspace(0, 1, 10000).astype(np.float32)
        a[1234] = bad
        X.sort_anchors(dev(a))
        with pytest.raises(X.LaplexError) as e:
            X.device_status()
        assert e.value.status == X.ENONFINITE
    X.device_status()  # cleared after being reported


def test_c2_full_size_exact():
    """n = 2^24, a ~ N(0, 2000^2): the permutation against the oracle, bit for bit."""
    check_exact(synth.normal(1 << 24, 0.0, 2000.0, seed=0, stream="a"))


def test_c5_full_size_properties():
    """n = 2^30, a ~ U(0, 2^30) (fp32 rounding makes ~64-way ties): perm is a
    permutation, a[perm] is non-decreasing, ties are in ascending index order and
    sorted == a[perm].  These properties define the stable order uniquely."""
    n = 1 << 30
    a = synth.uniform(n, 0.0, float(1 << 30), seed=0, stream="a")
    s, p = gpu_sort(a)
    seen = np.zeros(n, dtype=np.bool_)
    seen[p] = True
    assert seen.all()
    del seen
    ap = a[p]
    assert np.array_equal(ap.view(np.uint32), s.view(np.uint32))
    d = np.diff(ap)
    assert (d >= 0).all()
    tie = d == 0
    assert (np.diff(p)[tie] > 0).all()


def test_expired_wait_reports_timeout():
    """A look-back wait that runs out ends with LAPLEX_ETIMEOUT in the device
    status instead of hanging: the test hook makes every look-back record count
    as unwritten and bounds each wait at 16 polls.  The status is cleared once
    reported, and the next sort (default bound) is exact again."""
    a = synth.normal(100_000, 0.0, 100.0, seed=5, stream="a")
    X.test_set_sort_wait(16, True)
    try:
        X.sort_anchors(dev(a))
    finally:
        X.test_set_sort_wait(0, False)
    with pytest.raises(X.LaplexError) as e:
        X.device_status()
    assert e.value.status == X.ETIMEOUT
    X.device_status()
    check_exact(a)
