"""GPU parity of the plan path (sort once, then move vectors into and out of
sorted order by bucketed scatters):

- laplex_permute, dst[idx[i]] = src[i], bit for bit against numpy's indexed
  assignment of the same definition, for 4- and 8-byte elements, with no digit
  pass (one group of outputs), one pass and two passes over the group number,
  and at the group-size boundaries;
- laplex_invert_perm, inv[perm[r]] = r, bit for bit;
- entries of idx outside [0, n) are skipped and leave dst untouched there;
- laplex_matvec_sym_planned against the fp64 oracle (the recurrences on the
  oracle's own stable sort), criterion max_i |y_i - y_ref_i| / (K0|x|)_i within
  1e-4 (fp32, terms below FLT_MIN may vanish) or 1e-10 (fp64)."""
import numpy as np
import pytest
import torch

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu

UINT = {4: np.uint32, 8: np.uint64}


def values(n, dtype, seed):
    rng = np.random.default_rng(seed)
    if np.dtype(dtype).kind == "i":
        return rng.integers(-2**31, 2**31 - 1, size=n).astype(dtype)
    return rng.normal(size=n).astype(dtype)


@pytest.mark.parametrize("dtype", [np.float32, np.float64, np.int32])
@pytest.mark.parametrize("n", [1, 2, 1000, 4097, 8192, 8193, 16384, 16385, (1 << 20) + 3, (1 << 24) + 13])
def test_permute_bit_exact(n, dtype):
    rng = np.random.default_rng(n)
    idx = rng.permutation(n).astype(np.int32)
    src = values(n, dtype, n + 1)
    got = host(X.permute(dev(src), dev(idx)))
    ref = np.empty_like(src)
    ref[idx] = src
    u = UINT[src.itemsize]
    assert np.array_equal(got.view(u), ref.view(u))


@pytest.mark.parametrize("n", [1, 3, 5000, (1 << 22) + 1, (1 << 25) + 7])
def test_invert_perm(n):
    perm = np.random.default_rng(n).permutation(n).astype(np.int32)
    inv = host(X.invert_perm(dev(perm)))
    ref = np.empty(n, dtype=np.int32)
    ref[perm] = np.arange(n, dtype=np.int32)
    assert np.array_equal(inv, ref)


@pytest.mark.parametrize("n", [1000, (1 << 24) + 13])
def test_permute_skips_out_of_range(n):
    rng = np.random.default_rng(7)
    idx = rng.permutation(n).astype(np.int32)
    bad = rng.choice(n, size=min(50, n // 4), replace=False)
    idx[bad[: len(bad) // 2]] = -1 - bad[: len(bad) // 2].astype(np.int32)
    idx[bad[len(bad) // 2:]] = n + bad[len(bad) // 2:].astype(np.int32)
    src = values(n, np.float32, 3)
    out = torch.full((n,), 7.5, dtype=torch.float32, device="cuda")
    got = host(X.permute(dev(src), dev(idx), out=out))
    ref = np.full(n, 7.5, dtype=np.float32)
    ok = (idx >= 0) & (idx < n)
    ref[idx[ok]] = src[ok]
    assert np.array_equal(got.view(np.uint32), ref.view(np.uint32))


def planned(a, x):
    s, perm = O.stable_sort(a)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(a.size)
    y = X.matvec_sym_planned(dev(s.astype(a.dtype)), dev(perm.astype(np.int32)), dev(inv.astype(np.int32)),
                             dev(x))
    return host(y)


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_planned_c1_against_dense(dtype):
    a, x = synth.sym_uniform(4096, 0.0, 64.0, seed=0, dtype=dtype)
    assert_close(planned(a, x), O.dense_matvec(a, x), O.norm_sym(a, x), dtype, "C1 planned")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [5, 300001])
def test_planned_sizes(n, dtype):
    a, x = synth.sym_uniform(n, -50.0, 50.0, seed=n, dtype=dtype)
    assert_close(planned(a, x), O.sym(a, x), O.norm_sym(a, x), dtype, f"n={n}",
                 slack=O.far_mass(a, x))


def test_planned_c2_full_size():
    """n = 2^24, a ~ N(0, 2000^2) unsorted: both moves take the bucketed path."""
    n = 1 << 24
    a, x = synth.sym_normal(n, 2000.0, B=1, seed=0)
    assert_close(planned(a, x), O.sym(a, x), O.norm_sym(a, x), np.float32, "C2 planned",
                 slack=O.far_mass(a, x))


def test_planned_equals_perm_path():
    """The plan path and the perm argument of laplex_matvec_sym compute the same
    sums (same kernels on the same sorted data)."""
    n = 1 << 22
    a, x = synth.sym_uniform(n, 0.0, float(n), seed=5)
    s, perm = O.stable_sort(a)
    inv = np.empty_like(perm)
    inv[perm] = np.arange(n)
    s_d, p_d = dev(s.astype(np.float32)), dev(perm.astype(np.int32))
    y_plan = host(X.matvec_sym_planned(s_d, p_d, dev(inv.astype(np.int32)), dev(x)))
    y_perm = host(X.matvec_sym(s_d, dev(x), p_d))
    assert_close(y_plan, y_perm, O.norm_sym(a, x), np.float32, "plan vs perm", slack=O.far_mass(a, x))
