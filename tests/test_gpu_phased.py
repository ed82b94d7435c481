"""GPU parity of laplex_matvec_phased and laplex_gram against the fp64 oracle.
Normaliser: the unphased K0|v| (and K0 K0|v| for the Gram operator)."""
import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


def _i32(p):
    return dev(p.astype(np.int32))


def phased_sym(a, phi, v):
    s, p = O.stable_sort(a)
    return host(X.matvec_phased(dev(s.astype(a.dtype)), dev(phi), dev(v), pa=_i32(p)))


def gram_sym(a, v, phi=None, D=None):
    s, p = O.stable_sort(a)
    return host(X.gram(dev(s.astype(a.dtype)), dev(v), pa=_i32(p),
                       phi=None if phi is None else dev(phi), D=None if D is None else dev(D)))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 2, 7, 2048, 2049, 65537])
def test_phased_sym_sizes(n, dtype):
    a, phi, v = synth.phased_image(n, hi=float(n), seed=n, dtype=dtype)
    assert_close(phased_sym(a, phi, v), O.phased(a, phi, v), O.norm_sym(a, v), dtype, f"n={n}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("B", [2, 3, 4, 5])
def test_phased_sym_columns(B, dtype):
    n = 20000
    a, phi, _ = synth.phased_image(n, hi=2000.0, seed=B, dtype=dtype)
    v = np.random.default_rng(B).normal(size=(n, B)).astype(dtype)
    ref = np.stack([O.phased(a, phi, v[:, c]) for c in range(B)], axis=1)
    assert_close(phased_sym(a, phi, v), ref, O.norm_sym(a, v), dtype, f"B={B}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_phased_general_and_transpose(dtype):
    n, k = 30001, 20011
    a, b, x, w = synth.general_ties(n, k, 0.0, 3000.0, seed=3, dtype=dtype)
    rng = np.random.default_rng(3)
    phi = rng.uniform(0, 2 * np.pi, n).astype(dtype)
    psi = rng.uniform(0, 2 * np.pi, k).astype(dtype)
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    y = host(X.matvec_phased(dev(sa.astype(dtype)), dev(phi), dev(x), pa=_i32(pa),
                             sb=dev(sb.astype(dtype)), psi=dev(psi), pb=_i32(pb)))
    assert_close(y, O.phased(a, phi, x, b, psi), O.norm_general(a, b, x), dtype, "K x",
                 O.far_mass(a, x, b))
    z = host(X.matvec_phased(dev(sa.astype(dtype)), dev(phi), dev(w), pa=_i32(pa),
                             sb=dev(sb.astype(dtype)), psi=dev(psi), pb=_i32(pb), transpose=True))
    assert_close(z, O.phased_T(a, phi, w, b, psi), O.norm_general(b, a, w), dtype, "K^T w",
                 O.far_mass(b, w, a))


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_gram_variants(dtype):
    n = 40009
    a, phi, v = synth.phased_image(n, hi=4000.0, seed=9, dtype=dtype)
    D = synth.uniform(n, 0.5, 2.0, seed=9, stream="D", dtype=dtype)
    assert_close(gram_sym(a, v), O.gram(a, v), O.norm_gram(a, v), dtype, "Gram")
    assert_close(gram_sym(a, v, D=D), O.gram(a, v, D=D), O.norm_gram(a, v, D), dtype, "Gram D")
    assert_close(gram_sym(a, v, phi=phi), O.gram(a, v, phi=phi), O.norm_gram(a, v), dtype,
                 "Gram phased")
    assert_close(gram_sym(a, v, phi=phi, D=D), O.gram(a, v, phi=phi, D=D), O.norm_gram(a, v, D),
                 dtype, "Gram phased D")
    # general Gram: K^T diag(D) K v with v on the b side
    k = 25013
    _, b, x, _ = synth.general_ties(n, k, 0.0, 4000.0, seed=10, dtype=dtype)
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    z = host(X.gram(dev(sa.astype(dtype)), dev(x), pa=_i32(pa), D=dev(D), sb=dev(sb.astype(dtype)),
                    pb=_i32(pb)))
    assert_close(z, O.gram(a, x, D=D, b=b), O.norm_gram(a, x, D, b=b), dtype, "general Gram")


def test_c4_full_size():
    """n = 3*1024*1024, a ~ U(0, 3e6), phi ~ U(0, 2 pi), v ~ N(0,1): y = K v and the
    Gram product K^T K v, every output against the oracle."""
    a, phi, v = synth.phased_image(seed=0)
    assert_close(phased_sym(a, phi, v), O.phased(a, phi, v), O.norm_sym(a, v), np.float32, "C4 Kv")
    assert_close(gram_sym(a, v, phi=phi), O.gram(a, v, phi=phi), O.norm_gram(a, v), np.float32,
                 "C4 K^T K v")
