"""GPU parity of laplex_backward_phased: the gradients of L = <g, K x> with
K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j) in x, the phases and the anchors,
against the fp64 oracle (oracle.backward_phased).  Normalisers, term by term with
|cos|, |sin| <= 1: K0^T|g| for dx, |g| K0|x| for dphi and da, |x| K0^T|g| for dpsi
and db (symmetric case: |g| K0|x| + |x| K0|g| for the totals).  fp32 slack: the
oracle's mass of the terms below FLT_MIN (oracle.far_mass)."""
import math

import numpy as np
import pytest

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close, dev, host

pytestmark = pytest.mark.gpu


def _phases(m, seed, stream, dtype):
    return synth.uniform(m, 0.0, 2 * math.pi, seed=seed, stream=stream, dtype=dtype)


def run_general(a, phi, b, psi, x, g, use_perm):
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    sa, sb = sa.astype(a.dtype), sb.astype(b.dtype)
    if use_perm:
        outs = X.backward_phased(dev(sa), dev(phi), dev(x), dev(g), pa=dev(pa.astype(np.int32)),
                                 sb=dev(sb), psi=dev(psi), pb=dev(pb.astype(np.int32)))
        return [host(t) for t in outs]
    dx, dphi, dpsi, da, db = [host(t) for t in X.backward_phased(dev(sa), dev(phi[pa]), dev(x[pb]),
                                                                 dev(g[pa]), sb=dev(sb), psi=dev(psi[pb]))]
    res = [np.empty_like(dx), np.empty_like(dphi), np.empty_like(dpsi), np.empty_like(da), np.empty_like(db)]
    res[0][pb], res[1][pa], res[2][pb], res[3][pa], res[4][pb] = dx, dphi, dpsi, da, db
    return res


def check_general(a, phi, b, psi, x, g, dtype, what):
    ref = O.backward_phased(a, phi, x, g, b=b, psi=psi)
    ndx, nda, ndb = O.norm_backward_phased(a, x, g, b=b)
    mg_b, mx_a = O.far_mass(b, g, a), O.far_mass(a, x, b)
    sa_slack, sb_slack = np.abs(g) * mx_a, np.abs(x) * mg_b
    for use_perm in (True, False):
        got = run_general(a, phi, b, psi, x, g, use_perm)
        for name, y, r, nrm, sl in zip(("dx", "dphi", "dpsi", "da", "db"), got, ref,
                                       (ndx, nda, ndb, nda, ndb), (mg_b, sa_slack, sb_slack, sa_slack, sb_slack)):
            assert_close(y, r, nrm, dtype, f"{what} {name} perm={use_perm}", sl)


def check_sym(a, phi, x, g, dtype, what):
    rdx, rdphi, rda = O.backward_phased(a, phi, x, g)
    ndx, ntot = O.norm_backward_phased(a, x, g)
    mg, mx = O.far_mass(a, g), O.far_mass(a, x)
    tslack = np.abs(g) * mx + np.abs(x) * mg
    s, p = O.stable_sort(a)
    s = s.astype(a.dtype)
    dx, dphi, da = [host(t) for t in X.backward_phased(dev(s), dev(phi), dev(x), dev(g),
                                                       pa=dev(p.astype(np.int32)))]
    assert_close(dx, rdx, ndx, dtype, f"{what} dx", mg)
    assert_close(dphi, rdphi, ntot, dtype, f"{what} dphi", tslack)
    assert_close(da, rda, ntot, dtype, f"{what} da", tslack)


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n,k", [(1, 1), (1, 5), (5, 1), (3, 2), (100, 37), (2047, 2049),
                                 (4097, 100), (100, 4097), (30011, 50021)])
def test_general_sizes(n, k, dtype):
    """a, b ~ U(-50, 50) with 1 % of b equal to entries of a (ties, sign 0);
    phases ~ U(0, 2 pi).  Sizes span one to many scan tiles with ragged tails."""
    a, b, x, _ = synth.general_ties(n, k, -50.0, 50.0, seed=n + k, dtype=dtype)
    g = np.random.default_rng(n * 7 + k).normal(size=n).astype(dtype)
    phi, psi = _phases(n, n + k, "phi", dtype), _phases(k, n + k, "psi", dtype)
    check_general(a, phi, b, psi, x, g, dtype, f"n={n} k={k}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
@pytest.mark.parametrize("n", [1, 2, 777, 2048, 5000, 40000])
def test_sym_sizes(n, dtype):
    """Symmetric case: a ~ U(0, n) (spacing about 1), phases ~ U(0, 2 pi)."""
    a, phi, x = synth.phased_image(n, hi=float(n), seed=n, dtype=dtype)
    g = np.random.default_rng(n).normal(size=n).astype(dtype)
    check_sym(a, phi, x, g, dtype, f"sym n={n}")


@pytest.mark.parametrize("dtype", [np.float32, np.float64])
def test_edge_cases(dtype):
    rng = np.random.default_rng(29)
    x = rng.normal(size=3000).astype(dtype)
    g = rng.normal(size=2000).astype(dtype)
    a = rng.uniform(0, 10, 2000).astype(dtype)
    phi = rng.uniform(0, 6.3, 2000).astype(dtype)
    psi = rng.uniform(0, 6.3, 3000).astype(dtype)
    check_general(a, phi, rng.uniform(40, 60, 3000).astype(dtype), psi, x, g, dtype, "b right")
    check_general(a, phi, rng.uniform(-30, -20, 3000).astype(dtype), psi, x, g, dtype, "b left")
    check_general(np.full(2000, 1.5, dtype=dtype), phi, np.full(3000, 1.5, dtype=dtype), psi, x, g, dtype,
                  "all tied")
    check_sym(np.full(2000, -3.0, dtype=dtype), phi, g, g[::-1].copy(), dtype, "sym all tied")
    # zero phases: the unphased general backward
    z = np.zeros(2000, dtype=dtype)
    b = rng.uniform(0, 10, 3000).astype(dtype)
    _, _, _, da, db = run_general(a, z, b, np.zeros(3000, dtype=dtype), x, g, True)
    sa, pa = O.stable_sort(a)
    sb, pb = O.stable_sort(b)
    _, da0, db0 = (host(t) for t in X.backward_general(dev(sa.astype(dtype)), dev(sb.astype(dtype)), dev(x),
                                                         dev(g), dev(pa.astype(np.int32)), dev(pb.astype(np.int32))))
    _, nda, ndb = O.norm_backward_general(a, b, x, g)
    assert_close(da, da0, nda, dtype, "phi = 0 da", np.abs(g) * O.far_mass(a, x, b))
    assert_close(db, db0, ndb, dtype, "phi = 0 db", np.abs(x) * O.far_mass(b, g, a))


def test_null_outputs_and_empty_sides():
    """Outputs left NULL are not written; n = 0 or k = 0 gives zeros on the other side."""
    import torch
    rng = np.random.default_rng(5)
    a, b = rng.uniform(0, 20, 300).astype(np.float32), rng.uniform(0, 20, 200).astype(np.float32)
    sa, sb = np.sort(a), np.sort(b)
    phi, psi = rng.uniform(0, 6, 300).astype(np.float32), rng.uniform(0, 6, 200).astype(np.float32)
    x, g = rng.normal(size=200).astype(np.float32), rng.normal(size=300).astype(np.float32)
    ref = O.backward_phased(sa, phi, x, g, b=sb, psi=psi)
    norms = O.norm_backward_phased(sa, x, g, b=sb)
    D = [dev(v) for v in (sa, phi, sb, psi, x, g)]
    sentinel = 1234.5
    outs = [torch.full((m,), sentinel, dtype=torch.float32, device="cuda") for m in (200, 300, 200, 300, 200)]
    keep = (True, False, True, False, True)
    ptr = [X._ptr(o) if k else None for o, k in zip(outs, keep)]
    ws, nb = X._ws(X.OP_BACKWARD_PHASED, 300, 200, 1, torch.float32, torch.device("cuda"))
    P = X._ptr
    X._check(X.lib().laplex_backward_phased(P(D[0]), None, P(D[1]), 300, P(D[2]), None, P(D[3]), 200, P(D[4]),
                                            P(D[5]), *ptr, 0, P(ws), nb, X._stream(torch.device("cuda"))))
    got = [host(o) for o in outs]
    for i, (k, nrm) in enumerate(zip(keep, (norms[0], norms[1], norms[2], norms[1], norms[2]))):
        if k:
            assert_close(got[i], ref[i], nrm, np.float32, f"output {i}")
        else:
            assert np.all(got[i] == sentinel), i
    e = np.zeros(0, np.float32)
    dx, dphi, dpsi, da, db = X.backward_phased(dev(e), dev(e), dev(x), dev(e), sb=dev(sb), psi=dev(psi))
    assert np.all(host(dx) == 0) and np.all(host(dpsi) == 0) and np.all(host(db) == 0)
    dx, dphi, dpsi, da, db = X.backward_phased(dev(sa), dev(phi), dev(e), dev(g), sb=dev(e), psi=dev(e))
    assert np.all(host(dphi) == 0) and np.all(host(da) == 0) and host(dx).size == 0


def test_c3_full_size_phased():
    """The general workload with phases: a in R^(2^22), b in R^(2^20) ~ U(-1000, 1000),
    1 % ties, phases ~ U(0, 2 pi), x ~ N(0, 1) on b, g ~ N(0, 1) on a."""
    a, b, x, g = synth.general_ties(1 << 22, 1 << 20, -1000.0, 1000.0, seed=0)
    phi, psi = _phases(1 << 22, 0, "phi", np.float32), _phases(1 << 20, 0, "psi", np.float32)
    check_general(a, phi, b, psi, x, g, np.float32, "C3 phased")


def test_c4_full_size_sym():
    """The phased workload, symmetric: n = 3 * 1024^2, a ~ U(0, 3e6), phi ~ U(0, 2 pi),
    x = v ~ N(0, 1), g ~ N(0, 1)."""
    a, phi, v = synth.phased_image(seed=0)
    g = synth.normal(a.size, seed=0, stream="g")
    check_sym(a, phi, v, g, np.float32, "C4 sym")
