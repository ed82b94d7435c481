"""Pins of the CPU oracle to facts other than itself (no GPU needed).

Each test ties an oracle route to something it does not compute the same way:
hand-worked examples (tests/golden/hand_examples.json), textbook closed forms
(the Ornstein-Uhlenbeck tridiagonal inverse, the Kac-Murdock-Szego Toeplitz
matrix through scipy), invariants of the definition, brute force on tiny inputs,
and central finite differences.  The sources are the LAPLEX technical summaries
("Riepilogo Tecnico: LAPLEX - La FFT dei Nuclei di Laplace Apprendibili" and its
French twin), cited by section.
"""
import json
import math
import os

import numpy as np
import pytest
import scipy.linalg

import oracle as O
from exact_laplace_b200 import synth

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "hand_examples.json")
NS = {"exp": math.exp, "cos": math.cos, "sin": math.sin, "pi": math.pi, "__builtins__": {}}


def ev(e):
    return float(eval(e, NS)) if isinstance(e, str) else float(e)


def _examples():
    with open(GOLDEN) as f:
        return json.load(f)["examples"]


@pytest.mark.parametrize("ex", _examples(), ids=lambda e: e["name"])
def test_hand_examples(ex):
    a = [ev(v) for v in ex["a"]]
    op = ex["op"]
    if op == "sort":
        s, perm = O.stable_sort(np.array(a))
        assert perm.tolist() == ex["expect_perm"]
        return
    x = [ev(v) for v in ex["x"]]
    if op == "backward":
        g = [ev(v) for v in ex["g"]]
        dx, da = O.backward(a, x, g)
        dxd, dad = O.dense_backward(a, x, g)
        np.testing.assert_allclose(dx, [ev(e) for e in ex["expect_dx"]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(da, [ev(e) for e in ex["expect_da"]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(dxd, [ev(e) for e in ex["expect_dx"]], rtol=0, atol=1e-14)
        np.testing.assert_allclose(dad, [ev(e) for e in ex["expect_da"]], rtol=0, atol=1e-14)
        return
    exp = np.array([ev(e) for e in ex["expect"]])
    if "decimal" in ex:  # the closed forms agree with the printed decimals
        np.testing.assert_allclose(exp, ex["decimal"], rtol=0, atol=6e-9)
    if op == "sym":
        outs = [O.sym(a, x), O.dense_matvec(a, x)]
    elif op == "phased":
        phi = [ev(v) for v in ex["phi"]]
        outs = [O.phased(a, phi, x), O.dense_matvec(a, x, phi=phi)]
    elif op == "gram_phased":
        phi = [ev(v) for v in ex["phi"]]
        K = O.dense_matrix(a, phi=phi)
        outs = [O.gram(a, x, phi=phi), K.T @ (K @ np.array(x))]
    elif op == "general":
        b = [ev(v) for v in ex["b"]]
        outs = [O.general(a, b, x), O.dense_matvec(a, x, b=b)]
    elif op == "general_T":
        b = [ev(v) for v in ex["b"]]
        outs = [O.general_T(a, b, x), O.dense_matrix(a, b).T @ np.array(x)]
    else:
        raise AssertionError(op)
    for y in outs:
        np.testing.assert_allclose(y, exp, rtol=0, atol=1e-14)


# ---------------------------------------------------------------------------
# closed forms
# ---------------------------------------------------------------------------

def _ou_precision(s):
    """Tridiagonal inverse of K_ij = exp(-|s_i - s_j|) for distinct ascending s: the
    covariance of an Ornstein-Uhlenbeck process sampled at s is Markov, so its
    precision matrix is tridiagonal with rho_i = exp(-(s_{i+1} - s_i)):
    Q_{i,i+1} = -rho_i / (1 - rho_i^2),
    Q_ii = 1 + rho_{i-1}^2 / (1 - rho_{i-1}^2) + rho_i^2 / (1 - rho_i^2)."""
    n = len(s)
    rho = np.exp(-np.diff(s))
    off = -rho / (1 - rho ** 2)
    t = rho ** 2 / (1 - rho ** 2)
    diag = np.ones(n)
    diag[1:] += t
    diag[:-1] += t
    return diag, off


@pytest.mark.parametrize("n,seed", [(2, 0), (7, 1), (200, 2), (3000, 3)])
def test_ou_tridiagonal_inverse(n, seed):
    rng = np.random.default_rng(seed)
    s = np.cumsum(rng.uniform(0.05, 2.0, size=n))
    x = rng.normal(size=n)
    y = O.sym_sorted(s, x)
    diag, off = _ou_precision(s)
    back = diag * y
    back[:-1] += off * y[1:]
    back[1:] += off * y[:-1]
    np.testing.assert_allclose(back, x, rtol=0, atol=1e-10 * max(1.0, np.abs(x).max()))


@pytest.mark.parametrize("n,h", [(1, 0.3), (64, 0.01), (512, 0.7)])
def test_uniform_grid_is_kms_toeplitz(n, h):
    """Anchors on a uniform grid make K the Toeplitz matrix rho^|i-j| (IT §2.3,
    relation with the FFT); scipy builds it independently."""
    rng = np.random.default_rng(n)
    s = 5.0 + h * np.arange(n)
    x = rng.normal(size=(n, 3))
    T = scipy.linalg.toeplitz(np.exp(-h) ** np.arange(n))
    np.testing.assert_allclose(O.sym_sorted(s, x), T @ x, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(O.sym(s[::-1].copy(), x[::-1]), (T @ x)[::-1], rtol=1e-12, atol=1e-12)


def test_unit_vectors_give_columns():
    rng = np.random.default_rng(5)
    a = rng.normal(size=40) * 2
    a[[3, 9]] = a[17]
    for i in (0, 3, 17, 39):
        e = np.zeros(40)
        e[i] = 1
        np.testing.assert_allclose(O.sym(a, e), np.exp(-np.abs(a - a[i])), rtol=0, atol=1e-15)


def test_all_equal_anchors_sum():
    x = np.random.default_rng(1).normal(size=(33, 2))
    y = O.sym(np.full(33, 7.25), x)
    np.testing.assert_allclose(y, np.broadcast_to(x.sum(0), y.shape), rtol=1e-13)


def test_far_apart_anchors_identity():
    rng = np.random.default_rng(2)
    a = rng.permutation(np.arange(20) * 800.0)
    x = rng.normal(size=20)
    assert np.array_equal(O.sym(a, x), x)


def test_temperature_zero_permutation_limit():
    """IT §2.3 / §2.1: as t -> 0, exp(-|a_i - b_j| / t) tends to the equality routing
    matrix; with b = a[pi] and distinct anchors, K x -> P x, (K x)_i = x_{pi^-1(i)}."""
    rng = np.random.default_rng(3)
    n = 50
    a = rng.permutation(np.linspace(-3, 3, n))
    pi = rng.permutation(n)
    b = a[pi]
    x = rng.normal(size=n)
    t = (6 / (n - 1)) / 800  # every off-equality term is exp(-800): exactly 0 in fp64
    y = O.general(a / t, b / t, x)
    inv = np.empty(n, dtype=int)
    inv[pi] = np.arange(n)
    np.testing.assert_array_equal(y, x[inv])


# ---------------------------------------------------------------------------
# invariants
# ---------------------------------------------------------------------------

def test_symmetry_translation_reflection_permutation():
    rng = np.random.default_rng(4)
    a = rng.normal(size=300) * 10
    a[::7] = a[1]
    u, v = rng.normal(size=300), rng.normal(size=300)
    Ku, Kv = O.sym(a, u), O.sym(a, v)
    assert abs(u @ Kv - Ku @ v) < 1e-10 * np.abs(u).sum() * np.abs(Kv).max()
    np.testing.assert_allclose(O.sym(a + 123.5, v), Kv, rtol=1e-9)
    np.testing.assert_allclose(O.sym(-a, v), Kv, rtol=1e-12)
    p = rng.permutation(300)
    np.testing.assert_allclose(O.sym(a[p], v[p]), Kv[p], rtol=1e-12)


def test_general_reduces_to_symmetric_and_transpose_identity():
    rng = np.random.default_rng(6)
    a = rng.uniform(-5, 5, size=120)
    b = rng.uniform(-5, 5, size=77)
    b[:10] = a[20:30]
    x, w = rng.normal(size=77), rng.normal(size=120)
    np.testing.assert_allclose(O.general(a, a, w), O.sym(a, w), rtol=1e-12, atol=1e-12)
    assert abs(w @ O.general(a, b, x) - O.general_T(a, b, w) @ x) < 1e-10


def test_phased_reduces_and_matches_definition():
    rng = np.random.default_rng(7)
    a = rng.uniform(0, 20, size=90)
    b = rng.uniform(0, 20, size=60)
    phi, psi = rng.uniform(0, 2 * np.pi, 90), rng.uniform(0, 2 * np.pi, 60)
    v, x = rng.normal(size=90), rng.normal(size=60)
    np.testing.assert_allclose(O.phased(a, np.zeros(90), v), O.sym(a, v), rtol=1e-13, atol=1e-13)
    np.testing.assert_allclose(O.phased(a, phi, v), O.dense_matvec(a, v, phi=phi), atol=1e-12)
    np.testing.assert_allclose(O.phased(a, phi, x, b, psi),
                               O.dense_matvec(a, x, b=b, phi=phi, psi=psi), atol=1e-12)
    # a common phase shift cancels in cos(phi_j - phi_k)
    np.testing.assert_allclose(O.phased(a, phi + 1.0, v), O.phased(a, phi, v), atol=1e-12)


def test_gram_is_psd_and_composes():
    rng = np.random.default_rng(8)
    a = rng.uniform(0, 30, size=150)
    phi = rng.uniform(0, 2 * np.pi, 150)
    D = rng.uniform(0.5, 2, 150)
    v = rng.normal(size=150)
    K = O.dense_matrix(a, phi=phi)
    z = O.gram(a, v, phi=phi, D=D)
    np.testing.assert_allclose(z, K.T @ (D * (K @ v)), atol=1e-11)
    assert v @ z >= 0
    np.testing.assert_allclose(v @ z, np.sum(D * (K @ v) ** 2), rtol=1e-10)
    b = rng.uniform(0, 30, size=70)
    w = rng.normal(size=70)
    Kg = O.dense_matrix(a, b)
    np.testing.assert_allclose(O.gram(a, w, b=b), Kg.T @ (Kg @ w), atol=1e-10)


def test_normaliser_bounds():
    rng = np.random.default_rng(9)
    a = rng.uniform(0, 10, size=80)
    phi = rng.uniform(0, 6, 80)
    x = rng.normal(size=80)
    nrm = O.norm_sym(a, x)
    assert np.all(np.abs(O.sym(a, x)) <= nrm + 1e-12)
    assert np.all(np.abs(O.phased(a, phi, x)) <= nrm + 1e-12)


# ---------------------------------------------------------------------------
# brute force / dense agreement of the sequential routes
# ---------------------------------------------------------------------------

@pytest.mark.parametrize("n,B,ties", [(0, 1, False), (1, 1, False), (2, 3, True), (3, 1, True),
                                      (17, 2, True), (257, 1, False), (1000, 4, True)])
def test_sequential_matches_dense(n, B, ties):
    rng = np.random.default_rng(n + B)
    a = rng.normal(size=n) * (n ** 0.5 + 1)
    if ties and n > 1:
        a[rng.integers(0, n, n // 3 + 1)] = a[0]
        a = np.round(a, 0)
    x = rng.normal(size=(n, B))
    np.testing.assert_allclose(O.sym(a, x), O.dense_matvec(a, x), rtol=1e-12, atol=1e-12)
    k = max(1, n // 2 + 3)
    b = np.round(rng.normal(size=k) * (n ** 0.5 + 1), 1)
    if n:
        b[: k // 4] = a[rng.integers(0, n, k // 4)]
    xb = rng.normal(size=(k, B))
    np.testing.assert_allclose(O.general(a, b, xb), O.dense_matvec(a, xb, b=b), rtol=1e-12, atol=1e-12)


def test_rows_window_matches_dense_rows():
    rng = np.random.default_rng(11)
    n = 2000
    a = rng.uniform(0, 3000, size=n)
    a[::5] = np.round(a[::5])
    phi = rng.uniform(0, 2 * np.pi, n)
    x = rng.normal(size=(n, 2))
    s, perm = O.stable_sort(a)
    rowsel = rng.integers(0, n, 50)
    out, sgn, absn = O.rows(a[rowsel], s, x[perm])
    K = O.dense_matrix(a)
    np.testing.assert_allclose(out, (K @ x)[rowsel], atol=1e-12)
    np.testing.assert_allclose(absn, (K @ np.abs(x))[rowsel], atol=1e-12)
    S = np.sign(a[:, None] - a[None, :]) * K
    np.testing.assert_allclose(sgn, (S @ x)[rowsel], atol=1e-12)
    outp, _, _ = O.rows(a[rowsel], s, x[perm, 0], rphi=phi[rowsel], spsi=phi[perm])
    np.testing.assert_allclose(outp, O.dense_matvec(a, x[:, 0], phi=phi)[rowsel], atol=1e-12)


def test_sort_matches_brute_force_comparator():
    rng = np.random.default_rng(12)
    specials = np.array([0.0, -0.0, 1e-45, -1e-45, 1e-40, 5e-324, -5e-324, 2.0, -2.0], dtype=np.float64)
    for trial in range(20):
        n = int(rng.integers(0, 40))
        a = rng.choice(np.concatenate([specials, rng.normal(size=5)]), size=n)
        a32 = a.astype(np.float32)
        s, perm = O.stable_sort(a32)
        brute = sorted(range(n), key=lambda i: (float(a32[i]), i))
        assert perm.tolist() == brute
        assert np.array_equal(s, a32[perm].astype(np.float64))
    with pytest.raises(ValueError):
        O.stable_sort(np.array([1.0, np.nan]))
    with pytest.raises(ValueError):
        O.stable_sort(np.array([np.inf, 1.0]))


# ---------------------------------------------------------------------------
# backward pass
# ---------------------------------------------------------------------------

def _loss(a, x, g):
    return float(g @ O.dense_matvec(a, x))


@pytest.mark.parametrize("tied", [False, True])
def test_backward_central_differences(tied):
    """Central differences of L = <g, K x>.  At a tie the two one-sided slopes of
    exp(-|t|) are opposite, so the central difference is the sign(0) = 0 value."""
    rng = np.random.default_rng(13 + tied)
    n = 40
    a = rng.uniform(0, 8, size=n)
    if tied:
        a[[4, 11, 30]] = a[2]
    x, g = rng.normal(size=n), rng.normal(size=n)
    dx, da = O.backward(a, x, g)
    h = 1e-6
    fd = np.empty(n)
    for m in range(n):
        ap, am = a.copy(), a.copy()
        ap[m] += h
        am[m] -= h
        fd[m] = (_loss(ap, x, g) - _loss(am, x, g)) / (2 * h)
    np.testing.assert_allclose(da, fd, rtol=0, atol=5e-8 * np.abs(fd).max())
    for m in (0, 7):
        e = np.zeros(n)
        e[m] = 1
        assert abs(dx[m] - (_loss(a, x + e, g) - _loss(a, x, g))) < 1e-10
    assert abs(da.sum()) < 1e-9 * np.abs(da).sum()  # translation invariance of L
    dxd, dad = O.dense_backward(a, x, g)
    np.testing.assert_allclose(dx, dxd, atol=1e-12)
    np.testing.assert_allclose(da, dad, atol=1e-12)


def test_signed_sums_brute_force():
    rng = np.random.default_rng(14)
    s = np.sort(np.round(rng.uniform(0, 6, size=60), 0))
    v = rng.normal(size=(60, 2))
    brute = np.zeros_like(v)
    for i in range(60):
        for j in range(60):
            brute[i] += np.sign(s[i] - s[j]) * math.exp(-abs(s[i] - s[j])) * v[j]
    np.testing.assert_allclose(O.signed_sorted(s, v), brute, atol=1e-13)


# ---------------------------------------------------------------------------
# the mass of the terms below a threshold (parity slack of fp32 results)
# ---------------------------------------------------------------------------

def _far_brute(a, b, v, dist):
    out = np.zeros((len(a),) + v.shape[1:])
    for i in range(len(a)):
        for j in range(len(b)):
            d = abs(a[i] - b[j])
            if d > dist:
                out[i] += math.exp(-d) * np.abs(v[j])
    return out


@pytest.mark.parametrize("dist", [0.0, 0.75, 2.5, 1e9])
def test_far_mass_brute_force(dist):
    """far_mass against the double loop, strict inequality included: b_4 sits
    exactly dist to the right of a_5 and b_9 exactly dist to the left of a_2."""
    rng = np.random.default_rng(16)
    a = np.round(rng.uniform(0, 8, 25), 2)
    b = np.round(rng.uniform(-1, 9, 17), 2)
    if dist < 1e6:
        b[4] = a[5] + dist
        b[9] = a[2] - dist
    for v in (rng.normal(size=17), rng.normal(size=(17, 3))):
        np.testing.assert_allclose(O.far_mass(a, v, b, dist), _far_brute(a, b, v, dist), rtol=1e-12,
                                   atol=1e-300)
    # symmetric form (b = a), with ties
    a2 = np.round(rng.uniform(0, 5, 30), 0)
    v2 = rng.normal(size=30)
    np.testing.assert_allclose(O.far_mass(a2, v2, dist=dist), _far_brute(a2, a2, v2, dist), rtol=1e-12,
                               atol=1e-300)


def test_far_mass_limits():
    """dist = 0 on distinct anchors keeps every term: K|v| by the general-case
    route; dist beyond the spread keeps none; the default threshold is the
    point where exp(-d) crosses the smallest normal fp32 number."""
    rng = np.random.default_rng(17)
    a = rng.uniform(0, 10, 40)
    b = rng.uniform(0, 10, 33) + 0.001
    v = rng.normal(size=33)
    np.testing.assert_allclose(O.far_mass(a, v, b, 0.0), O.general(a, b, np.abs(v)), rtol=1e-12)
    assert np.all(O.far_mass(a, v, b, 50.0) == 0.0)
    assert math.exp(-O.FAR_F32) == pytest.approx(float(np.finfo(np.float32).tiny), rel=1e-13)
    # two anchors 90 apart: each sees the other's term, below FLT_MIN
    m = O.far_mass(np.array([0.0, 90.0]), np.array([2.0, -3.0]))
    np.testing.assert_allclose(m, [3.0 * math.exp(-90.0), 2.0 * math.exp(-90.0)], rtol=1e-14)


# ---------------------------------------------------------------------------
# general-case anchor gradients (learnable a and b)
# ---------------------------------------------------------------------------

def test_signed_general_brute_force():
    """S(a <- b, v) against the double loop with sign(0) = 0: ties between a and
    b, ties inside b, several columns, a and b of different sizes."""
    rng = np.random.default_rng(18)
    a = np.round(rng.uniform(0, 6, 40), 1)
    b = np.concatenate([np.round(rng.uniform(-1, 7, 30), 1), a[:5]])
    v = rng.normal(size=(35, 2))
    brute = np.zeros((40, 2))
    for i in range(40):
        for j in range(35):
            brute[i] += np.sign(a[i] - b[j]) * math.exp(-abs(a[i] - b[j])) * v[j]
    np.testing.assert_allclose(O.signed_general(a, b, v), brute, atol=1e-13)
    # b = a reduces to the symmetric signed sums (a separate C routine)
    s2 = np.sort(np.round(rng.uniform(0, 6, 50), 0))
    v2 = rng.normal(size=50)
    np.testing.assert_allclose(O.signed_general(s2, s2, v2), O.signed_sorted(s2, v2), atol=1e-13)


def _loss_general(a, b, x, g):
    return float(g @ O.dense_matvec(a, x, b=b))


def test_backward_general_central_differences():
    """dx, da, db of L = <g, K(a, b) x> against central differences of the dense
    definition (distinct anchors; a and b interleaved)."""
    rng = np.random.default_rng(19)
    a = rng.uniform(0, 4, 12)
    b = rng.uniform(0, 4, 9)
    x, g = rng.normal(size=9), rng.normal(size=12)
    dx, da, db = O.backward_general(a, b, x, g)
    np.testing.assert_allclose(dx, O.dense_matrix(a, b=b).T @ g, atol=1e-13)
    h = 1e-6
    for i in range(12):
        ap, am = a.copy(), a.copy()
        ap[i] += h
        am[i] -= h
        fd = (_loss_general(ap, b, x, g) - _loss_general(am, b, x, g)) / (2 * h)
        assert abs(da[i] - fd) < 1e-7, i
    for j in range(9):
        bp, bm = b.copy(), b.copy()
        bp[j] += h
        bm[j] -= h
        fd = (_loss_general(a, bp, x, g) - _loss_general(a, bm, x, g)) / (2 * h)
        assert abs(db[j] - fd) < 1e-7, j


# ---------------------------------------------------------------------------
# phased backward (trainable anchors and phases)
# ---------------------------------------------------------------------------

def _loss_phased(a, phi, b, psi, x, g):
    return float(g @ O.dense_matvec(a, x, b=b, phi=phi, psi=psi))


def _cd(f, v, i, h=1e-6):
    vp, vm = v.copy(), v.copy()
    vp[i] += h
    vm[i] -= h
    return (f(vp) - f(vm)) / (2 * h)


def test_backward_phased_central_differences():
    """dx, dphi, dpsi, da, db of L = <g, K x>, K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j),
    against central differences of the dense definition (distinct anchors)."""
    rng = np.random.default_rng(31)
    a, b = rng.uniform(0, 4, 11), rng.uniform(0, 4, 8)
    phi, psi = rng.uniform(0, 2 * math.pi, 11), rng.uniform(0, 2 * math.pi, 8)
    x, g = rng.normal(size=8), rng.normal(size=11)
    dx, dphi, dpsi, da, db = O.backward_phased(a, phi, x, g, b=b, psi=psi)
    np.testing.assert_allclose(dx, O.dense_matrix(a, b, phi, psi).T @ g, atol=1e-13)
    for i in range(11):
        assert abs(dphi[i] - _cd(lambda v: _loss_phased(a, v, b, psi, x, g), phi, i)) < 1e-7, i
        assert abs(da[i] - _cd(lambda v: _loss_phased(v, phi, b, psi, x, g), a, i)) < 1e-7, i
    for j in range(8):
        assert abs(dpsi[j] - _cd(lambda v: _loss_phased(a, phi, b, v, x, g), psi, j)) < 1e-7, j
        assert abs(db[j] - _cd(lambda v: _loss_phased(a, phi, v, psi, x, g), b, j)) < 1e-7, j


def test_backward_phased_pins_reject_planted_mistakes():
    """Plausible slips in the phase and anchor gradients (channels swapped, the
    sine's sign flipped, the sides' phases exchanged), built from the oracle's own
    parts, each fail the central differences of the dense definition."""
    rng = np.random.default_rng(33)
    a, b = rng.uniform(0, 4, 9), rng.uniform(0, 4, 7)
    phi, psi = rng.uniform(0, 2 * math.pi, 9), rng.uniform(0, 2 * math.pi, 7)
    x, g = rng.normal(size=7), rng.normal(size=9)
    xc = np.stack([np.cos(psi) * x, np.sin(psi) * x], axis=1)
    P, S = O.general(a, b, xc), O.signed_general(a, b, xc)
    fd_phi = np.array([_cd(lambda v: _loss_phased(a, v, b, psi, x, g), phi, i) for i in range(9)])
    fd_a = np.array([_cd(lambda v: _loss_phased(v, phi, b, psi, x, g), a, i) for i in range(9)])
    c, s = np.cos(phi), np.sin(phi)
    good_phi = g * (c * P[:, 1] - s * P[:, 0])
    good_a = -g * (c * S[:, 0] + s * S[:, 1])
    assert np.abs(good_phi - fd_phi).max() < 1e-7 and np.abs(good_a - fd_a).max() < 1e-7
    mutants_phi = {
        "channels swapped": g * (c * P[:, 0] - s * P[:, 1]),
        "sine sign flipped": g * (s * P[:, 0] - c * P[:, 1]),
        "cos/sin of the wrong side": g * (np.cos(psi[:1]) * P[:, 1] - np.sin(psi[:1]) * P[:, 0]),
    }
    for name, m in mutants_phi.items():
        assert np.abs(m - fd_phi).max() > 1e-3, name
    mutants_a = {
        "plain sums for signed": -g * (c * P[:, 0] + s * P[:, 1]),
        "sign of the anchor gradient": g * (c * S[:, 0] + s * S[:, 1]),
        "sine combination": -g * (c * S[:, 1] - s * S[:, 0]),
    }
    for name, m in mutants_a.items():
        assert np.abs(m - fd_a).max() > 1e-3, name


def test_backward_phased_ties_and_invariants():
    """Tied anchors: the dense derivative with sign(0) = 0, entry by entry.  A
    common phase shift and a common translation of both anchor sets leave L
    unchanged, so sum dphi + sum dpsi = 0 and sum da + sum db = 0.  The symmetric
    case returns the totals of the general one with b = a, psi = phi, and phi = 0
    reduces it to the unphased backward pass."""
    rng = np.random.default_rng(32)
    a = np.round(rng.uniform(0, 3, 10), 1)
    b = np.concatenate([np.round(rng.uniform(0, 3, 5), 1), a[:3]])
    phi, psi = rng.uniform(-3, 3, 10), rng.uniform(-3, 3, 8)
    x, g = rng.normal(size=8), rng.normal(size=10)
    dx, dphi, dpsi, da, db = O.backward_phased(a, phi, x, g, b=b, psi=psi)
    for i in range(10):
        t_phi = t_a = 0.0
        for j in range(8):
            e = math.exp(-abs(a[i] - b[j]))
            t_phi += -g[i] * e * math.sin(phi[i] - psi[j]) * x[j]
            t_a += -g[i] * np.sign(a[i] - b[j]) * e * math.cos(phi[i] - psi[j]) * x[j]
        assert abs(dphi[i] - t_phi) < 1e-13 and abs(da[i] - t_a) < 1e-13, i
    for j in range(8):
        t_psi = t_b = 0.0
        for i in range(10):
            e = math.exp(-abs(a[i] - b[j]))
            t_psi += x[j] * e * math.sin(phi[i] - psi[j]) * g[i]
            t_b += -x[j] * np.sign(b[j] - a[i]) * e * math.cos(phi[i] - psi[j]) * g[i]
        assert abs(dpsi[j] - t_psi) < 1e-13 and abs(db[j] - t_b) < 1e-13, j
    assert abs(dphi.sum() + dpsi.sum()) < 1e-12
    assert abs(da.sum() + db.sum()) < 1e-12
    xs = rng.normal(size=10)
    sdx, sdphi, sda = O.backward_phased(a, phi, xs, g)
    gdx, gdphi, gdpsi, gda, gdb = O.backward_phased(a, phi, xs, g, b=a, psi=phi)
    np.testing.assert_allclose(sdx, gdx, atol=1e-13)
    np.testing.assert_allclose(sdphi, gdphi + gdpsi, atol=1e-13)
    np.testing.assert_allclose(sda, gda + gdb, atol=1e-13)
    udx, uda = O.backward(a, xs, g)
    zdx, zdphi, zda = O.backward_phased(a, np.zeros(10), xs, g)
    np.testing.assert_allclose(zdx, udx, atol=1e-13)
    np.testing.assert_allclose(zda, uda, atol=1e-13)
    assert np.abs(zdphi).max() < 1e-13


# ---------------------------------------------------------------------------
# weighted Gram matrix A diag(D) A^T
# ---------------------------------------------------------------------------

def test_gram_matrix_brute_force_and_structure():
    """The triple loop of the definition; symmetric, positive semi-definite for
    D >= 0; one b point gives the rank-one D e^{-|a_i - b|} e^{-|a_j - b|}."""
    rng = np.random.default_rng(20)
    a = np.round(rng.uniform(0, 5, 9), 1)
    b = np.concatenate([np.round(rng.uniform(-1, 6, 6), 1), a[:2]])
    D = rng.uniform(0.1, 2.0, 8)
    brute = np.zeros((9, 9))
    for i in range(9):
        for j in range(9):
            brute[i, j] = sum(D[l] * math.exp(-abs(a[i] - b[l])) * math.exp(-abs(a[j] - b[l]))
                              for l in range(8))
    M = O.gram_matrix(a, b, D)
    np.testing.assert_allclose(M, brute, rtol=1e-13)
    np.testing.assert_allclose(M, M.T, rtol=1e-15)
    assert np.linalg.eigvalsh(M).min() > -1e-12
    one = O.gram_matrix(a, np.array([2.3]), np.array([0.7]))
    u = np.exp(-np.abs(a - 2.3))
    np.testing.assert_allclose(one, 0.7 * np.outer(u, u), rtol=1e-14)


# ---------------------------------------------------------------------------
# the pins catch planted mistakes (mutants built on the CPU from the oracle)
# ---------------------------------------------------------------------------

def _lower_only(s, x):
    out, acc = np.empty_like(x), 0.0
    for i in range(len(x)):
        acc = x[i] + (math.exp(s[i - 1] - s[i]) * acc if i else 0.0)
        out[i] = acc
    return out


def test_pins_reject_planted_mistakes():
    rng = np.random.default_rng(15)
    s = np.cumsum(rng.uniform(0.05, 2.0, size=64))
    x = rng.normal(size=64)
    diag, off = _ou_precision(s)

    def ou_residual(y):
        back = diag * y
        back[:-1] += off * y[1:]
        back[1:] += off * y[:-1]
        return np.abs(back - x).max()

    good = O.sym_sorted(s, x)
    assert ou_residual(good) < 1e-10
    mutants = {
        "diagonal counted twice (dropped -x)": good + x,
        "lower part only": _lower_only(s, x),
        "reversed anchor order": O.sym_sorted(s[::-1].copy(), x),
        "operand transposed (x reversed)": O.sym_sorted(s, x[::-1].copy()),
    }
    for name, y in mutants.items():
        assert ou_residual(y) > 1e-3, name
    # general case with a and b swapped is K^T, not K
    a = rng.uniform(0, 5, 30)
    b = rng.uniform(0, 5, 30)
    xb = rng.normal(size=30)
    assert np.abs(O.general(b, a, xb) - O.dense_matvec(a, xb, b=b)).max() > 1e-3
    # backward with the sign of the signed sums flipped fails the finite differences
    xx, gg = rng.normal(size=30), rng.normal(size=30)
    _, da = O.backward(a, xx, gg)
    h = 1e-6
    ap, am = a.copy(), a.copy()
    ap[3] += h
    am[3] -= h
    fd = (_loss(ap, xx, gg) - _loss(am, xx, gg)) / (2 * h)
    assert abs(da[3] - fd) < 1e-6 and abs(-da[3] - fd) > 1e-3


def test_generator_is_seeded_and_sorted():
    a1 = synth.uniform(1000, 0, 64, seed=0)
    assert np.array_equal(a1, synth.uniform(1000, 0, 64, seed=0))
    assert not np.array_equal(a1, synth.uniform(1000, 0, 64, seed=1))
    assert np.array_equal(synth.uniform(1000, 0, 64)[500:], synth.uniform(1000, 0, 64)[500:])
    s = synth.sorted_uniform(100000, 0, 2.0 ** 30)
    assert np.all(np.diff(s) >= 0) and s[0] >= 0 and s[-1] <= 2.0 ** 30
    # sorted order statistics have the uniform distribution: compare quartiles
    assert abs(np.median(s) / 2.0 ** 30 - 0.5) < 0.01
    z = synth.normal(200000)
    assert abs(z.mean()) < 0.01 and abs(z.std() - 1) < 0.01
