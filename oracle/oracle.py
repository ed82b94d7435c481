"""LAPLEX oracle -- TEST INFRASTRUCTURE ONLY.

A plain, slow, obviously-correct fp64 CPU statement of what the LAPLEX hot path
computes.  Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of
``bench.py`` may import it.  It shares no code with the CUDA library and never
calls it; inputs are the same seeded arrays the GPU receives, promoted to fp64.

Two independent routes are provided for every operator:

* ``dense_*`` -- the definition written out with numpy: the matrix
  K_ij = exp(-|a_i - b_j|) (times cos(phi_i - psi_j) when phased) is built and
  multiplied ("LAPLEX - La FFT dei Nuclei di Laplace Apprendibili", technical
  summary, §2.1 "L'Operatore").  Small sizes only.
* sequential -- sort plus the prefix/suffix recurrences of the same summary's
  §2.2 ("Algebra di Scansione Esatta"), in plain C (``laplex_oracle.c``), O(n).

and ``rows_*`` evaluates chosen rows of the dense definition at any size.
Parity of every function is pinned in tests/test_oracle_*.py against closed
forms, invariants, brute force and hand-worked examples (see the test headers).
"""
from __future__ import annotations

import ctypes

import numpy as np

from . import build as _build

_lib = None
_D = ctypes.POINTER(ctypes.c_double)
_I64 = ctypes.c_int64

#: fp64 exp underflows to exactly 0.0 below -745.14, so terms with |a_i - b_j|
#: >= 746 are exactly zero in an fp64 evaluation of the definition.
CUTOFF_F64 = 746.0

#: -ln(FLT_MIN) = 126 ln 2: a kernel value exp(-d) is below the smallest normal
#: fp32 number exactly when d > FAR_F32.
FAR_F32 = 126.0 * float(np.log(2.0))


def _L():
    global _lib
    if _lib is None:
        lib = ctypes.CDLL(_build.build())
        lib.orc_sym_sorted.argtypes = [_I64, _I64, _D, _D, _D]
        lib.orc_general_sorted.argtypes = [_I64, _I64, _I64, _D, _D, _D, _D]
        lib.orc_signed_sorted.argtypes = [_I64, _I64, _D, _D, _D]
        lib.orc_rows_window.argtypes = [_I64, _D, _D, _I64, _I64, _D, _D, _D, ctypes.c_double,
                                        _D, _D, _D]
        lib.orc_onesided_sorted.argtypes = [_I64, _I64, _I64, _D, _D, _D, ctypes.c_int, _D]
        for f in (lib.orc_sym_sorted, lib.orc_general_sorted, lib.orc_signed_sorted,
                  lib.orc_rows_window, lib.orc_onesided_sorted):
            f.restype = None
        _lib = lib
    return _lib


def _f64(x):
    return np.ascontiguousarray(np.asarray(x, dtype=np.float64))


def _p(x):
    return None if x is None else x.ctypes.data_as(_D)


def _cols(x):
    x = _f64(x)
    return (x.reshape(-1, 1), True) if x.ndim == 1 else (x, False)


# ---------------------------------------------------------------------------
# sort (the O(n log n) step; the recurrences run in sorted order, summary §2.2)
# ---------------------------------------------------------------------------

def stable_sort(a):
    """Ascending order of the anchors, ties by ascending index.

    Returns (s, perm) with s = a[perm] (fp64) and perm int64.  A library stable
    sort is the step; numeric comparison treats -0.0 and +0.0 as equal.
    Non-finite anchors are rejected (the operator is undefined there).
    """
    a64 = _f64(a)
    if a64.size and not np.all(np.isfinite(a64)):
        raise ValueError("non-finite anchor")
    perm = np.argsort(a64, kind="stable")
    return a64[perm], perm


# ---------------------------------------------------------------------------
# dense definition (summary §2.1)
# ---------------------------------------------------------------------------

def dense_matrix(a, b=None, phi=None, psi=None):
    """K_ij = exp(-|a_i - b_j|) [* cos(phi_i - psi_j)]; b = a, psi = phi when omitted."""
    a = _f64(a)
    b = a if b is None else _f64(b)
    K = np.exp(-np.abs(a[:, None] - b[None, :]))
    if phi is not None:
        phi = _f64(phi)
        psi = phi if psi is None else _f64(psi)
        K = K * np.cos(phi[:, None] - psi[None, :])
    return K


def gram_matrix(a, b, D=None):
    """M = A diag(D) A^T with A_ij = exp(-|a_i - b_j|) (a in R^n, b in R^k; D = 1
    when omitted): the weighted Gram matrix of the anchors ("LAPLEX - La FFT dei
    Nuclei di Laplace Apprendibili", technical summary §2.2 "Operatori di Gram"),
    by its definition, densely.  Small sizes only."""
    A = dense_matrix(a, b)
    d = np.ones(A.shape[1]) if D is None else _f64(D)
    return (A * d[None, :]) @ A.T


def dense_matvec(a, x, b=None, phi=None, psi=None):
    return dense_matrix(a, b, phi, psi) @ _f64(x)


def dense_backward(a, x, g):
    """For L = <g, K x>, K = K(a, a): dx = K^T g and
    da_m = -sum_j sign(a_m - a_j) exp(-|a_m - a_j|) (g_m x_j + x_m g_j),
    the derivative of the definition with d|t|/dt = sign(t), sign(0) = 0."""
    a, x, g = _f64(a), _f64(x), _f64(g)
    K = dense_matrix(a)
    S = np.sign(a[:, None] - a[None, :]) * K
    dx = K.T @ g
    da = -(g * (S @ x) + x * (S @ g))
    return dx, da


# ---------------------------------------------------------------------------
# sequential routes (summary §2.2)
# ---------------------------------------------------------------------------

def sym_sorted(s, x):
    """y = K x for anchors s already ascending; x, y in that order (C recurrences)."""
    s = _f64(s)
    x2, flat = _cols(x)
    n, B = x2.shape
    y = np.empty_like(x2)
    _L().orc_sym_sorted(n, B, _p(s), _p(x2), _p(y))
    return y.ravel() if flat else y


def sym(a, x):
    """y = K x, K_ij = exp(-|a_i - a_j|), any anchor order (sort, recur, un-permute)."""
    s, perm = stable_sort(a)
    x2, flat = _cols(x)
    ys = sym_sorted(s, x2[perm])
    y = np.empty_like(ys)
    y[perm] = ys
    return y.ravel() if flat else y


def general(a, b, x):
    """y = K x with K_ij = exp(-|a_i - b_j|), a in R^n, b in R^k, x in R^k (or [k, B]).

    The u/v interval aggregation of summary §2.2 "Caso Generale" (C code)."""
    sa, pa = stable_sort(a)
    sb, pb = stable_sort(b)
    x2, flat = _cols(x)
    xs = np.ascontiguousarray(x2[pb])
    n, k, B = sa.size, sb.size, x2.shape[1]
    ys = np.zeros((n, B))
    if n and k:
        _L().orc_general_sorted(n, k, B, _p(sa), _p(sb), _p(xs), _p(ys))
    y = np.empty_like(ys)
    y[pa] = ys
    return y.ravel() if flat else y


def general_T(a, b, w):
    """z = K^T w for K = K(a, b): K^T_ji = exp(-|b_j - a_i|) = K(b, a)_ji."""
    return general(b, a, w)


def phased(a, phi, v, b=None, psi=None):
    """y = K v with K_jk = exp(-|a_j - b_k|) cos(phi_j - psi_k) (summary §2.1),
    through cos(p - q) = cos p cos q + sin p sin q: two unphased channels
    cos(psi) v and sin(psi) v, recombined with cos(phi) and sin(phi)."""
    phi = _f64(phi)
    v = _f64(v)
    sym_case = b is None
    psi = phi if psi is None else _f64(psi)
    ch = np.stack([np.cos(psi) * v, np.sin(psi) * v], axis=1)
    u = sym(a, ch) if sym_case else general(a, b, ch)
    return np.cos(phi) * u[:, 0] + np.sin(phi) * u[:, 1]


def phased_T(a, phi, w, b, psi):
    """K^T w for the phased K(a, phi; b, psi): the phased operator with roles swapped."""
    return phased(b, psi, w, a, phi)


def gram(a, v, phi=None, D=None, b=None, psi=None):
    """z = K^T diag(D) K v (D = 1 when omitted), the Gram operator of summary §2.2
    "Operatori di Gram" applied to a vector: two chained products."""
    if phi is None:
        u = sym(a, v) if b is None else general(a, b, v)
    else:
        u = phased(a, phi, v) if b is None else phased(a, phi, v, b, psi)
    if D is not None:
        u = u * _f64(D)
    if phi is None:
        return sym(a, u) if b is None else general_T(a, b, u)
    return phased(a, phi, u) if b is None else phased_T(a, phi, u, b, psi)


def signed_sorted(s, v):
    """D_i = sum_j sign(s_i - s_j) exp(-|s_i - s_j|) v_j for ascending s (C code)."""
    s = _f64(s)
    v2, flat = _cols(v)
    n, B = v2.shape
    out = np.empty_like(v2)
    _L().orc_signed_sorted(n, B, _p(s), _p(v2), _p(out))
    return out.ravel() if flat else out


def backward(a, x, g):
    """Backward pass of L = <g, K x> w.r.t. x and the anchors (K = K(a, a)):
    dx = K^T g = K g;  da = -(g * Dx + x * Dg) with D the signed sums above."""
    s, perm = stable_sort(a)
    x, g = _f64(x), _f64(g)
    xs, gs = x[perm], g[perm]
    dxs = sym_sorted(s, gs)
    das = -(gs * signed_sorted(s, xs) + xs * signed_sorted(s, gs))
    dx = np.empty_like(dxs)
    da = np.empty_like(das)
    dx[perm] = dxs
    da[perm] = das
    return dx, da


def _onesided(sq, sb, vs, dirn):
    """One-sided decayed sums at ascending query points sq over ascending anchors
    sb with values vs [k, B] (C routine orc_onesided_sorted, strict inequalities)."""
    out = np.zeros((sq.size, vs.shape[1]))
    if sq.size and sb.size:
        _L().orc_onesided_sorted(sb.size, sq.size, vs.shape[1], _p(sb), _p(vs), _p(sq), dirn, _p(out))
    return out


def signed_general(a, b, v):
    """S_i = sum_j sign(a_i - b_j) exp(-|a_i - b_j|) v_j with sign(0) = 0: the
    derivative of the general kernel with respect to a_i ("LAPLEX - La FFT dei
    Nuclei di Laplace Apprendibili", technical summary §2.3: learnable anchors).
    The b_j below a_i minus the b_j above it, each side a one-sided decayed sum."""
    sa, pa = stable_sort(a)
    sb, pb = stable_sort(b)
    v2, flat = _cols(v)
    vs = np.ascontiguousarray(v2[pb])
    ss = _onesided(sa, sb, vs, 1) - _onesided(sa, sb, vs, -1)
    out = np.empty_like(ss)
    out[pa] = ss
    return out.ravel() if flat else out


def backward_general(a, b, x, g):
    """Backward pass of L = <g, K x>, K_ij = exp(-|a_i - b_j|), a in R^n,
    b in R^k: dx = K^T g, da_i = -g_i S(a <- b, x)_i, db_j = -x_j S(b <- a, g)_j
    with S the signed sums above (the derivative of exp(-|a_i - b_j|) is
    -sign(a_i - b_j) exp(-|a_i - b_j|) in a_i and +sign(a_i - b_j) ... in b_j)."""
    x, g = _f64(x), _f64(g)
    dx = general_T(a, b, g)
    da = -g * signed_general(a, b, x)
    db = -x * signed_general(b, a, g)
    return dx, da, db


def backward_phased(a, phi, x, g, b=None, psi=None):
    """Backward pass of L = <g, K x> for the phased kernel
    K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j) (summary §2.1; trainable anchors
    and phases, §2.3), w.r.t. x, the phases and the anchors:
        dx_j   = sum_i K_ij g_i,
        dphi_i = -g_i sum_j exp(-|a_i - b_j|) sin(phi_i - psi_j) x_j,
        dpsi_j =  x_j sum_i exp(-|a_i - b_j|) sin(phi_i - psi_j) g_i,
        da_i   = -g_i sum_j sign(a_i - b_j) K_ij x_j,
        db_j   = -x_j sum_i sign(b_j - a_i) K_ij g_i          (sign(0) = 0).
    Through cos(p - q) = cos p cos q + sin p sin q and
    sin(p - q) = sin p cos q - cos p sin q every sum is a combination of two
    unphased channels, (cos psi x, sin psi x) seen from a and (cos phi g, sin phi g)
    seen from b, each summed plainly (general) and signed (signed_general).
    b = None: the symmetric case (b = a, psi = phi); the anchors and phases are
    shared, so (dx, dphi + dpsi, da + db) is returned.  Otherwise
    (dx, dphi, dpsi, da, db)."""
    sym_case = b is None
    phi, x, g = _f64(phi), _f64(x), _f64(g)
    if sym_case:
        b, psi = a, phi
    psi = _f64(psi)
    cphi, sphi, cpsi, spsi = np.cos(phi), np.sin(phi), np.cos(psi), np.sin(psi)
    xc = np.stack([cpsi * x, spsi * x], axis=1)  # channels on b
    gc = np.stack([cphi * g, sphi * g], axis=1)  # channels on a
    Pa, Sa = general(a, b, xc), signed_general(a, b, xc)
    Pb, Sb = general(b, a, gc), signed_general(b, a, gc)
    dx = cpsi * Pb[:, 0] + spsi * Pb[:, 1]
    dphi = g * (cphi * Pa[:, 1] - sphi * Pa[:, 0])
    dpsi = x * (cpsi * Pb[:, 1] - spsi * Pb[:, 0])
    da = -g * (cphi * Sa[:, 0] + sphi * Sa[:, 1])
    db = -x * (cpsi * Sb[:, 0] + spsi * Sb[:, 1])
    if sym_case:
        return dx, dphi + dpsi, da + db
    return dx, dphi, dpsi, da, db


def norm_backward_phased(a, x, g, b=None):
    """Bounds of the phased gradients term by term (|cos|, |sin| <= 1), with the
    unphased K0: (K0^T|g|, |g| K0|x|, |x| K0^T|g|) for dx, (dphi, da), (dpsi, db);
    symmetric (b = None): (K0|g|, |g| K0|x| + |x| K0|g|) for dx and the totals."""
    if b is None:
        return norm_backward(a, x, g)
    return norm_backward_general(a, b, x, g)


def norm_backward_general(a, b, x, g):
    """Bounds of |dx|, |da|, |db| term by term: K^T|g|, |g| K|x|, |x| K^T|g|."""
    x, g = np.abs(_f64(x)), np.abs(_f64(g))
    ktg = general(b, a, g)
    return ktg, g * general(a, b, x), x * ktg


# ---------------------------------------------------------------------------
# rows of the dense definition at any size (sampled parity)
# ---------------------------------------------------------------------------

def rows(ra, sb, xs, rphi=None, spsi=None, cutoff=CUTOFF_F64):
    """For chosen rows (anchors ra, phases rphi) against ascending b-anchors sb with
    values xs ([k] or [k, B], phases spsi, all in sorted-b order) return
    (K x, signed sums, K0 |x|) for those rows; see orc_rows_window."""
    ra = _f64(ra)
    sb = _f64(sb)
    x2, flat = _cols(xs)
    m, (k, B) = ra.size, x2.shape
    out = np.empty((m, B))
    sgn = np.empty((m, B))
    absn = np.empty((m, B))
    rphi = None if rphi is None else _f64(rphi)
    spsi = None if spsi is None else _f64(spsi)
    _L().orc_rows_window(m, _p(ra), _p(rphi), k, B, _p(sb), _p(spsi), _p(x2), float(cutoff),
                         _p(out), _p(sgn), _p(absn))
    if flat:
        return out.ravel(), sgn.ravel(), absn.ravel()
    return out, sgn, absn


# ---------------------------------------------------------------------------
# normalisers for the parity criterion max_i |y_i - y_ref_i| / norm_i
# ---------------------------------------------------------------------------

def norm_sym(a, x):
    """K0 |x| with the unphased kernel: an upper bound of |K| |x| for every variant."""
    return sym(a, np.abs(_f64(x)))


def norm_general(a, b, x):
    return general(a, b, np.abs(_f64(x)))


def norm_gram(a, v, D=None, b=None):
    u = norm_sym(a, v) if b is None else norm_general(a, b, v)
    if D is not None:
        u = u * np.abs(_f64(D))
    return sym(a, u) if b is None else general_T(a, b, u)


def norm_backward(a, x, g):
    """(K0|g|, |g| K0|x| + |x| K0|g|): bounds of |dx| and |da| term by term."""
    x, g = np.abs(_f64(x)), np.abs(_f64(g))
    kx, kg = sym(a, x), sym(a, g)
    return kg, g * kx + x * kg


def far_mass(a, v, b=None, dist=FAR_F32):
    """m_i = sum over j with |a_i - b_j| > dist of exp(-|a_i - b_j|) |v_j|
    (b = a when None): the |v|-weighted mass of the terms whose kernel value is
    below exp(-dist) (FLT_MIN for the default).  Not a step of the method: the
    parity criterion of fp32 results allows terms below FLT_MIN to be lost.
    Computed as exp(-dist) times one-sided decayed sums at the shifted points
    a_i - dist and a_i + dist (strict inequalities)."""
    a = _f64(a)
    b = a if b is None else _f64(b)
    v, one = _cols(np.abs(_f64(v)))
    B = v.shape[1]
    ob = np.argsort(b, kind="stable")
    sb = np.ascontiguousarray(b[ob])
    vs = np.ascontiguousarray(v[ob])
    out = np.zeros((a.size, B))
    for dirn, shift in ((1, -dist), (-1, dist)):
        q = a + shift
        oq = np.argsort(q, kind="stable")
        qs = np.ascontiguousarray(q[oq])
        r = np.zeros((a.size, B))
        _L().orc_onesided_sorted(sb.size, qs.size, B, _p(sb), _p(vs), _p(qs), dirn, _p(r))
        out[oq] += r
    out *= np.exp(-dist)
    return out[:, 0] if one else out


def max_norm_err(y, y_ref, norm):
    """max_i |y_i - y_ref_i| / norm_i (norm_i = 0 only where y_ref_i = 0 exactly)."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = _f64(y_ref)
    norm = _f64(norm)
    err = np.abs(y - y_ref)
    safe = np.where(norm > 0, norm, 1.0)
    return float(np.max(err / safe)) if err.size else 0.0
