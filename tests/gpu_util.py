"""Helpers for the GPU parity tests: numpy <-> CUDA tensors, and the parity
criterion max_i |y_i - y_ref_i| / (K0 |x|)_i from the fp64 oracle."""
import numpy as np
import torch

TOL = {np.float32: 1e-4, np.float64: 1e-10}


def dev(a):
    return torch.from_numpy(np.ascontiguousarray(a)).cuda()


def host(t):
    return t.detach().cpu().numpy()


def tol(dtype):
    return TOL[np.dtype(dtype).type]


def assert_close(y, y_ref, norm, dtype, what="", slack=None):
    """max_i max(0, |y_i - y_ref_i| - tiny - slack_i) / norm_i <= tol, tiny = the
    smallest normal number of the dtype: below it the format has fewer mantissa
    bits than the relative tolerance needs (subnormal range), so differences
    under tiny are not counted.  slack (fp32): the oracle's mass of the terms
    whose kernel value is below FLT_MIN (oracle.far_mass), which the fp32 path
    may flush to zero."""
    y = np.asarray(y, dtype=np.float64)
    y_ref = np.asarray(y_ref, dtype=np.float64)
    norm = np.asarray(norm, dtype=np.float64)
    tiny = float(np.finfo(dtype).tiny)
    assert np.all(np.isfinite(y)), f"{what}: non-finite output"
    diff = np.abs(y - y_ref) - tiny
    if slack is not None and np.dtype(dtype) == np.float32:
        diff = diff - np.asarray(slack, dtype=np.float64)
    diff = np.maximum(diff, 0.0)
    err = float(np.max(diff / np.where(norm > 0, norm, 1.0))) if diff.size else 0.0
    assert err <= tol(dtype), f"{what}: normalised error {err:.3e} > {tol(dtype):.0e}"
    return err


def rows_local(s, xs, idx, cutoff=746.0):
    """Oracle rows (K x, signed sums, K0|x|) for rows idx of ascending anchors s with
    values xs in the same order, passing the oracle only the window of s that can
    hold a non-zero fp64 term (|s_i - s_j| <= cutoff), so huge arrays are never
    converted whole."""
    import oracle as O
    outs, sgns, norms = [], [], []
    lo = np.searchsorted(s, s[idx] - cutoff, side="left")
    hi = np.searchsorted(s, s[idx] + cutoff, side="right")
    for i, l, h in zip(idx, lo, hi):
        o, g, a = O.rows(s[i:i + 1], s[l:h], xs[l:h], cutoff=cutoff)
        outs.append(o[0]); sgns.append(g[0]); norms.append(a[0])
    return np.array(outs), np.array(sgns), np.array(norms)
