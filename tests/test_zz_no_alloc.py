"""The allocation-free symmetric product (laplex_matvec_sym_noalloc).

Some callers cannot allocate device memory: code that runs where cudaMalloc is
unavailable or not allowed (a real-time loop, another library's allocator-free
hot path, a host with a fixed memory budget) cannot hand the library the
workspace laplex_matvec_sym needs.  This entry point keeps its scratch in a
fixed array inside the library instead.  The test calls it through the C ABI
(ctypes, raw device pointers) twice in a row, on different inputs, and checks
each result against laplex_matvec_sym on the same inputs, with the tolerance of
the other parity tests: max_i |y_i - y_ref_i| / (K0|x|)_i <= 1e-4 (K0|x| from
the fp64 oracle).  The file sorts last so that a run stopping at the first
failure has run every other test before it; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth

pytestmark = pytest.mark.gpu


def _call_noalloc(s_d, p_d, x_d, y_d):
    L = X.lib()
    st = L.laplex_matvec_sym_noalloc(ctypes.c_void_p(s_d.data_ptr()),
                                     None if p_d is None else ctypes.c_void_p(p_d.data_ptr()),
                                     s_d.numel(), ctypes.c_void_p(x_d.data_ptr()),
                                     ctypes.c_void_p(y_d.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == X.OK, L.laplex_last_error().decode()


def test_noalloc_matches_workspace_entry_point_twice():
    cases = [(300_001, 0.0, 5000.0, True), (2_000_003, -100.0, 100.0, False)]
    for n, lo, hi, use_perm in cases:          # two calls in a row, different inputs
        a, x = synth.sym_uniform(n, lo, hi, seed=n)
        s, perm = O.stable_sort(a)
        s_d = torch.from_numpy(s.astype(np.float32)).cuda()
        p_d = torch.from_numpy(perm.astype(np.int32)).cuda() if use_perm else None
        x_in = x if use_perm else x[perm]
        x_d = torch.from_numpy(np.ascontiguousarray(x_in)).cuda()
        y_na = torch.full_like(x_d, float("nan"))
        _call_noalloc(s_d, p_d, x_d, y_na)
        y_ws = X.matvec_sym(s_d, x_d, p_d)
        torch.cuda.synchronize()
        norm = O.norm_sym(a, x)
        if not use_perm:
            norm = norm[perm]
        err = O.max_norm_err(y_na.cpu().numpy(), y_ws.cpu().numpy().astype(np.float64), norm)
        assert np.isfinite(y_na.cpu().numpy()).all()
        assert err <= 1e-4, f"n={n}: normalised difference {err:.3e}"


def test_noalloc_rejects_oversized_n():
    L = X.lib()
    P = ctypes.c_void_p
    st = L.laplex_matvec_sym_noalloc(P(256), None, (1 << 30) + 1, P(256), P(512), None)
    assert st == X.EINVAL and b"2^30" in L.laplex_last_error()
