"""The allocation-free symmetric product (laplex_matvec_sym_noalloc).

Some callers cannot allocate device memory: code that runs where cudaMalloc is
unavailable or not allowed (a real-time loop, another library's allocator-free
hot path, a host with a fixed memory budget) cannot hand the library the
workspace laplex_matvec_sym needs.  This entry point keeps its scratch in a
fixed array inside the library instead.

The test calls it through the C ABI (ctypes, raw device pointers), several
times in a row on different inputs, and checks every result against the fp64
oracle (the sequential recurrences on the same seeded inputs) and against
laplex_matvec_sym on the same inputs, with the tolerance of the other parity
tests: max_i |y_i - y_ref_i| / (K0|x|)_i <= 1e-4, fp32 terms below FLT_MIN
allowed to vanish (oracle.far_mass).  The cases reach the carry kernels in
every shape they take over the fixed scratch: one carry block (up to 2048
tiles of 4096 anchors, the carries written over the tile totals in place) and
several (4097 tiles: three blocks, with carries between blocks), threads with
fewer than 8 tiles at the end, a run of equal anchors across a tile boundary,
and carries that cross every tile (all anchors equal; 10^6 anchors inside one
unit).  The file sorts last so that a run stopping at
the first failure has run every other test before it; it also passes on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

import oracle as O
from exact_laplace_b200 import laplex as X
from exact_laplace_b200 import synth
from gpu_util import assert_close

pytestmark = pytest.mark.gpu

TILE = 4096  # anchors per tile of the allocation-free product


def _call_noalloc(s_d, p_d, x_d, y_d):
    L = X.lib()
    st = L.laplex_matvec_sym_noalloc(ctypes.c_void_p(s_d.data_ptr()),
                                     None if p_d is None else ctypes.c_void_p(p_d.data_ptr()),
                                     s_d.numel(), ctypes.c_void_p(x_d.data_ptr()),
                                     ctypes.c_void_p(y_d.data_ptr()),
                                     ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))
    assert st == X.OK, L.laplex_last_error().decode()


def _equal_run_across_tile(n):
    """a ~ U(0, n) with the anchors of sorted positions 700*TILE - 40 ..
    700*TILE + 39 set to one value (they stay in sorted order)."""
    a, x = synth.sym_uniform(n, 0.0, float(n), seed=7)
    _, perm = O.stable_sort(a)
    r = perm[700 * TILE - 40: 700 * TILE + 40]
    a[r] = a[perm[700 * TILE]]
    return a, x


CASES = [
    ("U(0,5000), perm", lambda: synth.sym_uniform(300_001, 0.0, 5000.0, seed=300_001), True),
    ("U(-100,100), sorted order", lambda: synth.sym_uniform(2_000_003, -100.0, 100.0, seed=3), False),
    ("1465 tiles, equal run across a tile boundary, perm", lambda: _equal_run_across_tile(6_000_007), True),
    ("4097 tiles (three carry blocks), U(0,2^24), sorted order",
     lambda: synth.sym_uniform((1 << 24) + 43, 0.0, float(1 << 24), seed=11), False),
    ("all anchors equal, perm",
     lambda: (np.full(1_000_003, 3.25, dtype=np.float32), synth.normal(1_000_003, seed=5, stream="x")), True),
    ("10^6 anchors in one unit, sorted order", lambda: synth.sym_uniform(1_000_000, 0.0, 1.0, seed=13), False),
]


def test_noalloc_matches_oracle_and_workspace_entry_point():
    for name, make, use_perm in CASES:  # calls in a row on different inputs share the scratch
        a, x = make()
        s, perm = O.stable_sort(a)
        s_d = torch.from_numpy(s.astype(np.float32)).cuda()
        p_d = torch.from_numpy(perm.astype(np.int32)).cuda() if use_perm else None
        x_in = x if use_perm else x[perm]
        x_d = torch.from_numpy(np.ascontiguousarray(x_in)).cuda()
        y_na = torch.full_like(x_d, float("nan"))
        _call_noalloc(s_d, p_d, x_d, y_na)
        y_ws = X.matvec_sym(s_d, x_d, p_d)
        torch.cuda.synchronize()
        y_ref, norm, slack = O.sym(a, x), O.norm_sym(a, x), O.far_mass(a, x)
        if not use_perm:
            y_ref, norm, slack = y_ref[perm], norm[perm], slack[perm]
        got = y_na.cpu().numpy()
        assert_close(got, y_ref, norm, np.float32, f"{name}: against the oracle", slack=slack)
        assert_close(got, y_ws.cpu().numpy(), norm, np.float32,
                     f"{name}: against laplex_matvec_sym", slack=slack)


def test_noalloc_rejects_oversized_n():
    L = X.lib()
    P = ctypes.c_void_p
    st = L.laplex_matvec_sym_noalloc(P(256), None, (1 << 30) + 1, P(256), P(512), None)
    assert st == X.EINVAL and b"2^30" in L.laplex_last_error()
