"""C-ABI library: loads, exports every symbol include/laplex.h declares, and
rejects bad arguments on the host (no kernel is launched; no GPU needed)."""
import ctypes
import os
import re

import pytest

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "laplex.h")


@pytest.fixture(scope="module")
def L():
    from exact_laplace_b200 import build, laplex
    build.build()
    return laplex.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(laplex_[a-z_0-9]+)\s*\(", text)))


def test_header_declares_the_product_calls():
    names = declared_functions()
    for req in ("laplex_sort_anchors", "laplex_matvec_sym", "laplex_matvec_general",
                "laplex_matvec_phased", "laplex_gram", "laplex_backward"):
        assert req in names


def test_every_declared_symbol_is_exported(L):
    from exact_laplace_b200 import laplex
    names = declared_functions()
    for name in names:
        assert hasattr(L, name), name
    assert set(names) <= set(laplex.SIGNATURES), set(names) - set(laplex.SIGNATURES)


def test_version_and_status_strings(L):
    assert L.laplex_version() >= 10000
    assert L.laplex_build_flags() in (0, 1)
    assert L.laplex_status_string(0) == b"LAPLEX_OK"
    assert L.laplex_status_string(5) == b"LAPLEX_ETIMEOUT"


def test_workspace_size_host_only(L):
    from exact_laplace_b200 import laplex as X
    for op in range(13):
        for n in (0, 1, 4096, 1 << 24):
            assert X.workspace_size(op, n, 1000 if op in (2, 3, 4, 6, 7, 8) else 0, 1) >= 256
    with pytest.raises(X.LaplexError) as e:
        X.workspace_size(1, -1)
    assert e.value.status == X.EINVAL
    with pytest.raises(X.LaplexError):
        X.workspace_size(1, 1 << 31)
    with pytest.raises(X.LaplexError):
        X.workspace_size(1, 10, 0, 0)
    with pytest.raises(X.LaplexError):
        X.workspace_size(13, 10)
    with pytest.raises(X.LaplexError):
        X.workspace_size(-1, 10)


def test_argument_errors_return_before_any_launch(L):
    from exact_laplace_b200 import laplex as X
    P = ctypes.c_void_p
    # NULL x with n > 0
    st = L.laplex_matvec_sym(P(256), None, 10, None, P(256), 1, 0, P(256), 1 << 20, None)
    assert st == X.EINVAL and b"x" in L.laplex_last_error()
    # misaligned pointer
    st = L.laplex_matvec_sym(P(256), None, 10, P(260), P(256), 1, 0, P(256), 1 << 20, None)
    assert st == X.EINVAL and b"aligned" in L.laplex_last_error()
    # bad dtype
    st = L.laplex_matvec_sym(P(256), None, 10, P(256), P(512), 1, 7, P(256), 1 << 20, None)
    assert st == X.EINVAL
    # workspace too small
    st = L.laplex_matvec_sym(P(256), None, 1 << 20, P(256), P(512), 1, 0, P(256), 300, None)
    assert st == X.EWORKSPACE
    # NULL workspace
    st = L.laplex_backward(P(256), None, 10, P(256), P(256), P(256), P(256), 0, None, 0, None)
    assert st == X.EINVAL
    # phased backward: NULL phases with n > 0, misaligned optional output
    size = ctypes.c_size_t()
    assert L.laplex_workspace_size(8, 10, 10, 1, 0, ctypes.byref(size)) == 0
    st = L.laplex_backward_phased(P(256), None, None, 10, P(256), None, P(256), 10, P(256), P(256),
                                  None, None, None, P(256), None, 0, P(256), size.value, None)
    assert st == X.EINVAL and b"phi" in L.laplex_last_error()
    st = L.laplex_backward_phased(P(256), None, P(256), 10, P(256), None, P(256), 10, P(256), P(256),
                                  None, P(260), None, None, None, 0, P(256), size.value, None)
    assert st == X.EINVAL and b"dphi" in L.laplex_last_error()
    st = L.laplex_backward_phased(P(256), None, P(256), 10, None, None, None, 0, P(256), P(256),
                                  None, None, None, P(256), None, 0, P(256), 300, None)
    assert st == X.EWORKSPACE
    # n = 0 is a no-op that needs no pointers
    size = ctypes.c_size_t()
    assert L.laplex_workspace_size(1, 0, 0, 1, 0, ctypes.byref(size)) == 0
    assert L.laplex_matvec_sym(None, None, 0, None, None, 1, 0, P(256), size.value, None) == 0


def test_carry_and_unsorted_argument_errors(L):
    """laplex_sort_anchors_carry and laplex_matvec_sym_unsorted check their
    arguments on the host and return before any launch."""
    from exact_laplace_b200 import laplex as X
    P = ctypes.c_void_p
    size = ctypes.c_size_t()
    assert L.laplex_workspace_size(X.OP_SORT_CARRY, 1000, 0, 1, 0, ctypes.byref(size)) == 0
    big = size.value
    # NULL values with n > 0
    st = L.laplex_sort_anchors_carry(P(256), None, 1000, 0, P(512), P(768), P(1024), P(256), big, None)
    assert st == X.EINVAL and b"x" in L.laplex_last_error()
    # misaligned xs
    st = L.laplex_sort_anchors_carry(P(256), P(512), 1000, 0, P(768), P(1024), P(1284), P(256), big, None)
    assert st == X.EINVAL and b"aligned" in L.laplex_last_error()
    # workspace too small
    st = L.laplex_sort_anchors_carry(P(256), P(512), 1000, 0, P(768), P(1024), P(1280), P(256), 300, None)
    assert st == X.EWORKSPACE
    # n out of range
    st = L.laplex_sort_anchors_carry(P(256), P(512), 1 << 31, 0, P(768), P(1024), P(1280), P(256), big, None)
    assert st == X.EINVAL
    assert L.laplex_workspace_size(X.OP_SYM_UNSORTED, 1000, 0, 1, 1, ctypes.byref(size)) == 0
    big = size.value
    # NULL perm output, bad dtype, small workspace
    st = L.laplex_matvec_sym_unsorted(P(256), P(512), 1000, 1, P(768), P(1024), None, P(256), big, None)
    assert st == X.EINVAL and b"perm" in L.laplex_last_error()
    st = L.laplex_matvec_sym_unsorted(P(256), P(512), 1000, 5, P(768), P(1024), P(1280), P(256), big, None)
    assert st == X.EINVAL
    st = L.laplex_matvec_sym_unsorted(P(256), P(512), 1000, 1, P(768), P(1024), P(1280), P(256), 300, None)
    assert st == X.EWORKSPACE
    # n = 0: no pointers needed
    assert L.laplex_workspace_size(X.OP_SYM_UNSORTED, 0, 0, 1, 0, ctypes.byref(size)) == 0
    assert L.laplex_matvec_sym_unsorted(None, None, 0, 0, None, None, None, P(256), size.value, None) == 0
    assert L.laplex_workspace_size(X.OP_SORT_CARRY, 0, 0, 1, 0, ctypes.byref(size)) == 0
    assert L.laplex_sort_anchors_carry(None, None, 0, 0, None, None, None, P(256), size.value, None) == 0


def test_workspace_of_new_ops_grows_with_n(L):
    from exact_laplace_b200 import laplex as X
    for op in (X.OP_SORT_CARRY, X.OP_SYM_UNSORTED):
        for dt in (0, 1):
            sizes = []
            for n in (1, 1 << 10, 1 << 20, 1 << 26):
                size = ctypes.c_size_t()
                assert L.laplex_workspace_size(op, n, 0, 1, dt, ctypes.byref(size)) == 0
                sizes.append(size.value)
            assert sizes == sorted(sizes) and sizes[-1] >= (1 << 26) * 12
