"""Thin Python binding of liblaplex.so (argument marshalling only).

Every function here checks tensor dtypes/devices/shapes, allocates outputs and
workspace with torch (device memory is the only thing torch provides), and calls
the C ABI of include/laplex.h with raw pointers and the current CUDA stream.
All arithmetic runs in the library's CUDA kernels; there is no CPU path and no
fallback: a missing or unloadable library raises ``LaplexError``.

Host (CPU) tensors are accepted by the ``*_host`` helpers, which copy inputs to
the device, call the same entry point and copy the result back (the end-to-end
path a user without device buffers takes).
"""
from __future__ import annotations

import ctypes
import os
import threading

import torch

_HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(_HERE, "liblaplex.so")

OK, EINVAL, ENONFINITE, EWORKSPACE, ECUDA, ETIMEOUT = range(6)
BUILD_ACCURATE_EXP = 1  # laplex_build_flags() bit
F32, F64 = 0, 1
(OP_SORT, OP_SYM, OP_GENERAL, OP_PHASED, OP_GRAM, OP_BACKWARD, OP_BACKWARD_GENERAL, OP_GRAM_MATRIX,
 OP_BACKWARD_PHASED, OP_PERMUTE, OP_SYM_PLANNED, OP_SORT_CARRY, OP_SYM_UNSORTED) = range(13)

_lib = None
_lock = threading.Lock()
_P = ctypes.c_void_p
_I64 = ctypes.c_int64


class LaplexError(RuntimeError):
    def __init__(self, status: int, msg: str):
        super().__init__(f"{_STATUS_NAMES.get(status, status)}: {msg}")
        self.status = status


_STATUS_NAMES = {OK: "LAPLEX_OK", EINVAL: "LAPLEX_EINVAL", ENONFINITE: "LAPLEX_ENONFINITE",
                 EWORKSPACE: "LAPLEX_EWORKSPACE", ECUDA: "LAPLEX_ECUDA",
                 ETIMEOUT: "LAPLEX_ETIMEOUT"}

#: every symbol include/laplex.h declares, with its ctypes signature
SIGNATURES = {
    "laplex_version": ([], ctypes.c_int),
    "laplex_build_flags": ([], ctypes.c_int),
    "laplex_status_string": ([ctypes.c_int], ctypes.c_char_p),
    "laplex_last_error": ([], ctypes.c_char_p),
    "laplex_workspace_size": ([ctypes.c_int, _I64, _I64, _I64, ctypes.c_int,
                               ctypes.POINTER(ctypes.c_size_t)], ctypes.c_int),
    "laplex_workspace_init": ([_P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_get_device_status": ([_P, _P], ctypes.c_int),
    "laplex_sort_anchors": ([_P, _I64, ctypes.c_int, _P, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_matvec_sym": ([_P, _P, _I64, _P, _P, _I64, ctypes.c_int, _P, ctypes.c_size_t, _P],
                          ctypes.c_int),
    "laplex_matvec_general": ([_P, _P, _I64, _P, _P, _I64, _P, _P, _I64, ctypes.c_int,
                               ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_matvec_phased": ([_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _I64, ctypes.c_int,
                              ctypes.c_int, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_gram": ([_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _P, _I64, ctypes.c_int, _P,
                     ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_backward": ([_P, _P, _I64, _P, _P, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P],
                        ctypes.c_int),
    "laplex_backward_general": ([_P, _P, _I64, _P, _P, _I64, _P, _P, _P, _P, _P, ctypes.c_int, _P,
                                 ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_backward_phased": ([_P, _P, _P, _I64, _P, _P, _P, _I64, _P, _P, _P, _P, _P, _P, _P, ctypes.c_int,
                                _P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_gram_matrix": ([_P, _P, _I64, _P, _P, _I64, _P, _P, _I64, ctypes.c_int, _P, ctypes.c_size_t, _P],
                           ctypes.c_int),
    "laplex_matvec_sym_noalloc": ([_P, _P, _I64, _P, _P, _P], ctypes.c_int),
    "laplex_set_profile_events": ([_P, _P], ctypes.c_int),
    "laplex_test_set_sort_wait": ([ctypes.c_uint32, ctypes.c_int], ctypes.c_int),
    "laplex_permute": ([_P, _P, _I64, ctypes.c_int, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_invert_perm": ([_P, _I64, _P, _P, ctypes.c_size_t, _P], ctypes.c_int),
    "laplex_matvec_sym_planned": ([_P, _P, _P, _I64, _P, _P, ctypes.c_int, _P, ctypes.c_size_t, _P],
                                  ctypes.c_int),
    "laplex_sort_anchors_carry": ([_P, _P, _I64, ctypes.c_int, _P, _P, _P, _P, ctypes.c_size_t, _P],
                                  ctypes.c_int),
    "laplex_matvec_sym_unsorted": ([_P, _P, _I64, ctypes.c_int, _P, _P, _P, _P, ctypes.c_size_t, _P],
                                   ctypes.c_int),
}


def lib():
    """The loaded library (raises LaplexError if it cannot be loaded)."""
    global _lib
    if _lib is None:
        with _lock:
            if _lib is None:
                if not os.path.exists(LIB_PATH):
                    raise LaplexError(ECUDA, f"{LIB_PATH} is missing: build it with "
                                             "`python -m exact_laplace_b200.build` (nvcc, sm_100a)")
                try:
                    L = ctypes.CDLL(LIB_PATH)
                except OSError as e:
                    raise LaplexError(ECUDA, f"cannot load {LIB_PATH}: {e}") from e
                for name, (args, res) in SIGNATURES.items():
                    f = getattr(L, name)
                    f.argtypes = args
                    f.restype = res
                _lib = L
    return _lib


def _check(status: int):
    if status != OK:
        raise LaplexError(status, lib().laplex_last_error().decode())


def _dt(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return F32
    if t.dtype == torch.float64:
        return F64
    raise LaplexError(EINVAL, f"dtype {t.dtype} is not float32/float64")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(device) -> ctypes.c_void_p:
    return ctypes.c_void_p(torch.cuda.current_stream(device).cuda_stream)


def _dev(*ts):
    dev = None
    for t in ts:
        if t is None:
            continue
        if not t.is_cuda:
            raise LaplexError(EINVAL, "tensors must be on a CUDA device (use the *_host helpers "
                                      "for host buffers)")
        if not t.is_contiguous():
            raise LaplexError(EINVAL, "tensors must be contiguous")
        if dev is None:
            dev = t.device
        elif t.device != dev:
            raise LaplexError(EINVAL, "tensors are on different devices")
    return dev


def _perm(p):
    if p is not None and p.dtype != torch.int32:
        raise LaplexError(EINVAL, "perm must be int32")
    return p


class Workspace:
    """Device workspace cache (one growing buffer per device and stream).

    The header is zeroed when the buffer is (re)allocated; the library then keeps
    its sticky status word there.  ``status()`` synchronises and reports it."""

    _cache: dict = {}

    @classmethod
    def get(cls, device, nbytes: int) -> "torch.Tensor":
        key = (device, torch.cuda.current_stream(device).cuda_stream)
        buf = cls._cache.get(key)
        if buf is None or buf.numel() < nbytes:
            buf = torch.zeros(max(nbytes, 256), dtype=torch.uint8, device=device)
            cls._cache[key] = buf
        return buf

    @classmethod
    def status(cls, device=None) -> None:
        device = torch.device("cuda", torch.cuda.current_device()) if device is None else device
        key = (device, torch.cuda.current_stream(device).cuda_stream)
        buf = cls._cache.get(key)
        if buf is not None:
            _check(lib().laplex_get_device_status(_ptr(buf), _stream(device)))


def workspace_size(op: int, n: int, k: int = 0, B: int = 1, dtype=torch.float32) -> int:
    out = ctypes.c_size_t(0)
    _check(lib().laplex_workspace_size(op, n, k, B, F64 if dtype == torch.float64 else F32,
                                       ctypes.byref(out)))
    return out.value


def _ws(op, n, k, B, dtype, device):
    nb = workspace_size(op, n, k, B, dtype)
    buf = Workspace.get(device, nb)
    return buf, buf.numel()


def set_profile_events(before=None, after=None) -> None:
    """Record two torch.cuda.Event objects around the dominant kernel of the
    following calls on this thread (both recorded once first, so that their CUDA
    events exist); None, None switches it off."""
    h = [None if e is None else ctypes.c_void_p(e.cuda_event) for e in (before, after)]
    _check(lib().laplex_set_profile_events(h[0], h[1]))


def test_set_sort_wait(polls: int = 0, force_expiry: bool = False) -> None:
    """Test hook: bound of the sort's look-back waits on this thread (0: the
    default) and whether every wait is made to run to that bound."""
    _check(lib().laplex_test_set_sort_wait(polls, 1 if force_expiry else 0))


def device_status(device=None) -> None:
    """Synchronise and raise if a kernel recorded a device-side error."""
    Workspace.status(device)


# ----------------------------------------------------------------------------- calls

def sort_anchors(a: torch.Tensor, sorted_out=None, perm_out=None):
    """(sorted, perm): the anchors ascending and the int32 permutation, ties by index."""
    dev = _dev(a, sorted_out, perm_out)
    n = a.numel()
    s = torch.empty_like(a) if sorted_out is None else sorted_out
    p = torch.empty(n, dtype=torch.int32, device=dev) if perm_out is None else perm_out
    ws, nb = _ws(OP_SORT, n, 0, 1, a.dtype, dev)
    _check(lib().laplex_sort_anchors(_ptr(a), n, _dt(a), _ptr(s), _ptr(p), _ptr(ws), nb,
                                     _stream(dev)))
    return s, p


def sort_anchors_carry(a: torch.Tensor, x: torch.Tensor, sorted_out=None, perm_out=None, xs_out=None):
    """(sorted, perm, xs): the sort of laplex_sort_anchors with x carried along,
    xs[r] = x[perm[r]]."""
    dev = _dev(a, x, sorted_out, perm_out, xs_out)
    n = a.numel()
    if x.numel() != n or x.dtype != a.dtype:
        raise LaplexError(EINVAL, "x must have n elements and the anchors' dtype")
    s = torch.empty_like(a) if sorted_out is None else sorted_out
    p = torch.empty(n, dtype=torch.int32, device=dev) if perm_out is None else perm_out
    xs = torch.empty_like(x) if xs_out is None else xs_out
    ws, nb = _ws(OP_SORT_CARRY, n, 0, 1, a.dtype, dev)
    _check(lib().laplex_sort_anchors_carry(_ptr(a), _ptr(x), n, _dt(a), _ptr(s), _ptr(p), _ptr(xs), _ptr(ws), nb,
                                           _stream(dev)))
    return s, p, xs


def matvec_sym_unsorted(a: torch.Tensor, x: torch.Tensor, out=None, sorted_out=None, perm_out=None):
    """(y, sorted, perm): y = K x on anchors and x in the caller's order (one
    column), in one call: the sort carrying x, the product, y back to caller order."""
    dev = _dev(a, x, out, sorted_out, perm_out)
    n = a.numel()
    if x.numel() != n or x.dtype != a.dtype:
        raise LaplexError(EINVAL, "x must have n elements and the anchors' dtype")
    y = torch.empty_like(x) if out is None else out
    s = torch.empty_like(a) if sorted_out is None else sorted_out
    p = torch.empty(n, dtype=torch.int32, device=dev) if perm_out is None else perm_out
    ws, nb = _ws(OP_SYM_UNSORTED, n, 0, 1, a.dtype, dev)
    _check(lib().laplex_matvec_sym_unsorted(_ptr(a), _ptr(x), n, _dt(a), _ptr(y), _ptr(s), _ptr(p), _ptr(ws), nb,
                                            _stream(dev)))
    return y, s, p


def matvec_sym(sorted_anchors: torch.Tensor, x: torch.Tensor, perm=None, out=None):
    """y = K x for K_ij = exp(-|a_i - a_j|) given the sorted anchors (and perm, if x is
    in the caller's order).  x: [n] or [n, B]."""
    dev = _dev(sorted_anchors, x, _perm(perm), out)
    n = sorted_anchors.numel()
    B = 1 if x.dim() == 1 else x.shape[1]
    if x.shape[0] != n or x.dtype != sorted_anchors.dtype:
        raise LaplexError(EINVAL, "x must have n rows and the anchors' dtype")
    y = torch.empty_like(x) if out is None else out
    ws, nb = _ws(OP_SYM, n, 0, B, x.dtype, dev)
    _check(lib().laplex_matvec_sym(_ptr(sorted_anchors), _ptr(perm), n, _ptr(x), _ptr(y), B,
                                   _dt(x), _ptr(ws), nb, _stream(dev)))
    return y


def permute(src: torch.Tensor, idx: torch.Tensor, out=None):
    """dst[idx[i]] = src[i] (4- or 8-byte elements, moved as bits); idx int32."""
    dev = _dev(src, _perm(idx), out)
    n = src.numel()
    if idx.numel() != n or src.element_size() not in (4, 8):
        raise LaplexError(EINVAL, "src and idx must have n elements; src of 4 or 8 bytes")
    dst = torch.empty_like(src) if out is None else out
    dt = F64 if src.element_size() == 8 else F32
    ws, nb = _ws(OP_PERMUTE, n, 0, 1, torch.float64 if dt == F64 else torch.float32, dev)
    _check(lib().laplex_permute(_ptr(src), _ptr(idx), n, dt, _ptr(dst), _ptr(ws), nb, _stream(dev)))
    return dst


def invert_perm(perm: torch.Tensor, out=None):
    """inv with inv[perm[r]] = r (int32)."""
    dev = _dev(_perm(perm), out)
    n = perm.numel()
    inv = torch.empty_like(perm) if out is None else out
    ws, nb = _ws(OP_PERMUTE, n, 0, 1, torch.float32, dev)
    _check(lib().laplex_invert_perm(_ptr(perm), n, _ptr(inv), _ptr(ws), nb, _stream(dev)))
    return inv


def matvec_sym_noalloc(sorted_anchors: torch.Tensor, x: torch.Tensor, perm=None, out=None):
    """laplex_matvec_sym_noalloc: y = K x (fp32, one column) with the library's
    fixed device scratch instead of a workspace (n <= 2^30)."""
    dev = _dev(sorted_anchors, x, _perm(perm), out)
    n = sorted_anchors.numel()
    if x.numel() != n or x.dtype != torch.float32 or sorted_anchors.dtype != torch.float32:
        raise LaplexError(EINVAL, "fp32 anchors and x with n elements")
    y = torch.empty_like(x) if out is None else out
    _check(lib().laplex_matvec_sym_noalloc(_ptr(sorted_anchors), _ptr(perm), n, _ptr(x), _ptr(y), _stream(dev)))
    return y


def matvec_sym_planned(sorted_anchors: torch.Tensor, perm: torch.Tensor, inv: torch.Tensor, x: torch.Tensor,
                       out=None):
    """y = K x for x, y in the caller's order (one column), through the plan
    (sorted, perm, inv): bucketed moves into and out of sorted order."""
    dev = _dev(sorted_anchors, _perm(perm), _perm(inv), x, out)
    n = sorted_anchors.numel()
    if x.numel() != n or x.dtype != sorted_anchors.dtype:
        raise LaplexError(EINVAL, "x must have n elements and the anchors' dtype")
    y = torch.empty_like(x) if out is None else out
    ws, nb = _ws(OP_SYM_PLANNED, n, 0, 1, x.dtype, dev)
    _check(lib().laplex_matvec_sym_planned(_ptr(sorted_anchors), _ptr(perm), _ptr(inv), n, _ptr(x), _ptr(y),
                                           _dt(x), _ptr(ws), nb, _stream(dev)))
    return y


def matvec_general(sa, sb, x, pa=None, pb=None, transpose=False, out=None):
    """y = K x (x on the b side) or, with transpose, y = K^T x (x on the a side)."""
    dev = _dev(sa, sb, x, _perm(pa), _perm(pb), out)
    n, k = sa.numel(), sb.numel()
    B = 1 if x.dim() == 1 else x.shape[1]
    nin, nout = (n, k) if transpose else (k, n)
    if x.shape[0] != nin:
        raise LaplexError(EINVAL, f"x must have {nin} rows")
    y = torch.empty((nout,) + tuple(x.shape[1:]), dtype=x.dtype, device=dev) if out is None else out
    ws, nb = _ws(OP_GENERAL, n, k, B, x.dtype, dev)
    _check(lib().laplex_matvec_general(_ptr(sa), _ptr(pa), n, _ptr(sb), _ptr(pb), k, _ptr(x),
                                       _ptr(y), B, int(bool(transpose)), _dt(x), _ptr(ws), nb,
                                       _stream(dev)))
    return y


def matvec_phased(sa, phi, x, pa=None, sb=None, psi=None, pb=None, transpose=False, out=None):
    """Phased product, K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j); sb=None: b = a."""
    dev = _dev(sa, phi, x, _perm(pa), sb, psi, _perm(pb), out)
    n = sa.numel()
    k = 0 if sb is None else sb.numel()
    B = 1 if x.dim() == 1 else x.shape[1]
    nout = n if sb is None else (k if transpose else n)
    y = torch.empty((nout,) + tuple(x.shape[1:]), dtype=x.dtype, device=dev) if out is None else out
    ws, nb = _ws(OP_PHASED, n, k, B, x.dtype, dev)
    _check(lib().laplex_matvec_phased(_ptr(sa), _ptr(pa), _ptr(phi), n, _ptr(sb), _ptr(pb),
                                      _ptr(psi), k, _ptr(x), _ptr(y), B, int(bool(transpose)),
                                      _dt(x), _ptr(ws), nb, _stream(dev)))
    return y


def gram(sa, v, pa=None, phi=None, D=None, sb=None, pb=None, psi=None, out=None):
    """z = K^T diag(D) K v (D = 1 when None); sb=None: symmetric K."""
    dev = _dev(sa, v, _perm(pa), phi, D, sb, _perm(pb), psi, out)
    n = sa.numel()
    k = 0 if sb is None else sb.numel()
    B = 1 if v.dim() == 1 else v.shape[1]
    z = torch.empty_like(v) if out is None else out
    ws, nb = _ws(OP_GRAM, n, k, B, v.dtype, dev)
    _check(lib().laplex_gram(_ptr(sa), _ptr(pa), _ptr(phi), n, _ptr(sb), _ptr(pb), _ptr(psi), k,
                             _ptr(D), _ptr(v), _ptr(z), B, _dt(v), _ptr(ws), nb, _stream(dev)))
    return z


def backward(sorted_anchors, x, g, perm=None, dx_out=None, da_out=None):
    """(dx, da) of L = <g, K x>: dx = K g, da = dL/da (sign(0) = 0 at ties)."""
    dev = _dev(sorted_anchors, x, g, _perm(perm), dx_out, da_out)
    n = sorted_anchors.numel()
    dx = torch.empty_like(x) if dx_out is None else dx_out
    da = torch.empty_like(x) if da_out is None else da_out
    ws, nb = _ws(OP_BACKWARD, n, 0, 1, x.dtype, dev)
    _check(lib().laplex_backward(_ptr(sorted_anchors), _ptr(perm), n, _ptr(x), _ptr(g), _ptr(dx),
                                 _ptr(da), _dt(x), _ptr(ws), nb, _stream(dev)))
    return dx, da


def backward_general(sa, sb, x, g, pa=None, pb=None):
    """(dx, da, db) of L = <g, K x>, K_ij = exp(-|a_i - b_j|): dx = K^T g and the
    anchor gradients (sign(0) = 0 at ties).  g, da follow pa; x, dx, db follow pb."""
    dev = _dev(sa, sb, x, g, _perm(pa), _perm(pb))
    n, k = sa.numel(), sb.numel()
    dx = torch.empty_like(x)
    da = torch.empty_like(g)
    db = torch.empty_like(x)
    ws, nb = _ws(OP_BACKWARD_GENERAL, n, k, 1, x.dtype, dev)
    _check(lib().laplex_backward_general(_ptr(sa), _ptr(pa), n, _ptr(sb), _ptr(pb), k, _ptr(x), _ptr(g),
                                         _ptr(dx), _ptr(da), _ptr(db), _dt(x), _ptr(ws), nb,
                                         _stream(dev)))
    return dx, da, db


def backward_phased(sa, phi, x, g, pa=None, sb=None, psi=None, pb=None):
    """Gradients of L = <g, K x>, K_ij = exp(-|a_i - b_j|) cos(phi_i - psi_j).

    sb given: (dx, dphi, dpsi, da, db); phi, g, dphi, da follow pa, and psi, x,
    dx, dpsi, db follow pb.  sb None (b = a, psi = phi): (dx, dphi, da) with the
    shared anchors' and phases' total gradients."""
    dev = _dev(sa, phi, x, g, _perm(pa), sb, psi, _perm(pb))
    n = sa.numel()
    sym = sb is None
    k = n if sym else sb.numel()
    dx, dphi, da = torch.empty_like(x), torch.empty_like(g), torch.empty_like(g)
    dpsi = None if sym else torch.empty_like(x)
    db = None if sym else torch.empty_like(x)
    ws, nb = _ws(OP_BACKWARD_PHASED, n, k, 1, x.dtype, dev)
    # a NULL sb selects the symmetric case: an empty b side gets a non-NULL
    # pointer (the workspace's; nothing is read from it when k = 0)
    sbp = _ptr(sb) if sym or k > 0 else _ptr(ws)
    _check(lib().laplex_backward_phased(_ptr(sa), _ptr(pa), _ptr(phi), n, sbp, _ptr(pb), _ptr(psi), k,
                                        _ptr(x), _ptr(g), _ptr(dx), _ptr(dphi), _ptr(dpsi), _ptr(da), _ptr(db),
                                        _dt(x), _ptr(ws), nb, _stream(dev)))
    return (dx, dphi, da) if sym else (dx, dphi, dpsi, da, db)


def gram_matrix(sa, sb, D=None, pa=None, pb=None, out=None):
    """M = A diag(D) A^T, A_ij = exp(-|a_i - b_j|), as an [n, n] tensor (rows and
    columns follow pa; sorted order without it).  D follows pb; None means 1."""
    dev = _dev(sa, sb, D, _perm(pa), _perm(pb), out)
    n, k = sa.numel(), sb.numel()
    M = torch.empty((n, n), dtype=sa.dtype, device=dev) if out is None else out
    ws, nb = _ws(OP_GRAM_MATRIX, n, k, 1, sa.dtype, dev)
    _check(lib().laplex_gram_matrix(_ptr(sa), _ptr(pa), n, _ptr(sb), _ptr(pb), k, _ptr(D), _ptr(M),
                                    M.stride(0) if n else max(n, 1), _dt(sa), _ptr(ws), nb, _stream(dev)))
    return M


def matvec_sym_noalloc(sorted_anchors: torch.Tensor, x: torch.Tensor, perm=None, out=None):
    """y = K x through laplex_matvec_sym_noalloc: fp32, x of shape [n], n <= 2^30.

    For callers that cannot give the library a workspace: the scratch is a fixed
    array inside the library (shared by all calls on a device, so calls that may
    overlap on the GPU must be serialised by the caller)."""
    dev = _dev(sorted_anchors, x, _perm(perm), out)
    if x.dtype != torch.float32 or x.dim() != 1:
        raise LaplexError(EINVAL, "matvec_sym_noalloc takes fp32 x of shape [n]")
    n = sorted_anchors.numel()
    y = torch.empty_like(x) if out is None else out
    _check(lib().laplex_matvec_sym_noalloc(_ptr(sorted_anchors), _ptr(perm), n, _ptr(x), _ptr(y),
                                           _stream(dev)))
    return y


# ----------------------------------------------------------------------------- host buffers

def matvec_sym_host(sorted_anchors: torch.Tensor, x: torch.Tensor, perm=None, device="cuda",
                    out=None):
    """End-to-end symmetric product from HOST tensors: copies the inputs to the device
    (non-blocking from pinned memory), runs laplex_matvec_sym, copies y back."""
    s_d = sorted_anchors.to(device, non_blocking=True)
    x_d = x.to(device, non_blocking=True)
    p_d = None if perm is None else perm.to(device, non_blocking=True)
    y_d = matvec_sym(s_d, x_d, p_d)
    if out is None:
        return y_d.cpu()
    out.copy_(y_d, non_blocking=True)
    return out


class HostStreamer:
    """Symmetric products of a stream of host batches (pinned tensors), with the
    copies overlapped: batch k's host-to-device copy runs on one CUDA stream
    while batch k-1 is computed on a second and batch k-2's result returns on a
    third.  Device buffers are double-buffered; events order each buffer's
    reuse.  Only copies and laplex_matvec_sym calls are enqueued (no host-side
    arithmetic).

    submit(sorted_h, x_h, y_h, perm_h=None) enqueues one batch and returns at
    once; y_h is complete after synchronize()."""

    def __init__(self, n: int, B: int = 1, dtype=torch.float32, device="cuda", with_perm=False):
        self.dev = torch.device(device)
        self.n, self.B = n, B
        shape = (n,) if B == 1 else (n, B)
        self.h2d = torch.cuda.Stream(self.dev)
        self.comp = torch.cuda.Stream(self.dev)
        self.d2h = torch.cuda.Stream(self.dev)
        self.bufs = []
        for _ in range(2):
            self.bufs.append({
                "s": torch.empty(n, dtype=dtype, device=self.dev),
                "x": torch.empty(shape, dtype=dtype, device=self.dev),
                "y": torch.empty(shape, dtype=dtype, device=self.dev),
                "p": torch.empty(n, dtype=torch.int32, device=self.dev) if with_perm else None,
                "loaded": torch.cuda.Event(), "computed": torch.cuda.Event(),
                "drained": torch.cuda.Event()})
        self.k = 0

    def submit(self, sorted_h, x_h, y_h, perm_h=None):
        b = self.bufs[self.k % 2]
        with torch.cuda.stream(self.h2d):
            self.h2d.wait_event(b["computed"])  # s, x, p free once the product that read them is done
            b["s"].copy_(sorted_h, non_blocking=True)
            b["x"].copy_(x_h, non_blocking=True)
            if perm_h is not None:
                b["p"].copy_(perm_h, non_blocking=True)
            b["loaded"].record(self.h2d)
        with torch.cuda.stream(self.comp):
            self.comp.wait_event(b["loaded"])
            self.comp.wait_event(b["drained"])  # y free once its last copy back is done
            matvec_sym(b["s"], b["x"], b["p"] if perm_h is not None else None, out=b["y"])
            b["computed"].record(self.comp)
        with torch.cuda.stream(self.d2h):
            self.d2h.wait_event(b["computed"])
            y_h.copy_(b["y"], non_blocking=True)
            b["drained"].record(self.d2h)
        self.k += 1

    def synchronize(self):
        """Wait for every submitted batch; raise if a product recorded a device error."""
        torch.cuda.synchronize(self.dev)
        with torch.cuda.stream(self.comp):
            Workspace.status(self.dev)
