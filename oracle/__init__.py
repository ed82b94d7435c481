"""LAPLEX oracle package -- TEST INFRASTRUCTURE, not part of the product.

Only tests/, ``__graft_entry__.smoke()`` and the CPU-baseline leg of bench.py
may import this package.  The product (``exact_laplace_b200``) never does.
"""
from .oracle import *  # noqa: F401,F403
from .oracle import CUTOFF_F64, max_norm_err  # noqa: F401
