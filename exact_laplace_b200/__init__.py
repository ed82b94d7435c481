"""exact_laplace_b200: the exact LAPLEX Laplace-kernel operator on NVIDIA B200 (sm_100a).

The compute path is the C-ABI library ``liblaplex.so`` built from ``csrc/``;
``exact_laplace_b200.laplex`` is its thin Python binding.  The library is loaded
on first use and a missing or unloadable library raises; there is no CPU path.
"""
__all__ = ["laplex", "synth"]
