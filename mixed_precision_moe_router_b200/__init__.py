"""Tiered mixed-precision MoE layer for B200 (sm_100a).

The compute lives in a C-ABI shared library (``libmoe_tiered.so``, built from
``csrc/``); :mod:`.binding` marshals arguments to it.  Importing this package
does not load the library; :func:`binding.lib` does, and raises if it is
missing.
"""
__all__ = ["inputs", "binding"]
