"""Chunkwise linear-recurrence layer (linear attention, scalar-gated linear
attention, gated delta rule) for B200 / sm_100a.

The compute lives in the C-ABI library ``libsf.so`` built from ``csrc/``;
``sf`` is the thin ctypes binding with the same entry-point names.  Importing
this package does not load the library: ``from
chunked_linear_recurrence_chunkwise_b200 import sf`` does, and fails loudly if
it has not been built.
"""
__all__ = ["inputs", "sf"]
