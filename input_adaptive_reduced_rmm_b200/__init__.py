"""Reduced Matrix Multiplication (RMM) on B200: the input-adaptive reduced product.

The compute lives in ``librmm.so`` (CUDA for sm_100a behind a C ABI declared in
``include/rmm.h``).  :mod:`.rmm` is the thin ctypes binding with the same
names; :mod:`.metrics` holds the host-side work formulas.  Importing the
package does not load the library; the first call into :mod:`.rmm` does, and
raises if the library has not been built.
"""
from . import metrics  # noqa: F401

__all__ = ["metrics"]
