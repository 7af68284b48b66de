"""NOSA decode step on B200: block scoring, locality-bounded selection, miss
gather from pinned host memory and block-sparse GQA attention, as sm_100a CUDA
kernels behind a C ABI (``libnosa.so``).

Importing the package loads nothing native; the binding in ``nosa`` loads the
library on first use and raises if it is missing.
"""

__all__ = ["configs", "inputs"]
