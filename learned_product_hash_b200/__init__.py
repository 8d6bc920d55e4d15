"""learned_product_hash_b200: learned product-hash routed attention (forward)
on B200 (sm_100a), behind the C ABI of include/mdr.h.

The Python surface is the ctypes binding in ``mdr`` (same names as the C
entry points).  Importing this package does not load the CUDA library; the
first binding call does, and raises if it has not been built.
"""
from . import mdr  # noqa: F401
