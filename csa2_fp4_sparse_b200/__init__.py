"""CSA2 FP4 sparse decode on B200 (sm_100a).

The decode path runs in the CUDA kernels of ``libcsa2.so`` behind the C ABI in
``include/csa2.h``; this package is its thin ctypes binding (``_lib``) plus the
in-tree build (``build``).  PyTorch, where the caller uses it, only provides
device memory and streams.
"""
from ._lib import *  # noqa: F401,F403
from ._lib import EXPORTED, check, lib  # noqa: F401
