"""B200 (sm_100a) DLRM hot path: sum-pooled embedding bags, the pairwise
dot-product interaction, the bottom/top MLPs and sigmoid, as hand-written
CUDA kernels behind the C ABI of ``libdlrm.so`` (declared in include/dlrm.h).

This package is the thin Python binding of that library (``_abi``) plus a
small model wrapper (``model``). Importing it does not touch the GPU; the
first call loads ``libdlrm.so`` and raises if it is missing.
"""
from ._abi import *  # noqa: F401,F403
from ._abi import DlrmError, MLP, Tables, lib  # noqa: F401
