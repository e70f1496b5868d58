"""B200 (sm_100a) Hymba hybrid-head layer: C ABI (libhymba.so) and its Python binding.

The compute path is entirely in the CUDA library; this package only loads it
and marshals arguments.  See include/hymba.h for the contract of every call.
"""
from ._abi import *  # noqa: F401,F403
from ._abi import EXPORTED, LIB_PATH, HymbaError, lib  # noqa: F401
