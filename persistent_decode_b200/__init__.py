"""Persistent single-kernel small-batch decode for B200 (sm_100a).

The compute path is the C-ABI library libxlpk.so (include/xlpk.h); this
package only marshals arguments to it.  The library is loaded on first use
and its absence raises ImportError: there is no CPU fallback.
"""
from ._abi import LIB_PATH, load  # noqa: F401
from .engine import Engine, XlpkError, get_lib, lib, tc_gemm_tile  # noqa: F401
