"""CPU oracle for the RNS-CKKS engine: plain, slow and written to be checked by eye.

TEST INFRASTRUCTURE ONLY.  The only code allowed to import, call or run
anything in this package is tests/, __graft_entry__.smoke() and the CPU
baseline / reference leg of bench.py.  The CUDA library never links it and
never falls back to it.
"""
from . import ckks  # noqa: F401
from ._core import build  # noqa: F401
