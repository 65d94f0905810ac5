"""ctypes loader for the oracle's C core (oracle/core.c).

Test infrastructure only.  The shared object is built with plain gcc; the CUDA
path neither links nor imports it.
"""
import ctypes
import os
import subprocess
import threading

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "core.c")
_LIB = os.path.join(_HERE, "liboracle.so")
_lock = threading.Lock()
_lib = None

_u64p = ctypes.POINTER(ctypes.c_uint64)


def build(force=False):
    """Compile core.c into liboracle.so next to it (gcc, -O2, no fast-math)."""
    if not force and os.path.exists(_LIB) and os.path.getmtime(_LIB) >= os.path.getmtime(_SRC):
        return _LIB
    tmp = _LIB + ".%d.tmp" % os.getpid()
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-fPIC", "-shared", "-o", tmp, _SRC])
    os.replace(tmp, _LIB)
    return _LIB


def lib():
    global _lib
    with _lock:
        if _lib is None:
            build()
            L = ctypes.CDLL(_LIB)
            L.ora_powmod.restype = ctypes.c_uint64
            L.ora_powmod.argtypes = [ctypes.c_uint64] * 3
            L.ora_ntt_fwd.restype = None
            L.ora_ntt_fwd.argtypes = [_u64p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64]
            L.ora_ntt_inv.restype = None
            L.ora_ntt_inv.argtypes = [_u64p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64]
            L.ora_vec_mul.restype = None
            L.ora_vec_mul.argtypes = [_u64p, _u64p, _u64p, ctypes.c_size_t, ctypes.c_uint64]
            L.ora_vec_scale.restype = None
            L.ora_vec_scale.argtypes = [_u64p, ctypes.c_uint64, _u64p, ctypes.c_size_t, ctypes.c_uint64]
            L.ora_base_conv.restype = None
            L.ora_base_conv.argtypes = [_u64p, ctypes.c_int, _u64p, _u64p, _u64p, ctypes.c_int,
                                        _u64p, _u64p, ctypes.c_size_t, ctypes.c_int]
            L.ora_automorph_coeff.restype = None
            L.ora_automorph_coeff.argtypes = [_u64p, _u64p, ctypes.c_int, ctypes.c_uint64, ctypes.c_uint64]
            _lib = L
    return _lib


def ptr(a):
    assert a.dtype == np.uint64 and a.flags["C_CONTIGUOUS"]
    return a.ctypes.data_as(_u64p)
