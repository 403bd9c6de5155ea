"""Loader of the oracle's C row quantizers (quant_rows.c) -- TEST
INFRASTRUCTURE ONLY.  build() compiles them with gcc next to this file; load()
returns the library, or None when it cannot be built, in which case the oracle
uses its numpy quantizers (same results, slower)."""

import ctypes
import os
import subprocess

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(HERE, "quant_rows.c")
LIB = os.path.join(HERE, "_quant_rows.so")
_lib = None


def build(force=False):
    if not force and os.path.exists(LIB) and os.path.getmtime(LIB) >= os.path.getmtime(SRC):
        return LIB
    subprocess.run(["gcc", "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math", "-shared",
                    "-fPIC", "-o", LIB, SRC, "-lm"], check=True)
    return LIB


def load():
    global _lib
    if _lib is None:
        try:
            build()
            L = ctypes.CDLL(LIB)
        except (OSError, subprocess.CalledProcessError):
            _lib = False
            return None
        dp = ctypes.POINTER(ctypes.c_double)
        L.oracle_mxfp8_qdq_rows.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_int64]
        L.oracle_mxfp8_qdq_rows.restype = None
        L.oracle_nvfp4_qdq_rows.argtypes = [dp, dp, ctypes.c_int64, ctypes.c_int64, ctypes.c_float]
        L.oracle_nvfp4_qdq_rows.restype = None
        _lib = L
    return _lib or None
