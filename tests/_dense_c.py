"""Loader for the plain-C dense attention used to pin the NumPy oracle."""
import ctypes
import os
import subprocess

import numpy as np

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
SRC = os.path.join(ROOT, "oracle", "dense_attention.c")
LIB = os.path.join(ROOT, "oracle", "libdense_attention.so")

_lib = None


def build(force=False):
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-shared", "-fPIC", SRC, "-o", LIB, "-lm"])
    return LIB


def lib():
    global _lib
    if _lib is None:
        _lib = ctypes.CDLL(build())
        dp = ctypes.POINTER(ctypes.c_double)
        _lib.dense_attention.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_double, dp]
        _lib.dense_causal_chunk.argtypes = [dp, dp, dp, ctypes.c_int, ctypes.c_int, ctypes.c_int,
                                            ctypes.c_double, dp]
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.POINTER(ctypes.c_double))


def dense_attention(q, K, V, scale):
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    out = np.zeros(V.shape[1] if V.ndim == 2 else q.shape[0], dtype=np.float64)
    lib().dense_attention(_p(q), _p(K), _p(V), K.shape[0], q.shape[0], scale, _p(out))
    return out


def dense_causal_chunk(q, K, V, scale):
    q = np.ascontiguousarray(q, dtype=np.float64)
    K = np.ascontiguousarray(K, dtype=np.float64)
    V = np.ascontiguousarray(V, dtype=np.float64)
    n, D = q.shape
    out = np.zeros((n, D), dtype=np.float64)
    lib().dense_causal_chunk(_p(q), _p(K), _p(V), K.shape[0], n, D, scale, _p(out))
    return out
