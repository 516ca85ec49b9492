"""Build and load the plain-C oracle (``oracle/c/pagedkv_oracle.c``) — test
infrastructure only, like the rest of this package."""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(_HERE, "c", "pagedkv_oracle.c")
LIB = os.path.join(_HERE, "c", "libpagedkv_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    if force or not os.path.exists(LIB) or os.path.getmtime(LIB) < os.path.getmtime(SRC):
        subprocess.check_call(["gcc", "-O2", "-fopenmp", "-fPIC", "-shared", "-std=c11",
                               "-o", LIB, SRC, "-lm"])
    return LIB


def lib():
    global _lib
    if _lib is None:
        build()
        L = ctypes.CDLL(LIB)
        P = ctypes.c_void_p
        I = ctypes.c_int
        L.oracle_paged_decode.argtypes = [P, P, P, P, P, P, I, I, I, I, I, I, ctypes.c_double, I, I]
        L.oracle_paged_decode.restype = I
        L.oracle_reshape_and_cache.argtypes = [P, P, P, P, P, I, I, I, I]
        L.oracle_reshape_and_cache.restype = I
        L.oracle_num_threads.restype = I
        _lib = L
    return _lib


def _p(a):
    return a.ctypes.data_as(ctypes.c_void_p)


def paged_decode_attention(q, k_cache, v_cache, block_tables, context_lens, scale, dtype,
                           nthreads=0):
    q = np.ascontiguousarray(q, dtype=np.uint16)
    k_cache = np.ascontiguousarray(k_cache, dtype=np.uint16)
    v_cache = np.ascontiguousarray(v_cache, dtype=np.uint16)
    bt = np.ascontiguousarray(block_tables, dtype=np.int32)
    lens = np.ascontiguousarray(context_lens, dtype=np.int32)
    B, Hq, d = q.shape
    _, Hkv, bs, _ = k_cache.shape
    out = np.empty((B, Hq, d), dtype=np.float64)
    rc = lib().oracle_paged_decode(_p(out), _p(q), _p(k_cache), _p(v_cache), _p(bt), _p(lens),
                                   B, Hq, Hkv, d, bs, bt.shape[1], float(scale), int(dtype),
                                   int(nthreads))
    if rc != 0:
        raise RuntimeError(f"oracle_paged_decode failed: {rc}")
    return out


def reshape_and_cache(k_new, v_new, k_cache, v_cache, slot_mapping):
    """Returns written copies of the caches."""
    kc = np.array(k_cache, dtype=np.uint16, copy=True, order="C")
    vc = np.array(v_cache, dtype=np.uint16, copy=True, order="C")
    kn = np.ascontiguousarray(k_new, dtype=np.uint16)
    vn = np.ascontiguousarray(v_new, dtype=np.uint16)
    sm = np.ascontiguousarray(slot_mapping, dtype=np.int64)
    T, Hkv, d = kn.shape
    lib().oracle_reshape_and_cache(_p(kn), _p(vn), _p(kc), _p(vc), _p(sm), T, Hkv, d, kc.shape[2])
    return kc, vc


def num_threads():
    return int(lib().oracle_num_threads())
