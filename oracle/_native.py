"""Build and load the plain-C twins in oracle/fast.c (test infrastructure only).

The shared object lands in oracle/_build/ (not committed) and is rebuilt when
fast.c is newer.  `lib()` returns None when no C compiler is available; the
numpy definitions then serve alone.
"""
from __future__ import annotations

import ctypes
import os
import shutil
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "fast.c")
_OUT = os.path.join(_HERE, "_build", "liboracle_fast.so")
_lib = None


def build(force: bool = False) -> str:
    os.makedirs(os.path.dirname(_OUT), exist_ok=True)
    if force or not os.path.exists(_OUT) or os.path.getmtime(_OUT) < os.path.getmtime(_SRC):
        cc = shutil.which("gcc") or shutil.which("cc")
        if cc is None:
            raise RuntimeError("no C compiler for the oracle's C twins")
        tmp = _OUT + ".tmp%d" % os.getpid()
        subprocess.check_call([cc, "-O2", "-fopenmp", "-ffp-contract=off", "-fno-fast-math",
                               "-fPIC", "-shared", "-o", tmp, _SRC, "-lm"])
        os.replace(tmp, _OUT)
    return _OUT


def lib():
    global _lib
    if _lib is None:
        try:
            path = build()
        except (RuntimeError, subprocess.CalledProcessError, OSError):
            return None
        L = ctypes.CDLL(path)
        P = ctypes.c_void_p
        L.oc_weights.argtypes = [ctypes.c_uint64, ctypes.c_uint32, ctypes.c_uint64, ctypes.c_uint64,
                                 ctypes.c_int, P]
        L.oc_weights.restype = None
        L.oc_sampler_rows.argtypes = [P, ctypes.c_int64, ctypes.c_int64, ctypes.c_uint64, ctypes.c_uint32,
                                      ctypes.c_uint32, ctypes.c_uint32, ctypes.c_float, P, P, P, P, P, P]
        L.oc_sampler_rows.restype = None
        _lib = L
    return _lib


def ptr(a: np.ndarray):
    return ctypes.c_void_p(a.ctypes.data) if a is not None else None


def weights(seed, tensor_id, start, count, bf16):
    out = np.empty(count, dtype=np.float32)
    lib().oc_weights(seed, tensor_id, start, count, int(bf16), ptr(out))
    return out


def sampler_rows(logits, seed, canvas_id, pos0, step, inv_t, want_probs):
    l = np.ascontiguousarray(logits, dtype=np.float32)
    R, V = l.shape
    H = np.empty(R, np.float32); am = np.empty(R, np.int32); tok = np.empty(R, np.int32)
    sq = np.empty(R, np.int64); uq = np.empty(R, np.int64)
    probs = np.empty_like(l) if want_probs else None
    lib().oc_sampler_rows(ptr(l), R, V, seed, canvas_id, pos0, step, float(inv_t), ptr(H), ptr(am),
                          ptr(tok), ptr(sq), ptr(uq), ptr(probs))
    return dict(H=H, amax=am, tokens=tok, S_q=sq, U_q=uq, p=probs)
