"""fp64 CPU oracle for the Gated DeltaNet decode step -- TEST INFRASTRUCTURE.

Only ``tests/`` and the benchmark's CPU-baseline leg may import this module.  It wraps
the plain C step in ``gdn_oracle.c``; the CUDA library never calls it and shares no
code with it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "gdn_oracle.c")
_LIB = os.path.join(_HERE, "libgdn_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, fp64, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def bind(path: str):
    lib = ctypes.CDLL(path)
    P, I = ctypes.c_void_p, ctypes.c_int
    lib.gdn_oracle_decode_step.argtypes = [P, P, P, P, P, P, I, I, I, I, I, P, I]
    lib.gdn_oracle_decode_step.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = bind(_LIB)
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def decode_step(state, q, k, v, gate, beta, nthreads: int = 0, lib=None):
    """One token, in place on ``state`` (fp64 [b][hv][dk][dv]).

    q, k [b][hqk][dk]; v [b][hv][dv]; gate, beta [b][hv].  Returns the output
    [b][hv][dv] (fp64).
    """
    lib = lib or _load()
    q, k, v, gate, beta = map(_f32, (q, k, v, gate, beta))
    b, hqk, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    assert state.dtype == np.float64 and state.flags.c_contiguous and state.shape == (b, hv, dk, dv)
    out = np.empty((b, hv, dv), dtype=np.float64)
    p = lambda a: a.ctypes.data_as(ctypes.c_void_p)
    rc = lib.gdn_oracle_decode_step(p(state), p(q), p(k), p(v), p(gate), p(beta), b, hqk, hv, dk, dv,
                                    p(out), int(nthreads))
    if rc != 0:
        raise ValueError("gdn_oracle_decode_step: bad sizes")
    return out
