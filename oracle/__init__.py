"""fp64 CPU oracle for the SSD recurrence -- TEST INFRASTRUCTURE.

Only ``tests/``, ``__graft_entry__.smoke()`` and the benchmark's CPU-baseline
leg may import this package.  The CUDA library never calls it and shares no
code with it.

``prefill`` and ``decode_step`` wrap the plain C recurrence in
``ssd_oracle.c`` (token by token, fp64).  ``forms`` holds the separately
written chunked and quadratic forms that pin it.
"""
from __future__ import annotations

import ctypes
import os
import subprocess

import numpy as np

_HERE = os.path.dirname(os.path.abspath(__file__))
_SRC = os.path.join(_HERE, "ssd_oracle.c")
_LIB = os.path.join(_HERE, "libssd_oracle.so")
_lib = None


def build(force: bool = False) -> str:
    """Compile the C oracle (gcc, fp64, OpenMP, no FMA contraction)."""
    if force or not os.path.exists(_LIB) or os.path.getmtime(_LIB) < os.path.getmtime(_SRC):
        subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fno-fast-math",
                               "-fopenmp", "-fPIC", "-shared", "-o", _LIB, _SRC, "-lm"])
    return _LIB


def bind(path: str):
    """Load a compiled oracle library from ``path`` and declare its signatures."""
    lib = ctypes.CDLL(path)
    P = ctypes.c_void_p
    I = ctypes.c_int
    lib.ssd_oracle_prefill.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, I, P, I, P, P, I]
    lib.ssd_oracle_prefill.restype = I
    lib.ssd_oracle_decode_step.argtypes = [P, P, P, P, P, P, P, I, I, I, I, I, P, I, P, I]
    lib.ssd_oracle_decode_step.restype = I
    lib.ssd_oracle_threads.argtypes = [I]
    lib.ssd_oracle_threads.restype = I
    return lib


def _load():
    global _lib
    if _lib is None:
        build()
        _lib = bind(_LIB)
    return _lib


def _f32(a):
    return np.ascontiguousarray(a, dtype=np.float32)


def _ptr(a):
    return None if a is None else a.ctypes.data_as(ctypes.c_void_p)


def softplus_dt(dt_raw, dt_bias=None):
    """dt = softplus(dt_raw + dt_bias[h]) in fp64, softplus(z) = log(1 + exp(z)), in the
    overflow-free form max(z, 0) + log1p(exp(-|z|)).  dt_raw [..][H], dt_bias [H] or None."""
    z = np.asarray(dt_raw, dtype=np.float64)
    if dt_bias is not None:
        z = z + np.asarray(dt_bias, dtype=np.float64)
    return np.maximum(z, 0.0) + np.log1p(np.exp(-np.abs(z)))


def threads(nthreads: int = 0) -> int:
    return _load().ssd_oracle_threads(int(nthreads))


def prefill(x, dt, A, B, C, D, init=None, units=None, nthreads: int = 0, lib=None):
    """Sequential fp64 prefill.

    x [b][T][H][P], dt [b][T][H], A [H], B/C [b][T][G][N], D [H]; ``init`` is
    [n_units][P][N] (fp64) or None; ``units`` lists (b * H + h) indices or None
    for all of them.  Returns ``y`` [n_units][T][P] and ``state``
    [n_units][P][N], both fp64.
    """
    lib = lib or _load()
    x, dt, A, B, C, D = map(_f32, (x, dt, A, B, C, D))
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    if units is None:
        n_units = b * H
        units_arr = None
    else:
        units_arr = np.ascontiguousarray(units, dtype=np.int32)
        n_units = units_arr.size
    if init is not None:
        init = np.ascontiguousarray(init, dtype=np.float64).reshape(n_units, P, N)
    y = np.empty((n_units, T, P), dtype=np.float64)
    state = np.empty((n_units, P, N), dtype=np.float64)
    rc = lib.ssd_oracle_prefill(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                _ptr(init), b, T, H, P, G, N, _ptr(units_arr), n_units,
                                _ptr(y), _ptr(state), int(nthreads))
    if rc != 0:
        raise ValueError("oracle prefill: invalid shape")
    return y, state


def decode_step(state, x_t, dt_t, A, B_t, C_t, D, units=None, nthreads: int = 0, lib=None):
    """One fp64 decode step; ``state`` [n_units][P][N] fp64 is updated in place.

    x_t [b][H][P], dt_t [b][H], B_t/C_t [b][G][N].  Returns y_t [n_units][P].
    """
    lib = lib or _load()
    x_t, dt_t, A, B_t, C_t, D = map(_f32, (x_t, dt_t, A, B_t, C_t, D))
    b, H, P = x_t.shape
    G, N = B_t.shape[1], B_t.shape[2]
    if units is None:
        n_units = b * H
        units_arr = None
    else:
        units_arr = np.ascontiguousarray(units, dtype=np.int32)
        n_units = units_arr.size
    if not (state.dtype == np.float64 and state.flags.c_contiguous and
            state.shape == (n_units, P, N)):
        raise ValueError("oracle decode: state must be contiguous fp64 [n_units][P][N]")
    y = np.empty((n_units, P), dtype=np.float64)
    rc = lib.ssd_oracle_decode_step(_ptr(state), _ptr(x_t), _ptr(dt_t), _ptr(A), _ptr(B_t),
                                    _ptr(C_t), _ptr(D), b, H, P, G, N, _ptr(units_arr),
                                    n_units, _ptr(y), int(nthreads))
    if rc != 0:
        raise ValueError("oracle decode: invalid shape")
    return y


def units_to_bthp(y_units, batch, nheads):
    """[b*H][T][P] (all units in order) -> [b][T][H][P]."""
    n, T, P = y_units.shape
    return y_units.reshape(batch, nheads, T, P).transpose(0, 2, 1, 3)
