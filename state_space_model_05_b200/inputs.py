"""Seeded synthetic inputs for the SSD prefill and decode workloads.

This module holds random draws and their distributions only; it contains no
step of the state-space recurrence.  Both the CUDA path (through the tests and
the benchmark) and the fp64 oracle read the arrays it returns, so the two
sides always see identical inputs.

Distributions (the workloads of the Mamba-2-shaped SSD layers):

* ``x ~ N(0, 1)``;
* ``B, C ~ N(0, 1) / sqrt(N)``;
* ``A_h = -exp(U(0, ln 16))`` so ``A_h`` lies in ``[-16, -1]``;
* ``D_h ~ N(0, 1)``;
* prefill ``dt = softplus(z + b_h)`` with ``z ~ N(0, 0.5^2)`` per
  (batch, token, head) and a per-head bias ``b_h = softplus^-1(u_h)`` where
  ``u_h`` is log-uniform in ``[1e-3, 0.1]``;
* decode ``dt_t`` log-uniform in ``[1e-3, 0.1]``, independent per
  (step, batch, head).

Draw order for one prefill problem (numpy ``Generator(PCG64(seed))``):
``A, D, b_h, x, z, B, C``.  Softplus is the positive-dt preprocessing that
precedes the SSD layer; the SSD entry points receive ``dt`` already positive.

All arrays are returned as numpy ``float32``.  When the workload is bf16 the
caller rounds ``x``, ``B`` and ``C`` to bf16 once (``round_bf16``) and both
sides use the rounded values.
"""
from __future__ import annotations

import math
from dataclasses import dataclass

import numpy as np

DT_MIN = 1e-3
DT_MAX = 0.1
A_LOG_MAX = math.log(16.0)


def _softplus(z: np.ndarray) -> np.ndarray:
    return np.logaddexp(0.0, z)


def _softplus_inv(y: np.ndarray) -> np.ndarray:
    # log(exp(y) - 1), written to stay accurate for small y
    return y + np.log(-np.expm1(-y))


@dataclass
class SSDShape:
    batch: int
    seqlen: int
    nheads: int
    headdim: int
    ngroups: int
    dstate: int


@dataclass
class PrefillInputs:
    x: np.ndarray    # [batch][seqlen][nheads][headdim]
    dt: np.ndarray   # [batch][seqlen][nheads], > 0
    A: np.ndarray    # [nheads], < 0
    B: np.ndarray    # [batch][seqlen][ngroups][dstate]
    C: np.ndarray    # [batch][seqlen][ngroups][dstate]
    D: np.ndarray    # [nheads]
    dt_raw: np.ndarray = None   # [batch][seqlen][nheads] fp32: 0.5 z, so dt = softplus(dt_raw + dt_bias)
    dt_bias: np.ndarray = None  # [nheads] fp32: b_h


@dataclass
class DecodeInputs:
    x: np.ndarray    # [steps][batch][nheads][headdim]
    dt: np.ndarray   # [steps][batch][nheads]
    B: np.ndarray    # [steps][batch][ngroups][dstate]
    C: np.ndarray    # [steps][batch][ngroups][dstate]


def head_params(rng: np.random.Generator, nheads: int):
    """A_h, D_h and the dt bias b_h, drawn in that order."""
    A = -np.exp(rng.uniform(0.0, A_LOG_MAX, size=nheads))
    D = rng.standard_normal(nheads)
    u = np.exp(rng.uniform(math.log(DT_MIN), math.log(DT_MAX), size=nheads))
    b = _softplus_inv(u)
    return A.astype(np.float32), D.astype(np.float32), b


def prefill_inputs(shape: SSDShape, seed: int = 0) -> PrefillInputs:
    """One prefill problem; see the module docstring for the recipe."""
    s = shape
    rng = np.random.Generator(np.random.PCG64(seed))
    A, D, bias = head_params(rng, s.nheads)
    x = rng.standard_normal((s.batch, s.seqlen, s.nheads, s.headdim), dtype=np.float32)
    z = rng.standard_normal((s.batch, s.seqlen, s.nheads), dtype=np.float32)
    dt = _softplus(0.5 * z.astype(np.float64) + bias[None, None, :]).astype(np.float32)
    inv = np.float32(1.0 / math.sqrt(s.dstate))
    B = rng.standard_normal((s.batch, s.seqlen, s.ngroups, s.dstate), dtype=np.float32) * inv
    C = rng.standard_normal((s.batch, s.seqlen, s.ngroups, s.dstate), dtype=np.float32) * inv
    return PrefillInputs(x=x, dt=dt, A=A, B=B, C=C, D=D, dt_raw=(0.5 * z).astype(np.float32),
                         dt_bias=bias.astype(np.float32))


def decode_inputs(shape: SSDShape, steps: int, seed: int = 1) -> DecodeInputs:
    """Per-step decode inputs: fresh x_t, B_t, C_t and log-uniform dt_t."""
    s = shape
    rng = np.random.Generator(np.random.PCG64(seed))
    x = rng.standard_normal((steps, s.batch, s.nheads, s.headdim), dtype=np.float32)
    dt = np.exp(rng.uniform(math.log(DT_MIN), math.log(DT_MAX),
                            size=(steps, s.batch, s.nheads))).astype(np.float32)
    inv = np.float32(1.0 / math.sqrt(s.dstate))
    B = rng.standard_normal((steps, s.batch, s.ngroups, s.dstate), dtype=np.float32) * inv
    C = rng.standard_normal((steps, s.batch, s.ngroups, s.dstate), dtype=np.float32) * inv
    return DecodeInputs(x=x, dt=dt, B=B, C=C)


def state_inputs(batch: int, nheads: int, headdim: int, dstate: int, seed: int = 2) -> np.ndarray:
    """An i.i.d. N(0, 1) fp32 state [batch][nheads][headdim][dstate]."""
    rng = np.random.Generator(np.random.PCG64(seed))
    return rng.standard_normal((batch, nheads, headdim, dstate), dtype=np.float32)


@dataclass
class GDNShape:
    batch: int
    heads_qk: int
    heads_v: int
    dk: int
    dv: int


@dataclass
class GDNInputs:
    q: np.ndarray       # [steps][b][hqk][dk] fp32, unit rows
    k: np.ndarray       # [steps][b][hqk][dk] fp32, unit rows
    v: np.ndarray       # [steps][b][hv][dv] fp32
    gate: np.ndarray    # [steps][b][hv] fp32 in [0.85, 1)
    beta: np.ndarray    # [steps][b][hv] fp32 in (0, 1)
    state: np.ndarray   # [b][hv][dk][dv] fp32, the state before the first step


def gdn_inputs(shape: GDNShape, steps: int, seed: int = 3) -> GDNInputs:
    """Seeded Gated DeltaNet decode inputs (draw order q, k, v, gate, beta, state):
    q, k unit vectors (normalised N(0, 1) rows), v ~ N(0, 1), gate ~ U(0.85, 1),
    beta = sigmoid(N(0, 1)), initial state ~ N(0, 0.1^2)."""
    rng = np.random.default_rng(seed)
    b, hqk, hv, dk, dv = shape.batch, shape.heads_qk, shape.heads_v, shape.dk, shape.dv
    unit = lambda a: (a / np.linalg.norm(a, axis=-1, keepdims=True)).astype(np.float32)
    q = unit(rng.standard_normal((steps, b, hqk, dk)))
    k = unit(rng.standard_normal((steps, b, hqk, dk)))
    v = rng.standard_normal((steps, b, hv, dv)).astype(np.float32)
    gate = rng.uniform(0.85, 1.0, (steps, b, hv)).astype(np.float32)
    beta = (1.0 / (1.0 + np.exp(-rng.standard_normal((steps, b, hv))))).astype(np.float32)
    state = (0.1 * rng.standard_normal((b, hv, dk, dv))).astype(np.float32)
    return GDNInputs(q, k, v, gate, beta, state)


def round_bf16(a: np.ndarray) -> np.ndarray:
    """Round fp32 values to the nearest bf16 (ties to even); returned as fp32.

    Every bf16 value is exact in fp32, so the returned array is exactly the
    bf16 tensor the device reads.
    """
    a = np.ascontiguousarray(a, dtype=np.float32)
    u = a.view(np.uint32).astype(np.uint64)
    rounding = ((u >> 16) & 1) + 0x7FFF
    r = ((u + rounding) >> 16) << 16
    # NaN inputs do not occur in these workloads; keep them NaN regardless
    nan = np.isnan(a)
    out = r.astype(np.uint32).view(np.float32).reshape(a.shape)
    if nan.any():
        out = out.copy()
        out[nan] = np.nan
    return out


# --------------------------------------------------------------------------------------
# Counter-based generator for inputs that are drawn on the device (the deep decode
# stack, whose states alone are tens of GB).  Philox4x32-10 (Salmon, Moraes, Dror,
# Shaw, "Parallel random numbers: as easy as 1, 2, 3", SC'11); the device side has its
# own implementation of the same published definition.  Normals are the Irwin-Hall sum
# of twelve 24-bit uniforms, formed in integers so that both sides round identically.
# --------------------------------------------------------------------------------------
PHILOX_M0 = 0xD2511F53
PHILOX_M1 = 0xCD9E8D57
PHILOX_W0 = 0x9E3779B9
PHILOX_W1 = 0xBB67AE85
MASK32 = 0xFFFFFFFF


def philox4x32_10(counter: np.ndarray, key: tuple[int, int]) -> np.ndarray:
    """Philox4x32 with 10 rounds.  counter: uint32 [..., 4] -> uint32 [..., 4]."""
    c = counter.astype(np.uint64)
    c0, c1, c2, c3 = c[..., 0], c[..., 1], c[..., 2], c[..., 3]
    k0 = np.uint64(key[0] & MASK32)
    k1 = np.uint64(key[1] & MASK32)
    m0 = np.uint64(PHILOX_M0)
    m1 = np.uint64(PHILOX_M1)
    mask = np.uint64(MASK32)
    for r in range(10):
        p0 = m0 * c0
        p1 = m1 * c2
        hi0, lo0 = p0 >> np.uint64(32), p0 & mask
        hi1, lo1 = p1 >> np.uint64(32), p1 & mask
        c0, c1, c2, c3 = (hi1 ^ c1 ^ k0) & mask, lo1, (hi0 ^ c3 ^ k1) & mask, lo0
        if r < 9:
            k0 = (k0 + np.uint64(PHILOX_W0)) & mask
            k1 = (k1 + np.uint64(PHILOX_W1)) & mask
    return np.stack([c0, c1, c2, c3], axis=-1).astype(np.uint32)


def philox_normal(stream: int, index: np.ndarray, seed: int) -> np.ndarray:
    """Irwin-Hall N(0,1) approximation for element ``index`` of ``stream``.

    Element i uses counters (i, stream, 0, 0), (i, stream, 1, 0), (i, stream, 2, 0):
    three Philox blocks = twelve 32-bit words, of which the top 24 bits are summed.
    The result is (sum - 6 * 2^24) * 2^-24, rounded once to fp32.
    """
    index = np.asarray(index, dtype=np.uint64)
    total = np.zeros(index.shape, dtype=np.int64)
    for j in range(3):
        ctr = np.zeros(index.shape + (4,), dtype=np.uint32)
        ctr[..., 0] = (index & np.uint64(MASK32)).astype(np.uint32)
        ctr[..., 1] = np.uint32(stream)
        ctr[..., 2] = np.uint32(j)
        ctr[..., 3] = (index >> np.uint64(32)).astype(np.uint32)
        words = philox4x32_10(ctr, (seed & MASK32, (seed >> 32) & MASK32))
        total += (words >> np.uint32(8)).astype(np.int64).sum(axis=-1)
    centred = total - 6 * (1 << 24)
    return (centred.astype(np.float64) * 2.0 ** -24).astype(np.float32)


def philox_uniform_index(stream: int, index: np.ndarray, seed: int, bits: int) -> np.ndarray:
    """An integer in [0, 2^bits) for element ``index`` of ``stream`` (first Philox word)."""
    index = np.asarray(index, dtype=np.uint64)
    ctr = np.zeros(index.shape + (4,), dtype=np.uint32)
    ctr[..., 0] = (index & np.uint64(MASK32)).astype(np.uint32)
    ctr[..., 1] = np.uint32(stream)
    ctr[..., 2] = np.uint32(3)
    ctr[..., 3] = (index >> np.uint64(32)).astype(np.uint32)
    words = philox4x32_10(ctr, (seed & MASK32, (seed >> 32) & MASK32))
    return (words[..., 0] >> np.uint32(32 - bits)).astype(np.int64)


DT_TABLE_BITS = 12


def dt_table() -> np.ndarray:
    """2^12 log-uniform levels in [1e-3, 0.1] (midpoints), fp32; indexed by random bits."""
    k = np.arange(1 << DT_TABLE_BITS, dtype=np.float64)
    lo, hi = math.log(DT_MIN), math.log(DT_MAX)
    return np.exp(lo + (k + 0.5) / (1 << DT_TABLE_BITS) * (hi - lo)).astype(np.float32)


# --------------------------------------------------------------------------------------
# Device-side twin of the counter-based generator (libssd_inputs.so, include/ssd_inputs.h),
# for workloads too large to draw on the host.  Same definitions as philox_normal /
# philox_uniform_index above; the two produce bit-identical values.
# --------------------------------------------------------------------------------------
_gen_lib = None


def _gen():
    global _gen_lib
    if _gen_lib is None:
        import ctypes
        import os
        path = os.path.join(os.path.dirname(os.path.abspath(__file__)), "libssd_inputs.so")
        if not os.path.exists(path):
            raise RuntimeError(f"input generator library not built: {path} is missing")
        lib = ctypes.CDLL(path)
        P, Z, U64, U32, F, I = (ctypes.c_void_p, ctypes.c_size_t, ctypes.c_uint64, ctypes.c_uint32,
                                ctypes.c_float, ctypes.c_int)
        lib.ssd_gen_normal.argtypes = [P, Z, U64, U32, F, U64, P]
        lib.ssd_gen_normal.restype = I
        lib.ssd_gen_table.argtypes = [P, Z, P, I, U64, U32, U64, P]
        lib.ssd_gen_table.restype = I
        _gen_lib = lib
    return _gen_lib


def _cuda_stream():
    import ctypes
    import torch
    return ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)


def device_normal(out, seed: int, stream_id: int, scale: float = 1.0, first_index: int = 0):
    """Fill the contiguous fp32 CUDA tensor `out` with philox_normal(stream_id, i) * scale."""
    import ctypes
    rc = _gen().ssd_gen_normal(ctypes.c_void_p(out.data_ptr()), out.numel(), seed, stream_id,
                               float(np.float32(scale)), first_index, _cuda_stream())
    if rc:
        raise RuntimeError(f"ssd_gen_normal failed ({rc})")
    return out


def device_table(out, table, bits: int, seed: int, stream_id: int, first_index: int = 0):
    """Fill `out` with table[philox_uniform_index(stream_id, i, bits)] (table on the device)."""
    import ctypes
    rc = _gen().ssd_gen_table(ctypes.c_void_p(out.data_ptr()), out.numel(),
                              ctypes.c_void_p(table.data_ptr()), bits, seed, stream_id, first_index,
                              _cuda_stream())
    if rc:
        raise RuntimeError(f"ssd_gen_table failed ({rc})")
    return out


# Stream numbering of the deep decode stack (L layers, fresh inputs every step): one
# Philox stream per (tensor, layer, step); element indices follow the tensor's layout.
DEEP_X, DEEP_B, DEEP_C, DEEP_DT, DEEP_STATE = 0, 1, 2, 3, 4
DEEP_SEED = 0


def deep_stream(tensor: int, layer: int, step: int = 0) -> int:
    assert 0 <= tensor < 16 and 0 <= layer < 4096 and 0 <= step < 65536
    return (tensor << 28) | (layer << 16) | step


def deep_head_params(layer: int, nheads: int):
    """A_h, D_h of one layer (host draws, PCG64 seeded by the layer index)."""
    rng = np.random.Generator(np.random.PCG64(1000 + layer))
    A, D, _ = head_params(rng, nheads)
    return A, D


def deep_unit_inputs(layer: int, b: int, h: int, steps: int, shape: SSDShape, seed: int = DEEP_SEED):
    """Host regeneration of one (layer, batch, head) unit of the deep decode stack:
    initial state [P][N], and per step x [P], dt, B [N], C [N]."""
    P, N, H, G = shape.headdim, shape.dstate, shape.nheads, shape.ngroups
    g = h // (H // G)
    st = philox_normal(deep_stream(DEEP_STATE, layer), (b * H + h) * P * N + np.arange(P * N), seed)
    xs, dts, Bs, Cs = [], [], [], []
    inv = np.float32(1.0 / math.sqrt(N))
    table = dt_table()
    for k in range(steps):
        xs.append(philox_normal(deep_stream(DEEP_X, layer, k), (b * H + h) * P + np.arange(P), seed))
        Bs.append(philox_normal(deep_stream(DEEP_B, layer, k), (b * G + g) * N + np.arange(N), seed) * inv)
        Cs.append(philox_normal(deep_stream(DEEP_C, layer, k), (b * G + g) * N + np.arange(N), seed) * inv)
        dts.append(table[philox_uniform_index(deep_stream(DEEP_DT, layer, k), np.array([b * H + h]),
                                              seed, DT_TABLE_BITS)][0])
    return (st.reshape(P, N), np.stack(xs), np.array(dts, dtype=np.float32), np.stack(Bs), np.stack(Cs))
