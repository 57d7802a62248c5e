"""Why the fp32 relative-error check is taken over elements of at least 1e-1 RMS.

The bound for the fp32 path is "max relative error 1e-4".  A relative error is only
meaningful where the reference is not close to zero: an fp32 evaluation of the chunked
method carries absolute rounding noise of roughly 1e-6 to 1e-5 of the output's RMS, which
is already 1e-4 relative on an element of 1e-2 RMS.  This test shows it with a plain,
correct fp32 evaluation of the chunked algorithm (numpy float32, written out below, no
GPU): on the fp32 parity workloads' seeds it exceeds 1e-4 relative on some state elements
when elements down to 1e-2 RMS are included, and it meets both checks of the reading in
use (relative error over elements >= 1e-1 RMS, and max |error| / RMS over all elements,
each <= 1e-4).  The token-by-token fp32 recurrence meets the reading too.

The chunked method ("Compiler-First State Space Duality and Portable O(1) Autoregressive
Caching for Inference", section "2. Metodologia"): per chunk, the cumulative sum Lam of
dt A; the masked intra-chunk product (L o C B^T)(dt x) with L = exp(Lam_t - Lam_s) below
the diagonal; the carried state's contribution exp(Lam_t) C_t H; the skip D x; and the
state update H <- exp(Lam_end) H + B^T (exp(Lam_end - Lam) dt o x).
"""
import numpy as np
import pytest

import oracle
from parity import FP32_TOL, fp32_errors, rms
from state_space_model_05_b200 import inputs as gen

F = np.float32
# (seqlen, chunk_len) of the fp32 parity tests, each with its seed seqlen + chunk_len
CASES = [(63, 64), (200, 64), (300, 128), (257, 256), (100, 7), (130, 33), (272, 64)]


def chunked_fp32(x, dt, A, B, C, D, Q):
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    y = np.zeros((b, T, H, P), F)
    state = np.zeros((b, H, N, P), F)
    for c0 in range(0, T, Q):
        c1 = min(c0 + Q, T)
        for bi in range(b):
            for h in range(H):
                g = h // (H // G)
                d = dt[bi, c0:c1, h].astype(F)
                lam = np.cumsum((d * F(A[h])).astype(F), dtype=F)
                Bc, Cc, xc = B[bi, c0:c1, g].astype(F), C[bi, c0:c1, g].astype(F), x[bi, c0:c1, h].astype(F)
                L = np.tril(np.exp((lam[:, None] - lam[None, :]).astype(F)).astype(F))
                Y = (((Cc @ Bc.T).astype(F) * L * d[None, :]).astype(F) @ xc).astype(F)
                Y += (np.exp(lam)[:, None] * (Cc @ state[bi, h])).astype(F)
                Y += (F(D[h]) * xc).astype(F)
                y[bi, c0:c1, h] = Y
                w = (np.exp(lam[-1] - lam) * d).astype(F)
                state[bi, h] = (np.exp(lam[-1]) * state[bi, h] + Bc.T @ (w[:, None] * xc)).astype(F)
    return y, state.transpose(0, 1, 3, 2)


def recurrence_fp32(x, dt, A, B, C, D):
    b, T, H, P = x.shape
    G, N = B.shape[2], B.shape[3]
    state = np.zeros((b, H, P, N), F)
    for bi in range(b):
        for h in range(H):
            g = h // (H // G)
            S = np.zeros((P, N), F)
            for t in range(T):
                a = np.exp(F(dt[bi, t, h] * A[h])).astype(F)
                S = (a * S + (F(dt[bi, t, h]) * x[bi, t, h])[:, None] * B[bi, t, g][None, :]).astype(F)
            state[bi, h] = S
    return state


def rel_error(g, o, floor):
    g, o = np.asarray(g, np.float64), np.asarray(o, np.float64)
    big = np.abs(o) >= floor * rms(o)
    return float((np.abs(g - o)[big] / np.abs(o[big])).max())


@pytest.fixture(scope="module")
def results():
    oracle.build()
    out = []
    for T, Q in CASES:
        inp = gen.prefill_inputs(gen.SSDShape(2, T, 4, 64, 2, 64), seed=T + Q)
        y, st = chunked_fp32(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D, Q)
        yo, so = oracle.prefill(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D)
        out.append(((T, Q), inp, y, st, oracle.units_to_bthp(yo, 2, 4), so.reshape(st.shape)))
    return out


def test_fp32_chunked_evaluation_breaks_a_1e2_floor(results):
    worst = max(rel_error(st, so, 1e-2) for _, _, _, st, _, so in results)
    assert worst > FP32_TOL, worst


def test_fp32_chunked_evaluation_meets_the_reading(results):
    for case, _, y, st, yo, so in results:
        for what, g, o in (("y", y, yo), ("state", st, so)):
            rel, nrm = fp32_errors(g, o)
            assert rel <= FP32_TOL and nrm <= FP32_TOL, (case, what, rel, nrm)


def test_fp32_recurrence_meets_the_reading(results):
    for case, inp, _, _, _, so in results[:4]:
        rel, nrm = fp32_errors(recurrence_fp32(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D), so)
        assert rel <= FP32_TOL and nrm <= FP32_TOL, (case, rel, nrm)
