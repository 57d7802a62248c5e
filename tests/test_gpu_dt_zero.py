"""Tokens with dt = 0 on the GPU: the decay is exp(0 * A) = 1 and the input term dt B x^T
vanishes, so such a token leaves the state exactly as it was and its output is
y_t = C_t^T H + D x_t with the unchanged state.  The chunked method relies on this for
the padding of a partial chunk ("Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching for Inference", section "2. Metodologia": chunks of a fixed size).

Runs of dt = 0 are placed at the sequence start, across the 128- and 256-token block
boundaries, and at the end, on both tensor-core prefill paths and the fp32 CUDA-core
path, and in single decode steps.  Each case is checked against the fp64 oracle (which
takes the recurrence literally) and against the identity itself: the final state of a
prefill whose last tokens have dt = 0 equals the final state of the prefill without them.
"""
import dataclasses

import numpy as np
import pytest
import torch

import oracle
from parity import (assert_bf16_y, assert_fp32, assert_state, gpu_prefill, oracle_prefill, problem,
                    to_dev)
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu

ZERO_RUNS = [(0, 5), (120, 140), (250, 262), (383, 385)]


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


@pytest.fixture(params=["fused", "two_pass"])
def tc_path(request):
    import state_space_model_05_b200 as ssd
    prev = ssd.ssd_set_prefill_path(request.param)
    yield request.param
    ssd.ssd_set_prefill_path(prev)


def _with_zero_runs(inp, T, tail):
    for a, b in ZERO_RUNS:
        inp.dt[:, a:min(b, T)] = 0.0
    inp.dt[:, T - tail:] = 0.0
    return inp


def _head(inp, T):
    """The same problem cut to its first T tokens."""
    return dataclasses.replace(inp, x=inp.x[:, :T].copy(), dt=inp.dt[:, :T].copy(), B=inp.B[:, :T].copy(),
                               C=inp.C[:, :T].copy())


@pytest.mark.parametrize("Q", [128, 256])
def test_bf16_dt_zero_runs(Q, tc_path):
    T, tail = 600, 40
    inp = _with_zero_runs(problem(gen.SSDShape(2, T, 4, 64, 1, 128), bf16=True, seed=31), T, tail)
    y, st = gpu_prefill(inp, Q, bf16=True)
    yo, so = oracle_prefill(inp)
    assert_bf16_y(y, oracle.units_to_bthp(yo, 2, 4), "y with dt = 0 runs")
    assert_state(st, so.reshape(st.shape), "state with dt = 0 runs")
    # the trailing dt = 0 tokens leave the state where the prefill of the rest left it
    _, st_head = gpu_prefill(_head(inp, T - tail), Q, bf16=True)
    assert_state(st, st_head, "final state unchanged by trailing dt = 0 tokens")


def test_fp32_dt_zero_runs():
    T, tail = 400, 16
    inp = _with_zero_runs(problem(gen.SSDShape(2, T, 4, 64, 1, 64), bf16=False, seed=32), T, tail)
    for Q in (64, 100):
        y, st = gpu_prefill(inp, Q, bf16=False)
        yo, so = oracle_prefill(inp)
        assert_fp32(y, oracle.units_to_bthp(yo, 2, 4), f"y with dt = 0 runs, Q={Q}")
        assert_fp32(st, so.reshape(st.shape), f"state with dt = 0 runs, Q={Q}")
        _, st_head = gpu_prefill(_head(inp, T - tail), Q, bf16=False)
        assert_fp32(st, st_head, f"final state unchanged by trailing dt = 0 tokens, Q={Q}")


def test_decode_dt_zero_leaves_state_bitwise():
    from state_space_model_05_b200 import ssd_decode_step
    b, H, P, N = 4, 8, 64, 128
    shape = gen.SSDShape(b, 1, H, P, 1, N)
    st0 = gen.state_inputs(b, H, P, N, seed=33)
    dec = gen.decode_inputs(shape, steps=1, seed=34)
    head = gen.prefill_inputs(shape, seed=35)
    dt = dec.dt[0].copy()
    dt[:, ::2] = 0.0                             # every other head of every batch row
    state = to_dev(st0)
    y = ssd_decode_step(state, to_dev(dec.x[0]), to_dev(dt), to_dev(head.A), to_dev(dec.B[0]),
                        to_dev(dec.C[0]), to_dev(head.D))
    torch.cuda.synchronize()
    got = state.cpu().numpy()
    # dt = 0: a = exp(0) = 1 and dt B x = 0, so the fp32 state is bit for bit what it was
    assert np.array_equal(got[:, ::2], st0[:, ::2])
    ref = st0.reshape(b * H, P, N).astype(np.float64)
    yo = oracle.decode_step(ref, dec.x[0], dt, head.A, dec.B[0], dec.C[0], head.D)
    assert_fp32(y.cpu().numpy().reshape(b * H, P), yo, "decode y with dt = 0 heads")
    assert_fp32(got.reshape(b * H, P, N), ref, "decode state with dt = 0 heads")
    # and y of those heads is C^T H + D x with the unchanged state
    C = dec.C[0][:, 0].astype(np.float64)                       # [b][N]
    want = np.einsum("bhpn,bn->bhp", st0.astype(np.float64), C) + head.D[None, :, None] * dec.x[0]
    assert_fp32(y.cpu().numpy()[:, ::2], want[:, ::2], "decode y = C^T H + D x at dt = 0")
