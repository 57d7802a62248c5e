"""GPU parity of ssd_decode_step against the fp64 oracle.

Workloads: the fp32 single layer (prefill 256 tokens, then 16 decode steps with
fresh inputs) and the 2.7B-shaped cached decode (batch 64, 80 heads, P 64, N 128,
state seeded by a 512-token prefill, 1024 steps; sampled (batch, head) units are
checked at every step).  The oracle computes its own prefill and decode from the
same seeded inputs; nothing of the GPU's is fed back to it.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_bf16_y, assert_fp32, gpu_prefill, oracle_prefill, problem, to_dev
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


def _decode_dev(dec, k, dtype=torch.float32):
    return (to_dev(dec.x[k], dtype), to_dev(dec.dt[k]), to_dev(dec.B[k], dtype), to_dev(dec.C[k], dtype))


def test_fp32_layer_prefill_then_16_steps():
    from state_space_model_05_b200 import ssd_decode_step
    s = gen.SSDShape(1, 256, 4, 64, 1, 64)
    inp = problem(s, bf16=False, seed=0)
    dec = gen.decode_inputs(s, steps=16, seed=1)
    _, st = gpu_prefill(inp, 64, bf16=False)
    state = to_dev(st)
    A, D = to_dev(inp.A), to_dev(inp.D)
    _, so = oracle_prefill(inp)
    for k in range(16):
        x, dt, B, C = _decode_dev(dec, k)
        y = ssd_decode_step(state, x, dt, A, B, C, D)
        yo = oracle.decode_step(so, dec.x[k], dec.dt[k], inp.A, dec.B[k], dec.C[k], inp.D)
        assert_fp32(y.cpu().numpy().reshape(4, 64), yo, f"y step {k}")
    assert_fp32(state.cpu().numpy().reshape(4, 64, 64), so, "state after 16 steps")


def test_prefill_then_decode_equals_longer_prefill_gpu():
    """prefill(256) + 16 decode steps == prefill(272), all on the GPU."""
    from state_space_model_05_b200 import ssd_decode_step
    inp = problem(gen.SSDShape(1, 272, 4, 64, 1, 64), bf16=False, seed=0)
    y_full, s_full = gpu_prefill(inp, 64, bf16=False)
    head = gen.PrefillInputs(inp.x[:, :256], inp.dt[:, :256], inp.A, inp.B[:, :256], inp.C[:, :256], inp.D)
    _, st = gpu_prefill(head, 64, bf16=False)
    state = to_dev(st)
    for k in range(256, 272):
        y = ssd_decode_step(state, to_dev(inp.x[:, k]), to_dev(inp.dt[:, k]), to_dev(inp.A),
                            to_dev(inp.B[:, k]), to_dev(inp.C[:, k]), to_dev(inp.D))
        assert_fp32(y.cpu().numpy(), y_full[:, k], f"token {k}")
    assert_fp32(state.cpu().numpy(), s_full, "state")


@pytest.mark.parametrize("b,H,P,G,N", [(3, 6, 24, 3, 40), (2, 4, 64, 2, 256), (1, 2, 16, 1, 512),
                                       (5, 8, 128, 1, 128), (4, 4, 64, 4, 64)])
def test_fp32_decode_shapes(b, H, P, G, N):
    from state_space_model_05_b200 import ssd_decode_step
    s = gen.SSDShape(b, 1, H, P, G, N)
    rng = np.random.default_rng(b * 100 + N)
    st0 = rng.standard_normal((b, H, P, N)).astype(np.float32)
    inp = problem(s, bf16=False, seed=N)
    dec = gen.decode_inputs(s, steps=3, seed=N + 1)
    state = to_dev(st0)
    so = st0.reshape(b * H, P, N).astype(np.float64)
    for k in range(3):
        x, dt, B, C = _decode_dev(dec, k)
        y = ssd_decode_step(state, x, dt, to_dev(inp.A), B, C, to_dev(inp.D))
        yo = oracle.decode_step(so, dec.x[k], dec.dt[k], inp.A, dec.B[k], dec.C[k], inp.D)
        assert_fp32(y.cpu().numpy().reshape(b * H, P), yo, f"y step {k}")
    assert_fp32(state.cpu().numpy().reshape(b * H, P, N), so, "state")


def test_fp32_decode_strong_decay():
    """Per-step decays from exp(-32) (the state almost fully replaced) to exp(-1.6e-5) (barely
    touched), next to each other in one call."""
    from state_space_model_05_b200 import ssd_decode_step
    b, H, P, N = 2, 4, 64, 128
    s = gen.SSDShape(b, 1, H, P, 1, N)
    rng = np.random.default_rng(77)
    st0 = rng.standard_normal((b, H, P, N)).astype(np.float32)
    inp = problem(s, bf16=False, seed=78)
    A = np.array([-16.0, -16.0, -0.5, -4.0], dtype=np.float32)
    dec = gen.decode_inputs(s, steps=4, seed=79)
    dec.dt[:] = np.array([2.0, 0.1, 3e-5, 0.05], dtype=np.float32)
    state = to_dev(st0)
    so = st0.reshape(b * H, P, N).astype(np.float64)
    for k in range(4):
        x, dt, B, C = _decode_dev(dec, k)
        y = ssd_decode_step(state, x, dt, to_dev(A), B, C, to_dev(inp.D))
        yo = oracle.decode_step(so, dec.x[k], dec.dt[k], A, dec.B[k], dec.C[k], inp.D)
        assert_fp32(y.cpu().numpy().reshape(b * H, P), yo, f"y step {k}")
    assert_fp32(state.cpu().numpy().reshape(b * H, P, N), so, "state")


def test_bf16_decode_io():
    from state_space_model_05_b200 import ssd_decode_step
    s = gen.SSDShape(4, 1, 8, 64, 1, 128)
    rng = np.random.default_rng(7)
    st0 = (rng.standard_normal((4, 8, 64, 128)) * 0.1).astype(np.float32)
    inp = problem(s, bf16=False, seed=3)
    dec = gen.decode_inputs(s, steps=4, seed=4)
    dec.x, dec.B, dec.C = gen.round_bf16(dec.x), gen.round_bf16(dec.B), gen.round_bf16(dec.C)
    state = to_dev(st0)
    so = st0.reshape(32, 64, 128).astype(np.float64)
    for k in range(4):
        x, dt, B, C = _decode_dev(dec, k, torch.bfloat16)
        y = ssd_decode_step(state, x, dt, to_dev(inp.A), B, C, to_dev(inp.D))
        yo = oracle.decode_step(so, dec.x[k], dec.dt[k], inp.A, dec.B[k], dec.C[k], inp.D)
        assert_bf16_y(y.float().cpu().numpy().reshape(32, 64), yo, f"bf16 y step {k}", tol=1e-4)
    assert_fp32(state.cpu().numpy().reshape(32, 64, 128), so, "state")


def test_graph_captured_steps_match_eager():
    from state_space_model_05_b200 import ssd_decode_step
    s = gen.SSDShape(8, 1, 16, 64, 1, 128)
    rng = np.random.default_rng(8)
    st0 = rng.standard_normal((8, 16, 64, 128)).astype(np.float32)
    inp = problem(s, bf16=False, seed=5)
    dec = gen.decode_inputs(s, steps=8, seed=6)
    A, D = to_dev(inp.A), to_dev(inp.D)
    ins = [_decode_dev(dec, k) for k in range(8)]
    eager = to_dev(st0)
    ye = [ssd_decode_step(eager, *ins[k][:1], ins[k][1], A, ins[k][2], ins[k][3], D).clone() for k in range(8)]
    graphed = to_dev(st0)
    ys = [torch.empty_like(ins[0][0]) for _ in range(8)]
    side = torch.cuda.Stream()
    side.wait_stream(torch.cuda.current_stream())
    g = torch.cuda.CUDAGraph()
    with torch.cuda.stream(side):
        with torch.cuda.graph(g, stream=side):
            for k in range(8):
                ssd_decode_step(graphed, ins[k][0], ins[k][1], A, ins[k][2], ins[k][3], D, y_t=ys[k])
    g.replay()
    torch.cuda.synchronize()
    assert torch.equal(graphed, eager)
    for k in range(8):
        assert torch.equal(ys[k], ye[k])


def test_27b_cached_decode_1024_steps_sampled():
    """2.7B-shaped cached decode at full size: b=64, H=80, P=64, N=128, state seeded by a
    512-token fp32 prefill, 1024 steps with fresh inputs; sampled units checked every step."""
    from state_space_model_05_b200 import ssd_decode_step
    b, H, P, N, steps = 64, 80, 64, 128, 1024
    s_pre = gen.SSDShape(b, 512, H, P, 1, N)
    inp = problem(s_pre, bf16=False, seed=0)
    dec = gen.decode_inputs(gen.SSDShape(b, 1, H, P, 1, N), steps=steps, seed=1)
    _, st = gpu_prefill(inp, 64, bf16=False)
    state = to_dev(st)
    A, D = to_dev(inp.A), to_dev(inp.D)
    X, DT, Bs, Cs = to_dev(dec.x), to_dev(dec.dt), to_dev(dec.B), to_dev(dec.C)
    rng = np.random.default_rng(1)
    units = sorted(rng.choice(b * H, size=12, replace=False).tolist())
    uidx = torch.tensor(units, device="cuda")
    ys = torch.empty((steps, len(units), P), device="cuda")
    y = torch.empty((b, H, P), device="cuda")
    for k in range(steps):
        ssd_decode_step(state, X[k], DT[k], A, Bs[k], Cs[k], D, y_t=y)
        ys[k] = y.reshape(b * H, P).index_select(0, uidx)
    torch.cuda.synchronize()
    # oracle: its own prefill of the sampled units, then the same 1024 steps
    _, so = oracle_prefill(inp, units=units)
    ys_h = ys.cpu().numpy()
    for k in range(steps):
        yo = oracle.decode_step(so, dec.x[k], dec.dt[k], inp.A, dec.B[k], dec.C[k], inp.D, units=units)
        assert_fp32(ys_h[k], yo, f"y step {k}")
    assert_fp32(state.reshape(b * H, P, N)[uidx].cpu().numpy(), so, "state after 1024 steps")


def test_dt_softplus_folded_into_decode():
    """ssd_decode_step_dtraw: dt_t = softplus(dt_raw_t + dt_bias) formed in the kernel; the
    oracle steps on the fp64 softplus of the same raw values."""
    from state_space_model_05_b200 import ssd_decode_step
    b, H, P, G, N = 3, 8, 64, 2, 128
    s = gen.SSDShape(b, 1, H, P, G, N)
    rng = np.random.default_rng(77)
    st0 = rng.standard_normal((b, H, P, N)).astype(np.float32)
    inp = problem(s, bf16=False, seed=78)
    dec = gen.decode_inputs(s, steps=4, seed=79)
    raw = (0.5 * rng.standard_normal((4, b, H))).astype(np.float32)
    bias = inp.dt_bias
    state = to_dev(st0)
    so = st0.reshape(b * H, P, N).astype(np.float64)
    for k in range(4):
        x, _, B, C = _decode_dev(dec, k)
        y = ssd_decode_step(state, x, to_dev(raw[k]), to_dev(inp.A), B, C, to_dev(inp.D), dt_softplus=True,
                            dt_bias=to_dev(bias))
        dt64 = oracle.softplus_dt(raw[k], bias)
        yo = oracle.decode_step(so, dec.x[k], dt64, inp.A, dec.B[k], dec.C[k], inp.D)
        assert_fp32(y.cpu().numpy().reshape(b * H, P), yo, f"dtraw y step {k}")
    assert_fp32(state.cpu().numpy().reshape(b * H, P, N), so, "dtraw state")
