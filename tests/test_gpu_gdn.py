"""GPU parity of the Gated DeltaNet decode step against the fp64 oracle, over many
successive steps on seeded inputs.

Workloads: the page's model shape at batch 1 (16 query/key heads, 32 value heads,
dk = dv = 128, a 2 MB fp32 state), a larger batch, grouped and ungrouped heads,
non-square states, bf16 inputs, and a CUDA graph of steps.
"""
import numpy as np
import pytest
import torch

from oracle import gdn
from parity import assert_bf16_y, assert_fp32, assert_state
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    gdn.build()


def _dev(a, dtype=torch.float32):
    return torch.from_numpy(np.ascontiguousarray(a)).to("cuda", dtype)


def _run(shape, steps, bf16=False, seed=3):
    import state_space_model_05_b200 as ssd
    inp = gen.gdn_inputs(shape, steps, seed=seed)
    if bf16:
        inp.q, inp.k, inp.v = gen.round_bf16(inp.q), gen.round_bf16(inp.k), gen.round_bf16(inp.v)
    dt_ = torch.bfloat16 if bf16 else torch.float32
    state = _dev(inp.state)
    ref = inp.state.astype(np.float64)
    outs, want = [], []
    for t in range(steps):
        q, k, v = _dev(inp.q[t], dt_), _dev(inp.k[t], dt_), _dev(inp.v[t], dt_)
        o = ssd.ssd_gdn_decode_step(state, q, k, v, _dev(inp.gate[t]), _dev(inp.beta[t]))
        outs.append(o.float().cpu().numpy())
        want.append(gdn.decode_step(ref, inp.q[t], inp.k[t], inp.v[t], inp.gate[t], inp.beta[t]))
    torch.cuda.synchronize()
    assert ssd.ssd_device_status() == 0
    return np.stack(outs), np.stack(want), state.cpu().numpy(), ref


def test_page_shape_batch1_64_steps():
    """16 query/key heads, 32 value heads, dk = dv = 128 (2 MB of fp32 state), batch 1."""
    o, w, st, ref = _run(gen.GDNShape(1, 16, 32, 128, 128), 64)
    assert_fp32(o, w, "gdn out")
    assert_fp32(st, ref, "gdn state")


@pytest.mark.parametrize("shape", [gen.GDNShape(4, 4, 8, 64, 128), gen.GDNShape(3, 2, 2, 128, 64),
                                   gen.GDNShape(2, 1, 3, 8, 4), gen.GDNShape(5, 8, 16, 128, 128)])
def test_shapes_16_steps(shape):
    o, w, st, ref = _run(shape, 16, seed=shape.dk + shape.dv)
    assert_fp32(o, w, f"gdn out {shape}")
    assert_fp32(st, ref, f"gdn state {shape}")


def test_degenerate_gates():
    """Per value head, the rule's limiting cases side by side: g = 0 (the old state is wiped and
    replaced by beta k v^T), g = 1 with beta = 0 (the state passes unchanged and o = S^T q), and
    beta = 1 (the full delta rule: S^T k becomes v after the step)."""
    import state_space_model_05_b200 as ssd
    shape = gen.GDNShape(2, 2, 4, 64, 64)
    inp = gen.gdn_inputs(shape, 3, seed=21)
    inp.gate[:] = np.array([0.0, 1.0, 0.9, 0.5], dtype=np.float32)
    inp.beta[:] = np.array([0.7, 0.0, 1.0, 1.0], dtype=np.float32)
    state = _dev(inp.state)
    ref = inp.state.astype(np.float64)
    for t in range(3):
        o = ssd.ssd_gdn_decode_step(state, _dev(inp.q[t]), _dev(inp.k[t]), _dev(inp.v[t]), _dev(inp.gate[t]),
                                    _dev(inp.beta[t]))
        want = gdn.decode_step(ref, inp.q[t], inp.k[t], inp.v[t], inp.gate[t], inp.beta[t])
        assert_fp32(o.cpu().numpy(), want, f"gdn degenerate out step {t}")
    torch.cuda.synchronize()
    assert ssd.ssd_device_status() == 0
    assert_fp32(state.cpu().numpy(), ref, "gdn degenerate state")
    # beta = 1 heads: after the last step S^T k equals v (unit-norm k)
    st = state.cpu().numpy().astype(np.float64)
    for bb in range(2):
        for h in (2, 3):
            kk = inp.k[2][bb, h // 2].astype(np.float64)
            np.testing.assert_allclose(st[bb, h].T @ kk, inp.v[2][bb, h], rtol=1e-4, atol=1e-4)


def test_bf16_inputs():
    o, w, st, ref = _run(gen.GDNShape(2, 16, 32, 128, 128), 32, bf16=True, seed=9)
    assert_bf16_y(o, w, "gdn out bf16")
    assert_state(st, ref, "gdn state (bf16 inputs)")


def test_graph_of_steps_matches_eager():
    """A CUDA graph of 32 steps (fresh device inputs per step) gives the eager result."""
    import state_space_model_05_b200 as ssd
    shape, steps = gen.GDNShape(2, 16, 32, 128, 128), 32
    inp = gen.gdn_inputs(shape, steps, seed=11)
    q, k, v = _dev(inp.q), _dev(inp.k), _dev(inp.v)
    g, bt = _dev(inp.gate), _dev(inp.beta)
    s_eager, s_graph = _dev(inp.state), _dev(inp.state)
    out_e = torch.empty_like(v)
    out_g = torch.empty_like(v)
    for t in range(steps):
        ssd.ssd_gdn_decode_step(s_eager, q[t], k[t], v[t], g[t], bt[t], out=out_e[t])
    torch.cuda.synchronize()
    stream = torch.cuda.Stream()
    graph = torch.cuda.CUDAGraph()
    with torch.cuda.graph(graph, stream=stream):
        for t in range(steps):
            ssd.ssd_gdn_decode_step(s_graph, q[t], k[t], v[t], g[t], bt[t], out=out_g[t])
    graph.replay()
    torch.cuda.synchronize()
    assert torch.equal(out_e, out_g) and torch.equal(s_eager, s_graph)
    assert ssd.ssd_device_status() == 0


def test_empty_batch_is_a_no_op():
    import state_space_model_05_b200 as ssd
    z = lambda *s: torch.zeros(s, device="cuda")
    out = ssd.ssd_gdn_decode_step(z(0, 32, 128, 128), z(0, 16, 128), z(0, 16, 128), z(0, 32, 128), z(0, 32),
                                  z(0, 32))
    assert out.shape == (0, 32, 128)
