"""The 64-layer deep decode stack (2.7B-shaped layers at batch 256, ~43 GB of fp32 states
resident, 256 steps, fresh inputs per layer and step drawn on the device) against the
fp64 oracle on sampled (layer, batch, head) units.

The inputs come from the counter-based generator; the host twin in inputs.py regenerates
the sampled units' initial states and per-step inputs independently, so no oracle input
comes from the GPU."""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_fp32
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


def test_device_generator_matches_host_twin():
    """Bit-identical values from the device generator and its host twin, including a
    range that crosses the 32-bit boundary of the element counter."""
    inv = float(np.float32(1 / np.sqrt(128)))
    for stream, scale in [(gen.deep_stream(gen.DEEP_X, 3, 17), 1.0),
                          (gen.deep_stream(gen.DEEP_B, 63, 255), inv)]:
        for first, n in [(0, 1000), (2 ** 32 - 3, 10), (123456789012, 5)]:
            out = torch.empty(n, device="cuda")
            gen.device_normal(out, gen.DEEP_SEED, stream, scale, first_index=first)
            want = gen.philox_normal(stream, first + np.arange(n, dtype=np.uint64), gen.DEEP_SEED) * np.float32(scale)
            np.testing.assert_array_equal(out.cpu().numpy(), want)
    table = gen.dt_table()
    t_dev = torch.from_numpy(table).cuda()
    out = torch.empty(5000, device="cuda")
    st = gen.deep_stream(gen.DEEP_DT, 9, 4)
    gen.device_table(out, t_dev, gen.DT_TABLE_BITS, gen.DEEP_SEED, st)
    want = table[gen.philox_uniform_index(st, np.arange(5000), gen.DEEP_SEED, gen.DT_TABLE_BITS)]
    np.testing.assert_array_equal(out.cpu().numpy(), want)


def test_deep_decode_stack_256_steps_sampled():
    import bench
    w = bench.WORKLOADS["deep_decode_2p7b"]
    L, b, H, P, G, N, steps = (w[k] for k in ("layers", "batch", "nheads", "headdim", "ngroups", "dstate", "steps"))
    stack = bench.DeepStack(w)
    rng = np.random.default_rng(5)
    units = [(int(rng.integers(L)), int(rng.integers(b)), int(rng.integers(H))) for _ in range(10)]
    units += [(0, 0, 0), (L - 1, b - 1, H - 1)]
    li = torch.tensor([u[0] for u in units], device="cuda")
    bi = torch.tensor([u[1] for u in units], device="cuda")
    hi = torch.tensor([u[2] for u in units], device="cuda")
    ys = torch.empty((steps, len(units), P), device="cuda")
    for k in range(steps):
        stack.draw(k)
        stack.step()
        ys[k] = stack.y[li, bi, hi]
    torch.cuda.synchronize()
    from state_space_model_05_b200 import ssd_device_status
    assert ssd_device_status() == 0
    st_gpu = stack.states[li, bi, hi].cpu().numpy()
    ys = ys.cpu().numpy()
    shape = gen.SSDShape(b, 1, H, P, G, N)
    for u, (l, bb, h) in enumerate(units):
        st0, xs, dts, Bs, Cs = gen.deep_unit_inputs(l, bb, h, steps, shape)
        A, D = gen.deep_head_params(l, H)
        state = st0.astype(np.float64)[None]
        for k in range(steps):
            yo = oracle.decode_step(state, xs[k][None, None], dts[k:k + 1][None], A[h:h + 1],
                                    Bs[k][None, None], Cs[k][None, None], D[h:h + 1])
            assert_fp32(ys[k, u], yo[0], f"unit {(l, bb, h)} step {k}")
        assert_fp32(st_gpu[u], state[0], f"unit {(l, bb, h)} final state")
    del stack
    torch.cuda.empty_cache()


def _small_stack(one_launch, layers=4, batch=8):
    import bench
    w = dict(bench.WORKLOADS["deep_decode_2p7b"], layers=layers, batch=batch)
    return bench.DeepStack(w, one_launch=one_launch)


def test_one_launch_stack_equals_per_layer_launches():
    """The stack in one launch does exactly the per-layer steps: bitwise equal states and y."""
    a, b = _small_stack(True), _small_stack(False)
    for k in range(5):
        a.draw(k)
        b.draw(k)
        a.step()
        b.step()
        torch.cuda.synchronize()
        assert torch.equal(a.y, b.y), f"y step {k}"
    assert torch.equal(a.states, b.states)
    from state_space_model_05_b200 import ssd_device_status
    assert ssd_device_status() == 0


def test_one_launch_stack_skips_and_reports_bad_entries():
    """An entry with a misaligned or NULL pointer is skipped and recorded in the device error
    word (checked on the device before any access); the other layers are stepped."""
    from state_space_model_05_b200 import binding, ssd_device_status
    a, b = _small_stack(True), _small_stack(False)
    a.draw(0)
    b.draw(0)
    before = a.states.clone()
    table = a.layers.clone()
    table[1, 0] += 4                       # layer 1: state pointer off by 4 bytes
    table[2, 7] = 0                        # layer 2: NULL y pointer
    w = a.w
    binding.ssd_decode_step_layers(table, w["batch"], w["nheads"], w["headdim"], w["ngroups"],
                                   w["dstate"], torch.float32)
    status = ssd_device_status()
    assert status in (binding.SSD_ERR_ALIGN, binding.SSD_ERR_NULL)
    assert ssd_device_status() == 0        # reading clears it
    b.step()
    torch.cuda.synchronize()
    for l in (0, 3):
        assert torch.equal(a.states[l], b.states[l]), f"layer {l} stepped"
    for l in (1, 2):
        assert torch.equal(a.states[l], before[l]), f"layer {l} untouched"
