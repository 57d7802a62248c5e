"""ssd_decode_steps: k decode steps of one layer in one launch.

The page's cache is advanced on the device by a compiled loop with no host round trip per
token ("Compiler-First State Space Duality and Portable O(1) Autoregressive Caching for
Inference", section "2. Metodologia").  For tokens whose inputs are on the device, one
launch runs the whole loop; it must give exactly what k launches of ssd_decode_step give
(same arithmetic per row, so bitwise), and match the fp64 oracle stepped k times.
Covered: the register-resident kernel (headdim <= 64 and <= 128, dstate <= 128; one head a
CTA, or two heads of a group when the units exceed a wave), the
looped kernel (dstate 256), bf16 inputs, odd small shapes, grouped B/C and steps = 0; and
ssd_decode_steps_layers, the same loop over every layer of a table in one launch (bitwise
equal to the per-layer call, oracle-checked, a bad entry skipped and reported).
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_fp32, to_dev
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


def _case(b, H, P, G, N, steps, seed, dtype=torch.float32):
    shape = gen.SSDShape(b, 1, H, P, G, N)
    dec = gen.decode_inputs(shape, steps=steps, seed=seed)
    head = gen.prefill_inputs(shape, seed=seed + 1)
    st0 = gen.state_inputs(b, H, P, N, seed=seed + 2)
    if dtype == torch.bfloat16:
        dec.x, dec.B, dec.C = gen.round_bf16(dec.x), gen.round_bf16(dec.B), gen.round_bf16(dec.C)
    return dec, head, st0


@pytest.mark.parametrize("b,H,P,G,N,steps,dtype", [
    (4, 8, 64, 1, 128, 37, torch.float32),      # register-resident, 2.7B head shape
    (2, 6, 64, 2, 128, 15, torch.float32),      # three heads a group: one head a CTA
    (8, 64, 64, 1, 128, 9, torch.float32),      # 512 units, more than a wave: two heads a CTA
    (8, 64, 64, 4, 128, 7, torch.bfloat16),     # the same in bf16, four groups
    (2, 6, 128, 2, 128, 20, torch.float32),     # register-resident, 16 rows a warp
    (3, 4, 64, 1, 256, 9, torch.float32),       # looped kernel (state too large for registers)
    (2, 4, 8, 2, 16, 50, torch.float32),        # small odd shape, lanes without a quad
    (4, 8, 64, 1, 128, 24, torch.bfloat16),     # bf16 inputs and outputs
    (2, 4, 128, 1, 64, 11, torch.bfloat16),     # 16 rows a warp with dstate < 128 (absent quads)
])
def test_steps_equal_single_step_launches_bitwise(b, H, P, G, N, steps, dtype):
    from state_space_model_05_b200 import ssd_decode_step, ssd_decode_steps
    dec, head, st0 = _case(b, H, P, G, N, steps, seed=50 + P + N + steps, dtype=dtype)
    A, D = to_dev(head.A), to_dev(head.D)
    X, DT, Bs, Cs = to_dev(dec.x, dtype), to_dev(dec.dt), to_dev(dec.B, dtype), to_dev(dec.C, dtype)
    s1 = to_dev(st0)
    y1 = torch.empty_like(X)
    for k in range(steps):
        ssd_decode_step(s1, X[k], DT[k], A, Bs[k], Cs[k], D, y_t=y1[k])
    s2 = to_dev(st0)
    y2 = ssd_decode_steps(s2, X, DT, A, Bs, Cs, D)
    torch.cuda.synchronize()
    assert torch.equal(y1, y2), "y differs from single-step launches"
    assert torch.equal(s1, s2), "state differs from single-step launches"
    if dtype == torch.float32:
        ref = st0.reshape(b * H, P, N).astype(np.float64)
        for k in range(steps):
            yo = oracle.decode_step(ref, dec.x[k], dec.dt[k], head.A, dec.B[k], dec.C[k], head.D)
            assert_fp32(y2[k].cpu().numpy().reshape(b * H, P), yo, f"decode_steps y, step {k}")
        assert_fp32(s2.cpu().numpy().reshape(b * H, P, N), ref, "decode_steps final state")


def test_zero_steps_leave_state_untouched():
    from state_space_model_05_b200 import ssd_decode_steps
    dec, head, st0 = _case(2, 4, 64, 1, 128, 1, seed=7)
    s = to_dev(st0)
    x = torch.empty((0, 2, 4, 64), device="cuda")
    y = ssd_decode_steps(s, x, torch.empty((0, 2, 4), device="cuda"), to_dev(head.A),
                         torch.empty((0, 2, 1, 128), device="cuda"), torch.empty((0, 2, 1, 128), device="cuda"),
                         to_dev(head.D))
    torch.cuda.synchronize()
    assert y.shape == (0, 2, 4, 64)
    assert np.array_equal(s.cpu().numpy(), st0)


def _stack(nl, b, H, P, G, N, steps, dtype, seed):
    """nl layers of one shape: per-layer tensors for the table, and what ssd_decode_steps
    gives for each layer on its own (copies of the same start states)."""
    from state_space_model_05_b200 import ssd_decode_steps
    layers, refs = [], []
    for l in range(nl):
        dec, head, st0 = _case(b, H, P, G, N, steps, seed=seed + 10 * l, dtype=dtype)
        X, DT, Bs, Cs = to_dev(dec.x, dtype), to_dev(dec.dt), to_dev(dec.B, dtype), to_dev(dec.C, dtype)
        A, D = to_dev(head.A), to_dev(head.D)
        layers.append(dict(state=to_dev(st0), x_t=X, dt_t=DT, A=A, B_t=Bs, C_t=Cs, D=D, y_t=torch.full_like(X, 7.0)))
        s_ref = to_dev(st0)
        refs.append((s_ref, ssd_decode_steps(s_ref, X, DT, A, Bs, Cs, D), dec, head, st0))
    return layers, refs


@pytest.mark.parametrize("P,N,dtype,H", [
    (64, 128, torch.float32, 4),       # register-resident, one row per lane group
    (64, 128, torch.float32, 96),      # 576 units over the layers: two heads a CTA
    (128, 128, torch.bfloat16, 4),     # register-resident, two rows per lane group, bf16
    (64, 256, torch.float32, 4),       # looped kernel
    (64, 32, torch.float32, 4),        # dstate < 128: lanes with absent quads
])
def test_stack_steps_equal_per_layer_calls_bitwise(P, N, dtype, H):
    """ssd_decode_steps_layers advances every layer of a table by k tokens in one launch:
    bit for bit what ssd_decode_steps gives per layer (itself bitwise equal to k single
    steps, above), and for fp32 within tolerance of the oracle stepped k times."""
    from state_space_model_05_b200 import decode_layer_table, ssd_decode_steps_layers, ssd_device_status
    b, G, steps, nl = 2, 2, 13, 3
    layers, refs = _stack(nl, b, H, P, G, N, steps, dtype, seed=300 + P + N)
    ssd_decode_steps_layers(decode_layer_table(layers), steps, b, H, P, G, N, dtype)
    assert ssd_device_status() == 0
    for l, (layer, (s_ref, y_ref, dec, head, st0)) in enumerate(zip(layers, refs)):
        assert torch.equal(layer["y_t"], y_ref), f"layer {l}: y differs from ssd_decode_steps"
        assert torch.equal(layer["state"], s_ref), f"layer {l}: state differs from ssd_decode_steps"
    if dtype == torch.float32:
        layer, (_, _, dec, head, st0) = layers[1], refs[1]
        ref = st0.reshape(b * H, P, N).astype(np.float64)
        for k in range(steps):
            yo = oracle.decode_step(ref, dec.x[k], dec.dt[k], head.A, dec.B[k], dec.C[k], head.D)
            assert_fp32(layer["y_t"][k].cpu().numpy().reshape(b * H, P), yo, f"stack steps y, step {k}")
        assert_fp32(layer["state"].cpu().numpy().reshape(b * H, P, N), ref, "stack steps final state")


def test_stack_steps_bad_entry_skipped_and_reported():
    """A table entry with a NULL pointer is skipped (its state and y untouched) and reported
    through the device error word; the other layers are still advanced."""
    from state_space_model_05_b200 import decode_layer_table, ssd_decode_steps_layers, ssd_device_status
    b, H, P, G, N, steps = 2, 4, 64, 1, 128, 5
    layers, refs = _stack(3, b, H, P, G, N, steps, torch.float32, seed=900)
    table = decode_layer_table(layers)
    table[1, 0] = 0                                   # layer 1: NULL state pointer
    s1_before = layers[1]["state"].clone()
    ssd_decode_steps_layers(table, steps, b, H, P, G, N, torch.float32)
    assert ssd_device_status() == 1                   # SSD_ERR_NULL
    assert torch.equal(layers[1]["state"], s1_before)
    assert bool((layers[1]["y_t"] == 7.0).all())
    for l in (0, 2):
        assert torch.equal(layers[l]["y_t"], refs[l][1])
        assert torch.equal(layers[l]["state"], refs[l][0])
