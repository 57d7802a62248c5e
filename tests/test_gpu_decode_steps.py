"""ssd_decode_steps: k decode steps of one layer in one launch.

The page's cache is advanced on the device by a compiled loop with no host round trip per
token ("Compiler-First State Space Duality and Portable O(1) Autoregressive Caching for
Inference", section "2. Metodologia").  For tokens whose inputs are on the device, one
launch runs the whole loop; it must give exactly what k launches of ssd_decode_step give
(same arithmetic per row, so bitwise), and match the fp64 oracle stepped k times.
Covered: the register-resident kernel (headdim <= 64 and <= 128, dstate <= 128), the
looped kernel (dstate 256), bf16 inputs, odd small shapes, grouped B/C and steps = 0.
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
    (2, 6, 128, 2, 128, 20, torch.float32),     # register-resident, 16 rows a warp
    (3, 4, 64, 1, 256, 9, torch.float32),       # looped kernel (state too large for registers)
    (2, 4, 8, 2, 16, 50, torch.float32),        # small odd shape, lanes without a quad
    (4, 8, 64, 1, 128, 24, torch.bfloat16),     # bf16 inputs and outputs
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
