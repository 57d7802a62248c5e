"""HostPrefill: batches in pinned host memory through ssd_prefill with the copies in and
out overlapped (two device buffer sets, one stream per copy direction).

Every batch must come back exactly as a direct ssd_prefill of the same inputs on the
device gives it (same kernels, same inputs: bitwise), including across the reuse of each
buffer set, and the first batch is checked against the fp64 oracle as well.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_bf16_y, assert_state, problem, to_dev
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


def _pinned(a, dtype):
    return torch.from_numpy(np.ascontiguousarray(a)).to(dtype).pin_memory()


@pytest.mark.parametrize("with_init", [False, True])
def test_pipelined_batches_equal_direct_calls(with_init):
    from state_space_model_05_b200 import ssd_prefill
    from state_space_model_05_b200.host_pipeline import HostPrefill
    shape = gen.SSDShape(2, 700, 8, 64, 1, 128)
    bf = torch.bfloat16
    probs = [problem(shape, bf16=True, seed=40 + i) for i in range(5)]
    rng = np.random.default_rng(41)
    inits = [(0.05 * rng.standard_normal((2, 8, 64, 128))).astype(np.float32) for _ in probs]
    A, D = to_dev(probs[0].A), to_dev(probs[0].D)
    for p in probs:                                   # one layer: the same A and D for every batch
        p.A, p.D = probs[0].A, probs[0].D
    pipe = HostPrefill(2, 700, 8, 64, 1, 128, 256, bf, A, D)
    outs = []
    for p, init in zip(probs, inits):
        y = torch.empty((2, 700, 8, 64), dtype=bf).pin_memory()
        st = torch.empty((2, 8, 64, 128), dtype=torch.float32).pin_memory()
        ev = pipe.submit(_pinned(p.x, bf), _pinned(p.dt, torch.float32), _pinned(p.B, bf), _pinned(p.C, bf),
                         y, st, init_state=_pinned(init, torch.float32) if with_init else None)
        outs.append((y, st, ev))
    pipe.synchronize()
    for i, ((y, st, ev), p, init) in enumerate(zip(outs, probs, inits)):
        assert ev.query()
        yd, sd = ssd_prefill(to_dev(p.x, bf), to_dev(p.dt), A, to_dev(p.B, bf), to_dev(p.C, bf), D, 256,
                             init_state=to_dev(init) if with_init else None)
        torch.cuda.synchronize()
        assert torch.equal(y, yd.cpu()), f"batch {i}: y differs from the direct call"
        assert torch.equal(st, sd.cpu()), f"batch {i}: state differs from the direct call"
    yo, so = oracle.prefill(probs[0].x, probs[0].dt, probs[0].A, probs[0].B, probs[0].C, probs[0].D,
                            init=inits[0].reshape(16, 64, 128) if with_init else None)
    assert_bf16_y(outs[0][0].float().numpy(), oracle.units_to_bthp(yo, 2, 8), "pipelined y")
    assert_state(outs[0][1].numpy(), so.reshape(2, 8, 64, 128), "pipelined state")
