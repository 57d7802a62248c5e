"""Failure detection without a GPU fault: the library's bounded device waits run against
conditions that never become true, give up after their limit, report SSD_ERR_TIMEOUT
through the device error word, and leave the CUDA context usable."""
import ctypes

import numpy as np
import pytest
import torch

import oracle
from parity import assert_fp32, problem, to_dev
from state_space_model_05_b200 import binding, inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


def test_bounded_waits_time_out_and_report():
    scratch = torch.zeros(4, dtype=torch.int32, device="cuda")
    stream = ctypes.c_void_p(torch.cuda.current_stream().cuda_stream)
    assert binding.ssd_device_status() == 0
    assert binding.lib().ssd_selftest_bounded_waits(ctypes.c_void_p(scratch.data_ptr()), stream) == 0
    assert binding.ssd_device_status() == binding.SSD_ERR_TIMEOUT
    assert scratch[1].item() == 0 and scratch[2].item() == 0      # both waits gave up
    assert binding.ssd_device_status() == 0                         # the word was cleared
    # the context is still usable: a prefill after the timeout matches the oracle
    inp = problem(gen.SSDShape(1, 130, 4, 64, 1, 64), bf16=False, seed=3)
    from state_space_model_05_b200 import ssd_prefill
    y, st = ssd_prefill(to_dev(inp.x), to_dev(inp.dt), to_dev(inp.A), to_dev(inp.B), to_dev(inp.C),
                        to_dev(inp.D), 64)
    yo, so = oracle.prefill(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D)
    assert_fp32(y.cpu().numpy(), oracle.units_to_bthp(yo, 1, 4), "prefill after timeout")
    assert binding.ssd_device_status() == 0
