"""ssd_prefill_noalloc, the prefill entry point for callers that cannot allocate device
memory (a framework hook that must stay inside pre-planned memory, or code running
during a CUDA stream capture, where cudaMalloc would break the capture).

Called through the C ABI with raw device pointers, twice in a row on different
inputs, and checked against ssd_prefill (which takes a caller-allocated workspace)
with the tolerances of the other parity tests.  Collected last so that a failure
here cannot hide any other test's result; it also passes when run on its own.
"""
import ctypes

import numpy as np
import pytest
import torch

from parity import BF16_TOL, FP32_TOL, assert_fp32, assert_state, problem, to_dev
from state_space_model_05_b200 import binding, inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()


def _p(t):
    return ctypes.c_void_p(t.data_ptr()) if t is not None else None


def _noalloc(args, y, st):
    x, dt, A, B, C, D, init, dims, code = args
    return binding.lib().ssd_prefill_noalloc(
        _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D), _p(init), *dims, code, _p(y), _p(st),
        ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _with_workspace(args, y, st):
    x, dt, A, B, C, D, init, dims, code = args
    need = binding.ssd_prefill_workspace_bytes(*dims, code)
    ws = torch.empty(max(need, 1), dtype=torch.uint8, device="cuda")
    return binding.lib().ssd_prefill(
        _p(x), _p(dt), _p(A), _p(B), _p(C), _p(D), _p(init), *dims, code, _p(y), _p(st), _p(ws),
        ws.numel(), ctypes.c_void_p(torch.cuda.current_stream().cuda_stream))


def _args(shape, Q, bf16, seed, with_init):
    inp = problem(shape, bf16=bf16, seed=seed)
    dt_ = torch.bfloat16 if bf16 else torch.float32
    init = None
    if with_init:
        rng = np.random.default_rng(seed)
        init = to_dev((rng.standard_normal((shape.batch, shape.nheads, shape.headdim, shape.dstate)) * 0.05)
                      .astype(np.float32))
    dims = (shape.batch, shape.seqlen, shape.nheads, shape.headdim, shape.ngroups, shape.dstate, Q)
    code = binding.SSD_BF16 if bf16 else binding.SSD_F32
    return (to_dev(inp.x, dt_), to_dev(inp.dt), to_dev(inp.A), to_dev(inp.B, dt_), to_dev(inp.C, dt_),
            to_dev(inp.D), init, dims, code)


def _run_both(args):
    x = args[0]
    b, T, H, P = x.shape
    N = args[3].shape[3]
    y0, y1 = torch.empty_like(x), torch.empty_like(x)
    s0 = torch.empty((b, H, P, N), device="cuda")
    s1 = torch.empty_like(s0)
    assert _with_workspace(args, y0, s0) == 0
    assert _noalloc(args, y1, s1) == 0
    torch.cuda.synchronize()
    return y0.float().cpu().numpy(), s0.cpu().numpy(), y1.float().cpu().numpy(), s1.cpu().numpy()


@pytest.mark.parametrize("bf16,Q,path", [(True, 256, "two_pass"), (True, 256, "fused"), (False, 64, "two_pass")])
def test_noalloc_matches_workspace_entry_two_calls(bf16, Q, path):
    # 130M-shaped layer (bf16, tensor-core path: both tensor-core prefill paths, which lay
    # the shared buffer out differently) and the fp32 layer shape
    import state_space_model_05_b200 as ssd
    shape = gen.SSDShape(8, 2048, 24, 64, 1, 128) if bf16 else gen.SSDShape(2, 300, 4, 64, 1, 64)
    tol = BF16_TOL if bf16 else FP32_TOL
    prev = ssd.ssd_set_prefill_path(path)
    try:
        for call, (seed, with_init) in enumerate([(0, False), (1, True)]):
            args = _args(shape, Q, bf16, seed, with_init)
            y_ref, s_ref, y, s = _run_both(args)
            assert np.isfinite(y).all() and np.isfinite(s).all()
            assert_fp32(y, y_ref, f"y, call {call}", tol=tol)
            assert_state(s, s_ref, f"state, call {call}", tol=tol)
    finally:
        ssd.ssd_set_prefill_path(prev)
    from state_space_model_05_b200 import ssd_device_status
    assert ssd_device_status() == 0


def test_noalloc_rejects_oversize_before_launch():
    # the 2.7B-shaped long prefill needs far more workspace than the built-in 64 MiB; the
    # size check comes before any pointer is looked at, so no buffer is passed at all
    dims = (4, 16384, 80, 64, 1, 128, 256)
    need = binding.ssd_prefill_workspace_bytes(*dims, binding.SSD_BF16)
    assert need > 64 << 20, need
    st = binding.lib().ssd_prefill_noalloc(None, None, None, None, None, None, None, *dims,
                                           binding.SSD_BF16, None, None, None)
    assert st == 8   # SSD_ERR_WORKSPACE
    from state_space_model_05_b200 import ssd_device_status
    assert ssd_device_status() == 0
