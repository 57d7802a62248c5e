"""GPU parity of ssd_prefill against the fp64 oracle on seeded inputs.

Workloads: the fp32 single SSD layer (batch 1, 256 tokens, 4 heads, P = N = 64,
chunk 64), the Mamba-2-130M-shaped bf16 layer (batch 8, 2048 tokens, 24 heads,
P 64, N 128, chunk 256) and the 2.7B-shaped long bf16 prefill (batch 4, 16384
tokens, 80 heads, chunk 256; sampled (batch, head) units), plus ragged, empty,
grouped, init-state and chunk-length cases.  The bf16 tensor-core cases run on both
tensor-core paths: the fused chain kernel and the two-pass (walk + block output) kernels.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import (assert_bf16_y, assert_fp32, assert_state, gpu_prefill, gpu_units,
                    oracle_prefill, problem, to_dev)
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


@pytest.fixture(params=["fused", "two_pass"])
def tc_path(request):
    """Runs the test once per tensor-core prefill path (process-wide setting, restored)."""
    import state_space_model_05_b200 as ssd
    prev = ssd.ssd_set_prefill_path(request.param)
    yield request.param
    ssd.ssd_set_prefill_path(prev)


def _check_fp32(inp, Q, init=None):
    b, T, H, P = inp.x.shape
    y, st = gpu_prefill(inp, Q, bf16=False, init=init)
    yo, so = oracle_prefill(inp, init=None if init is None else init.reshape(b * H, P, -1))
    assert_fp32(y, oracle.units_to_bthp(yo, b, H), f"y Q={Q}")
    assert_fp32(st, so.reshape(st.shape), f"state Q={Q}")
    return y, st


def _check_bf16(inp, Q, init=None):
    b, T, H, P = inp.x.shape
    y, st = gpu_prefill(inp, Q, bf16=True, init=init)
    yo, so = oracle_prefill(inp, init=None if init is None else init.reshape(b * H, P, -1))
    assert_bf16_y(y, oracle.units_to_bthp(yo, b, H), f"y Q={Q}")
    assert_state(st, so.reshape(st.shape), f"state Q={Q}")
    return y, st


# --------------------------------------------------------------------- fp32 path
def test_fp32_single_layer_workload():
    """fp32 single layer: b=1, T=256, H=4, P=N=64, G=1, chunk 64, seed 0."""
    inp = problem(gen.SSDShape(1, 256, 4, 64, 1, 64), bf16=False, seed=0)
    _check_fp32(inp, 64)


@pytest.mark.parametrize("T,Q", [(1, 64), (63, 64), (200, 64), (300, 128), (257, 256), (100, 1),
                                 (100, 7), (130, 33)])
def test_fp32_ragged_and_chunk_lengths(T, Q):
    inp = problem(gen.SSDShape(2, T, 4, 64, 2, 64), bf16=False, seed=T + Q)
    _check_fp32(inp, Q)


def test_fp32_chunk_length_invariance():
    inp = problem(gen.SSDShape(1, 320, 2, 32, 1, 128), bf16=False, seed=5)
    ys = [gpu_prefill(inp, Q, bf16=False)[0] for Q in (16, 64, 100, 256)]
    for y in ys[1:]:
        assert_fp32(y, ys[0], "chunk invariance")
    _check_fp32(inp, 64)


def test_fp32_odd_dims_and_groups():
    inp = problem(gen.SSDShape(3, 150, 6, 24, 3, 40), bf16=False, seed=9)
    _check_fp32(inp, 32)


def test_fp32_init_state_and_resume():
    rng = np.random.default_rng(3)
    inp = problem(gen.SSDShape(2, 272, 4, 64, 1, 64), bf16=False, seed=11)
    init = (rng.standard_normal((2, 4, 64, 64)) * 0.1).astype(np.float32)
    _check_fp32(inp, 64, init=init)
    # prefill(T1) then prefill(T2, init = final of the first) == prefill(T1 + T2)
    from state_space_model_05_b200 import ssd_prefill
    dev = lambda a: to_dev(a)
    y_full, s_full = ssd_prefill(dev(inp.x), dev(inp.dt), dev(inp.A), dev(inp.B), dev(inp.C), dev(inp.D), 64)
    T1 = 100
    y1, s1 = ssd_prefill(dev(inp.x[:, :T1]), dev(inp.dt[:, :T1]), dev(inp.A), dev(inp.B[:, :T1]),
                         dev(inp.C[:, :T1]), dev(inp.D), 64)
    y2, s2 = ssd_prefill(dev(inp.x[:, T1:]), dev(inp.dt[:, T1:]), dev(inp.A), dev(inp.B[:, T1:]),
                         dev(inp.C[:, T1:]), dev(inp.D), 64, init_state=s1)
    assert_fp32(torch.cat([y1, y2], 1).cpu().numpy(), y_full.cpu().numpy(), "split prefill y")
    assert_fp32(s2.cpu().numpy(), s_full.cpu().numpy(), "split prefill state")


def test_fp32_init_aliases_final():
    rng = np.random.default_rng(4)
    inp = problem(gen.SSDShape(1, 90, 2, 16, 1, 32), bf16=False, seed=12)
    init = rng.standard_normal((1, 2, 16, 32)).astype(np.float32)
    from state_space_model_05_b200 import ssd_prefill
    st = to_dev(init)
    y, st2 = ssd_prefill(to_dev(inp.x), to_dev(inp.dt), to_dev(inp.A), to_dev(inp.B), to_dev(inp.C),
                         to_dev(inp.D), 32, init_state=st, final_state=st)
    assert st2.data_ptr() == st.data_ptr()
    yo, so = oracle_prefill(inp, init=init.reshape(2, 16, 32))
    assert_fp32(st.cpu().numpy(), so.reshape(1, 2, 16, 32), "aliased state")


def test_empty_sequence_copies_init():
    from state_space_model_05_b200 import ssd_prefill
    rng = np.random.default_rng(5)
    init = to_dev(rng.standard_normal((2, 3, 8, 16)).astype(np.float32))
    x = torch.empty((2, 0, 3, 8), device="cuda")
    dt = torch.empty((2, 0, 3), device="cuda")
    B = torch.empty((2, 0, 1, 16), device="cuda")
    A = -torch.ones(3, device="cuda")
    D = torch.ones(3, device="cuda")
    y, st = ssd_prefill(x, dt, A, B, B, D, 16, init_state=init)
    assert y.shape == (2, 0, 3, 8)
    assert torch.equal(st, init)
    _, st0 = ssd_prefill(x, dt, A, B, B, D, 16)
    assert torch.count_nonzero(st0) == 0


# --------------------------------------------------------------------- bf16 path
def test_bf16_130m_layer_full(tc_path):
    """130M-shaped layer: b=8, T=2048, H=24, P=64, N=128, G=1, chunk 256, all outputs."""
    inp = problem(gen.SSDShape(8, 2048, 24, 64, 1, 128), bf16=True, seed=0)
    _check_bf16(inp, 256)


@pytest.mark.parametrize("T,Q,G", [(1000, 256, 2), (300, 128, 1), (129, 128, 4), (1, 256, 1),
                                   (512, 64, 1), (700, 100, 1)])
def test_bf16_ragged_groups_chunks(T, Q, G, tc_path):
    """Tensor-core path (Q 128/256, partial last chunk, G > 1) and the SIMT path (other Q)."""
    inp = problem(gen.SSDShape(2, T, 4, 64, G, 128), bf16=True, seed=T + Q + G)
    _check_bf16(inp, Q)


def test_bf16_init_state(tc_path):
    rng = np.random.default_rng(6)
    inp = problem(gen.SSDShape(2, 600, 4, 64, 1, 128), bf16=True, seed=21)
    init = (rng.standard_normal((2, 4, 64, 128)) * 0.05).astype(np.float32)
    _check_bf16(inp, 256, init=init)


def test_bf16_chunk_length_invariance(tc_path):
    inp = problem(gen.SSDShape(1, 1024, 8, 64, 1, 128), bf16=True, seed=22)
    b, T, H, P = inp.x.shape
    yo, so = oracle_prefill(inp)
    for Q in (128, 256, 64):
        y, st = gpu_prefill(inp, Q, bf16=True)
        assert_bf16_y(y, oracle.units_to_bthp(yo, b, H), f"Q={Q}")
        assert_state(st, so.reshape(st.shape), f"Q={Q}")


@pytest.mark.parametrize("G,with_init", [(1, False), (2, True)])
def test_bf16_many_chains_full(G, with_init, tc_path):
    """More (batch, head) chains than two per SM (here 320): the chunk-state walk packs up to
    three heads per CTA.  Every token and the final state are checked."""
    inp = problem(gen.SSDShape(4, 384, 80, 64, G, 128), bf16=True, seed=30 + G)
    init = None
    if with_init:
        init = (np.random.default_rng(7).standard_normal((4, 80, 64, 128)) * 0.05).astype(np.float32)
    _check_bf16(inp, 256, init=init)


def test_bf16_27b_long_prefill_sampled(tc_path):
    """2.7B-shaped long prefill (b=4, T=16384, H=80, P=64, N=128, chunk 256) at full size,
    checked on sampled (batch, head) units: all tokens of y and the final state."""
    inp = problem(gen.SSDShape(4, 16384, 80, 64, 1, 128), bf16=True, seed=0)
    y, st = gpu_prefill(inp, 256, bf16=True)
    rng = np.random.default_rng(0)
    units = sorted(rng.choice(4 * 80, size=8, replace=False).tolist())
    yo, so = oracle_prefill(inp, units=units)
    assert_bf16_y(gpu_units(y, units, 80), yo, "y sampled")
    assert_state(st.reshape(4 * 80, 64, 128)[units], so, "state sampled")
    assert np.isfinite(y).all() and np.isfinite(st).all()


def test_bf16_init_aliases_final(tc_path):
    """init_state may be the final_state buffer: each state element is read before it is
    written."""
    from state_space_model_05_b200 import ssd_prefill
    rng = np.random.default_rng(12)
    inp = problem(gen.SSDShape(2, 300, 4, 64, 1, 128), bf16=True, seed=44)
    init = (rng.standard_normal((2, 4, 64, 128)) * 0.05).astype(np.float32)
    bf = torch.bfloat16
    st = to_dev(init)
    ssd_prefill(to_dev(inp.x, bf), to_dev(inp.dt), to_dev(inp.A), to_dev(inp.B, bf), to_dev(inp.C, bf),
                to_dev(inp.D), 256, init_state=st, final_state=st)
    torch.cuda.synchronize()
    yo, so = oracle_prefill(inp, init=init.reshape(8, 64, 128))
    assert_state(st.cpu().numpy(), so.reshape(2, 4, 64, 128), "aliased state")


def test_paths_agree_closely():
    """The fused and two-pass kernels compute the same algorithm in bf16/fp32: their outputs
    differ only by rounding (well inside the oracle tolerance).  Each setting runs its own
    kernels and no others."""
    import state_space_model_05_b200 as ssd
    from state_space_model_05_b200 import binding
    inp = problem(gen.SSDShape(2, 1000, 8, 64, 2, 128), bf16=True, seed=45)
    out, ran = {}, {}
    for path in ("fused", "two_pass"):
        prev = ssd.ssd_set_prefill_path(path)
        binding.ssd_profile_reset()
        binding.ssd_profile_enable(True)
        try:
            out[path] = gpu_prefill(inp, 256, bf16=True)
        finally:
            binding.ssd_profile_enable(False)
            ssd.ssd_set_prefill_path(prev)
        ran[path] = set(binding.ssd_profile_read())
        binding.ssd_profile_reset()
    # the setting really selects the kernels (the library's launch records name them)
    assert ran["fused"] == {"chunk_cumsum", "block_gram_tc", "chain_prefill_tc"}, ran["fused"]
    assert ran["two_pass"] == {"chunk_cumsum", "chunk_state_scan_tc", "chunk_output_tc"}, ran["two_pass"]
    (yf, sf), (yt, stt) = out["fused"], out["two_pass"]
    ry = float(np.sqrt(np.mean(yt.astype(np.float64) ** 2)))
    rs = float(np.sqrt(np.mean(stt.astype(np.float64) ** 2)))
    assert float(np.abs(yf - yt).max()) / ry < 2e-2
    assert float(np.abs(sf - stt).max()) / rs < 1e-2


def test_device_status_clean():
    from state_space_model_05_b200 import ssd_device_status
    assert ssd_device_status() == 0


@pytest.mark.parametrize("bf16,shape,Q,seed", [
    (False, gen.SSDShape(1, 256, 4, 64, 1, 64), 64, 0),       # the fp32 single-layer workload
    (False, gen.SSDShape(2, 300, 4, 64, 1, 64), 64, 340),
    (True, gen.SSDShape(2, 700, 4, 64, 1, 128), 256, 740),
    (True, gen.SSDShape(2, 256, 4, 64, 2, 128), 128, 41)])
def test_dt_softplus_folded_in(bf16, shape, Q, seed, tc_path):
    """ssd_prefill_dtraw forms dt = softplus(dt_raw + dt_bias) itself.  It must equal, bit for
    bit, the plain call given that dt (formed in fp64 by the oracle's softplus and rounded to
    fp32 once), and match the fp64 oracle within the path's tolerance."""
    import state_space_model_05_b200 as ssd
    inp = problem(shape, bf16=bf16, seed=seed)
    b, _, H, P = inp.x.shape
    dt_ = torch.bfloat16 if bf16 else torch.float32
    f32 = torch.float32
    dt64 = oracle.softplus_dt(inp.dt_raw, inp.dt_bias)
    x, A, B, C, D = to_dev(inp.x, dt_), to_dev(inp.A, f32), to_dev(inp.B, dt_), to_dev(inp.C, dt_), to_dev(inp.D, f32)
    y, st = ssd.ssd_prefill(x, to_dev(inp.dt_raw, f32), A, B, C, D, Q, dt_softplus=True,
                            dt_bias=to_dev(inp.dt_bias, f32))
    y2, st2 = ssd.ssd_prefill(x, to_dev(dt64.astype(np.float32), f32), A, B, C, D, Q)
    torch.cuda.synchronize()
    assert ssd.ssd_device_status() == 0
    assert torch.equal(y, y2) and torch.equal(st, st2), "folded dt differs from the plain call"
    if seed == 340:
        return                        # exactness only: see the plain fp32 path's own parity tests
    yo, so = oracle.prefill(inp.x, dt64, inp.A, inp.B, inp.C, inp.D)
    y = y.float().cpu().numpy()
    st = st.cpu().numpy()
    what = f"dtraw {shape} Q={Q}"
    if bf16:
        assert_bf16_y(y, oracle.units_to_bthp(yo, b, H), what + " y")
        assert_state(st, so.reshape(st.shape), what + " state")
    else:
        assert_fp32(y, oracle.units_to_bthp(yo, b, H), what + " y")
        assert_fp32(st, so.reshape(st.shape), what + " state")


def _strong_decay(inp, seed, scale=1.0):
    """Heads spanning the decay range: A = -16 with dt in [0.5, 1] scale (at scale 1 the state
    forgets within a few tokens and a 32-token sub-block of P spans e^-250 and more), A = -0.5
    with dt = 1e-3 (almost no decay), and bursts of dt = 2 scale among dt = 0.01 on A = -16."""
    rng = np.random.default_rng(seed)
    b, T, H, P = inp.x.shape
    A = np.array([-16.0, -0.5, -16.0, -4.0][:H] + [-1.0] * max(0, H - 4), dtype=np.float32)
    dt = np.empty((b, T, H), dtype=np.float32)
    dt[..., 0] = rng.uniform(0.5, 1.0, (b, T)) * scale
    dt[..., 1] = 1e-3
    dt[..., 2] = np.where(rng.random((b, T)) < 0.1, 2.0 * scale, 0.01)
    if H > 3:
        dt[..., 3:] = rng.uniform(0.05, 0.3, (b, T, H - 3))
    inp.A, inp.dt = A, dt
    return inp


def test_bf16_strong_decay(tc_path):
    """Decay far past the e^40 guard inside 32-token sub-blocks (the per-element path of P),
    block decays that underflow to zero, and w o x underflowing in fp16."""
    inp = _strong_decay(problem(gen.SSDShape(2, 700, 4, 64, 1, 128), bf16=True, seed=46), 47)
    init = (np.random.default_rng(48).standard_normal((2, 4, 64, 128)) * 0.05).astype(np.float32)
    _check_bf16(inp, 256, init=init)


@pytest.mark.parametrize("scale", [1.0, 0.1])
def test_fp32_strong_decay(scale):
    """The same heads on the fp32 path, at full strength (within-chunk decay sums near -2000,
    where a single fp32 ulp is 1.2e-4: the path keeps them as double-float hi/lo pairs) and
    with dt capped at the workloads' largest value, 0.1."""
    inp = _strong_decay(problem(gen.SSDShape(2, 300, 4, 64, 1, 64), bf16=False, seed=49), 50, scale=scale)
    _check_fp32(inp, 64)


@pytest.mark.parametrize("bf16,Q", [(False, 256), (False, 100), (True, 256)])
def test_max_dims(bf16, Q):
    """headdim 128 and dstate 256, the largest prefill sizes the ABI takes (the CUDA-core path,
    whose output kernel then holds a 128 x 257 state tile in shared memory), ragged length."""
    inp = problem(gen.SSDShape(2, 300, 2, 128, 1, 256), bf16=bf16, seed=51 + Q)
    if bf16:
        _check_bf16(inp, Q)
    else:
        _check_fp32(inp, Q)
