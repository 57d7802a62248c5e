"""GPU parity of the packed variable-length prefill (ssd_prefill_varlen).

Sequences of mixed lengths (empty, shorter than a block, exactly a block, block + 1, several
chunks) are packed end to end; every sequence must match the fp64 oracle run on that
sequence alone, from its own initial state.  With equal lengths the packed call must equal
the batched call bit for bit.
"""
import numpy as np
import pytest
import torch

import oracle
from parity import assert_bf16_y, assert_state, to_dev
from state_space_model_05_b200 import inputs as gen

pytestmark = pytest.mark.gpu


@pytest.fixture(autouse=True, scope="module")
def _built():
    from state_space_model_05_b200.build import build
    build()
    oracle.build()


def _packed(lengths, H=4, G=1, seed=0):
    """One seeded problem of sum(lengths) tokens (batch 1), bf16-rounded x/B/C."""
    T = int(sum(lengths))
    inp = gen.prefill_inputs(gen.SSDShape(1, max(T, 1), H, 64, G, 128), seed=seed)
    inp.x, inp.B, inp.C = gen.round_bf16(inp.x), gen.round_bf16(inp.B), gen.round_bf16(inp.C)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    return inp, cu, T


def _run(inp, cu, T, Q, init=None):
    import state_space_model_05_b200 as ssd
    bf, f32 = torch.bfloat16, torch.float32
    y, st = ssd.ssd_prefill_varlen(to_dev(inp.x[0, :T], bf), to_dev(inp.dt[0, :T], f32), to_dev(inp.A, f32),
                                   to_dev(inp.B[0, :T], bf), to_dev(inp.C[0, :T], bf), to_dev(inp.D, f32),
                                   torch.from_numpy(cu).cuda(), Q,
                                   init_states=None if init is None else to_dev(init, f32))
    torch.cuda.synchronize()
    return y.float().cpu().numpy(), st.cpu().numpy()


@pytest.mark.parametrize("Q", [128, 256])
def test_mixed_lengths_match_per_sequence_oracle(Q):
    lengths = [300, 0, 1, 127, 128, 129, 700, 64, 256, 3]
    inp, cu, T = _packed(lengths, seed=7)
    H = inp.x.shape[2]
    rng = np.random.default_rng(8)
    init = (0.05 * rng.standard_normal((len(lengths), H, 64, 128))).astype(np.float32)
    y, st = _run(inp, cu, T, Q, init=init)
    import state_space_model_05_b200 as ssd
    assert ssd.ssd_device_status() == 0
    for i, n in enumerate(lengths):
        a, b = cu[i], cu[i + 1]
        if n > 0:
            yo, so = oracle.prefill(inp.x[:, a:b], inp.dt[:, a:b], inp.A, inp.B[:, a:b], inp.C[:, a:b], inp.D,
                                    init=init[i].astype(np.float64))
            assert_bf16_y(y[a:b], oracle.units_to_bthp(yo, 1, H)[0], f"varlen Q={Q} seq {i} (len {n}) y")
            assert_state(st[i], so.reshape(st[i].shape), f"varlen Q={Q} seq {i} (len {n}) state")
        else:
            assert np.array_equal(st[i], init[i]), f"empty sequence {i} keeps its initial state"


def test_equal_lengths_equal_batched_call_bitwise():
    """Two sequences of 300 tokens packed equal a batch of two 300-token problems bit for bit
    (the padding rows of a partial block are the next sequence's tokens with dt = 0)."""
    import state_space_model_05_b200 as ssd
    shape = gen.SSDShape(2, 300, 8, 64, 2, 128)
    inp = gen.prefill_inputs(shape, seed=3)
    bf, f32 = torch.bfloat16, torch.float32
    x, dt, B, C = to_dev(inp.x, bf), to_dev(inp.dt, f32), to_dev(inp.B, bf), to_dev(inp.C, bf)
    A, D = to_dev(inp.A, f32), to_dev(inp.D, f32)
    y1, s1 = ssd.ssd_prefill(x, dt, A, B, C, D, 256)
    cu = torch.tensor([0, 300, 600], dtype=torch.int32, device="cuda")
    y2, s2 = ssd.ssd_prefill_varlen(x.reshape(600, 8, 64), dt.reshape(600, 8), A, B.reshape(600, 2, 128),
                                    C.reshape(600, 2, 128), D, cu, 256)
    torch.cuda.synchronize()
    assert torch.equal(y1.reshape(600, 8, 64), y2) and torch.equal(s1, s2)
    assert ssd.ssd_device_status() == 0


def test_many_short_sequences():
    """More sequences than SMs hold chains at once, of lengths 1 .. 200."""
    rng = np.random.default_rng(9)
    lengths = rng.integers(1, 200, size=400).tolist()
    inp, cu, T = _packed(lengths, H=2, seed=11)
    y, st = _run(inp, cu, T, 128)
    import state_space_model_05_b200 as ssd
    assert ssd.ssd_device_status() == 0
    for i in rng.choice(len(lengths), size=12, replace=False):
        a, b = cu[i], cu[i + 1]
        yo, so = oracle.prefill(inp.x[:, a:b], inp.dt[:, a:b], inp.A, inp.B[:, a:b], inp.C[:, a:b], inp.D)
        assert_bf16_y(y[a:b], oracle.units_to_bthp(yo, 1, 2)[0], f"short seq {i} y")
        assert_state(st[i], so.reshape(st[i].shape), f"short seq {i} state")


def test_bad_offsets_are_reported_not_read():
    """Decreasing offsets: the table kernel records SSD_ERR_SHAPE before any kernel uses them,
    and no block is computed."""
    import state_space_model_05_b200 as ssd
    inp, cu, T = _packed([200, 200], seed=5)
    bad = np.array([0, 250, 150, 400], dtype=np.int32)         # three sequences, one of negative length
    bf, f32 = torch.bfloat16, torch.float32
    y = torch.zeros((T, 4, 64), device="cuda", dtype=bf)
    ssd.ssd_prefill_varlen(to_dev(inp.x[0, :T], bf), to_dev(inp.dt[0, :T], f32), to_dev(inp.A, f32),
                           to_dev(inp.B[0, :T], bf), to_dev(inp.C[0, :T], bf), to_dev(inp.D, f32),
                           torch.from_numpy(bad).cuda(), 256, y=y)
    torch.cuda.synchronize()
    assert ssd.ssd_device_status() == 2               # SSD_ERR_SHAPE
    assert torch.count_nonzero(y) == 0


@pytest.mark.parametrize("bf16,Q,N", [(False, 64, 64), (False, 100, 128), (True, 64, 128)])
def test_cuda_core_path_mixed_lengths(bf16, Q, N):
    """The CUDA-core path (fp32, or chunk lengths the tensor-core path does not take)."""
    import state_space_model_05_b200 as ssd
    from parity import assert_fp32
    lengths = [150, 0, 1, 63, 64, 65, 300, 7]
    T = sum(lengths)
    inp = gen.prefill_inputs(gen.SSDShape(1, T, 4, 64, 2, N), seed=Q + N)
    if bf16:
        inp.x, inp.B, inp.C = gen.round_bf16(inp.x), gen.round_bf16(inp.B), gen.round_bf16(inp.C)
    cu = np.concatenate([[0], np.cumsum(lengths)]).astype(np.int32)
    dt_ = torch.bfloat16 if bf16 else torch.float32
    f32 = torch.float32
    rng = np.random.default_rng(3)
    init = (0.1 * rng.standard_normal((len(lengths), 4, 64, N))).astype(np.float32)
    y, st = ssd.ssd_prefill_varlen(to_dev(inp.x[0], dt_), to_dev(inp.dt[0], f32), to_dev(inp.A, f32),
                                   to_dev(inp.B[0], dt_), to_dev(inp.C[0], dt_), to_dev(inp.D, f32),
                                   torch.from_numpy(cu).cuda(), Q, init_states=to_dev(init, f32))
    torch.cuda.synchronize()
    assert ssd.ssd_device_status() == 0
    y, st = y.float().cpu().numpy(), st.cpu().numpy()
    for i, n in enumerate(lengths):
        a, b = cu[i], cu[i + 1]
        if n == 0:
            assert np.array_equal(st[i], init[i])
            continue
        yo, so = oracle.prefill(inp.x[:, a:b], inp.dt[:, a:b], inp.A, inp.B[:, a:b], inp.C[:, a:b], inp.D,
                                init=init[i].astype(np.float64))
        what = f"varlen CUDA-core Q={Q} seq {i} (len {n})"
        if bf16:
            assert_bf16_y(y[a:b], oracle.units_to_bthp(yo, 1, 4)[0], what + " y")
            assert_state(st[i], so.reshape(st[i].shape), what + " state")
        else:
            assert_fp32(y[a:b], oracle.units_to_bthp(yo, 1, 4)[0], what + " y")
            assert_fp32(st[i], so.reshape(st[i].shape), what + " state")


def test_cuda_core_equal_lengths_equal_batched_call_bitwise():
    import state_space_model_05_b200 as ssd
    inp = gen.prefill_inputs(gen.SSDShape(3, 200, 4, 32, 1, 64), seed=12)
    f32 = torch.float32
    x, dt, B, C = (to_dev(a, f32) for a in (inp.x, inp.dt, inp.B, inp.C))
    A, D = to_dev(inp.A, f32), to_dev(inp.D, f32)
    y1, s1 = ssd.ssd_prefill(x, dt, A, B, C, D, 64)
    cu = torch.tensor([0, 200, 400, 600], dtype=torch.int32, device="cuda")
    y2, s2 = ssd.ssd_prefill_varlen(x.reshape(600, 4, 32), dt.reshape(600, 4), A, B.reshape(600, 1, 64),
                                    C.reshape(600, 1, 64), D, cu, 64)
    torch.cuda.synchronize()
    assert torch.equal(y1.reshape(600, 4, 32), y2) and torch.equal(s1, s2)
