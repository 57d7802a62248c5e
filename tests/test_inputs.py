"""The seeded input generators: reproducibility, distributions, bf16 rounding, Philox."""
import math

import numpy as np
import torch

from state_space_model_05_b200 import inputs as gen


def test_philox_known_answers():
    """Philox4x32-10 known-answer vectors published with the Random123 library
    (Salmon et al., SC'11)."""
    cases = [
        ((0, 0, 0, 0), (0, 0), (0x6627E8D5, 0xE169C58D, 0xBC57AC4C, 0x9B00DBD8)),
        ((0xFFFFFFFF,) * 4, (0xFFFFFFFF, 0xFFFFFFFF), (0x408F276D, 0x41C83B0E, 0xA20BC7C6, 0x6D5451FD)),
        ((0x243F6A88, 0x85A308D3, 0x13198A2E, 0x03707344), (0xA4093822, 0x299F31D0),
         (0xD16CFE09, 0x94FDCCEB, 0x5001E420, 0x24126EA1)),
    ]
    for ctr, key, expect in cases:
        out = gen.philox4x32_10(np.array([ctr], dtype=np.uint32), key)
        assert tuple(int(v) for v in out[0]) == expect


def test_irwin_hall_normal_moments():
    z = gen.philox_normal(7, np.arange(200000), seed=123)
    assert abs(z.mean()) < 0.01
    assert abs(z.std() - 1.0) < 0.01
    assert np.abs(z).max() <= 6.0


def test_round_bf16_matches_torch():
    rng = np.random.default_rng(0)
    a = (rng.standard_normal(100000) * np.exp(rng.uniform(-20, 20, 100000))).astype(np.float32)
    a[:4] = [0.0, -0.0, 1.0 + 2 ** -8, 1.0 + 3 * 2 ** -8]   # ties
    ours = gen.round_bf16(a)
    ref = torch.from_numpy(a).to(torch.bfloat16).to(torch.float32).numpy()
    np.testing.assert_array_equal(ours, ref)


def test_prefill_inputs_reproducible_and_distributed():
    s = gen.SSDShape(2, 512, 8, 16, 1, 64)
    a = gen.prefill_inputs(s, seed=0)
    b = gen.prefill_inputs(s, seed=0)
    for k in ("x", "dt", "A", "B", "C", "D"):
        np.testing.assert_array_equal(getattr(a, k), getattr(b, k))
    assert np.all(a.A <= -1.0) and np.all(a.A >= -16.0)
    assert np.all(a.dt > 0)
    # per-head dt centre is log-uniform in [1e-3, 0.1]: medians sit inside a widened range
    med = np.median(a.dt, axis=(0, 1))
    assert np.all(med > 1e-3 * 0.5) and np.all(med < 0.1 * 2.0)
    assert abs(a.x.std() - 1) < 0.02
    assert abs(a.B.std() * math.sqrt(64) - 1) < 0.05


def test_decode_inputs_dt_range():
    s = gen.SSDShape(4, 1, 8, 16, 1, 32)
    d = gen.decode_inputs(s, steps=64, seed=1)
    assert d.dt.min() >= 1e-3 * (1 - 1e-6) and d.dt.max() <= 0.1 * (1 + 1e-6)
    lg = np.log(d.dt)
    # log-uniform: mean of log dt is the midpoint
    assert abs(lg.mean() - 0.5 * (math.log(1e-3) + math.log(0.1))) < 0.1


def test_dt_table_log_uniform_levels():
    t = gen.dt_table()
    assert t.size == 1 << gen.DT_TABLE_BITS
    assert t[0] > 1e-3 and t[-1] < 0.1
    r = np.diff(np.log(t.astype(np.float64)))
    assert np.allclose(r, r[0], rtol=2e-3)
