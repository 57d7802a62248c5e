"""Pins of the fp64 sequential oracle against facts fixed outside it.

Source of the method: "Compiler-First State Space Duality and Portable O(1)
Autoregressive Caching for Inference", section "2. Metodologia" (chunkable
recurrence with per-head diagonal decay, static lower-triangular masks, an O(1)
state cache advanced one token at a time) and section "4. Resultados"
(constant-size state during generation).

Each test checks the oracle against something other than itself: a hand-worked
case, a closed form, a separately written chunked or quadratic form, or an
identity of the recurrence.
"""
import json
import math
import os

import numpy as np
import pytest
from hypothesis import given, settings, strategies as st

from state_space_model_05_b200 import inputs as gen

GOLDEN = os.path.join(os.path.dirname(__file__), "golden", "ssd_tiny_hand.json")


def _eval_expr(s):
    return float(eval(s, {"__builtins__": {}}, {"exp": math.exp}))


def _rand_problem(rng, b, T, H, P, G, N, scale_dt=1.0):
    x = rng.standard_normal((b, T, H, P)).astype(np.float32)
    dt = (np.exp(rng.uniform(np.log(1e-3), np.log(0.3), (b, T, H))) * scale_dt).astype(np.float32)
    A = (-np.exp(rng.uniform(0, np.log(16), H))).astype(np.float32)
    B = (rng.standard_normal((b, T, G, N)) / np.sqrt(N)).astype(np.float32)
    C = (rng.standard_normal((b, T, G, N)) / np.sqrt(N)).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    return x, dt, A, B, C, D


def _seq(oracle_mod, x, dt, A, B, C, D, init=None):
    b, T, H, P = x.shape
    y, st_ = oracle_mod.prefill(x, dt, A, B, C, D, init=init)
    return oracle_mod.units_to_bthp(y, b, H), st_.reshape(b, H, P, -1)


# ---------------------------------------------------------------- hand-worked case
@pytest.mark.parametrize("case", [0, 1])
def test_golden_hand_case(oracle_mod, case):
    g = json.load(open(GOLDEN))
    inp = {k: np.array(v, dtype=np.float32) for k, v in g["inputs"].items()}
    c = g["cases"][case]
    init = None if c["init"] is None else np.array(c["init"], dtype=np.float64)[None]
    y, st_ = oracle_mod.prefill(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"], init=init)
    y_exp = np.array([[_eval_expr(v) for v in row] for row in c["y"]])
    s_exp = np.array([[_eval_expr(v) for v in row] for row in c["state"]])
    np.testing.assert_allclose(y[0], y_exp, rtol=1e-14, atol=1e-14)
    np.testing.assert_allclose(st_[0], s_exp, rtol=1e-14, atol=1e-14)


# ---------------------------------------------------------------- closed forms
def test_A_zero_is_cumulative_sum(oracle_mod):
    """A = 0: no decay, H_t = sum_{s<=t} dt_s B_s x_s^T; with N=P=1 and B=C=1,
    y_t = sum_{s<=t} dt_s x_s + D x_t."""
    rng = np.random.default_rng(3)
    T = 300
    x = rng.standard_normal((1, T, 1, 1)).astype(np.float32)
    dt = rng.uniform(0.01, 0.2, (1, T, 1)).astype(np.float32)
    A = np.zeros(1, np.float32)
    B = np.ones((1, T, 1, 1), np.float32)
    C = np.ones((1, T, 1, 1), np.float32)
    D = np.array([0.7], np.float32)
    y, st_ = oracle_mod.prefill(x, dt, A, B, C, D)
    xd = x[0, :, 0, 0].astype(np.float64)
    dd = dt[0, :, 0].astype(np.float64)
    cs = np.cumsum(dd * xd)
    np.testing.assert_allclose(y[0, :, 0], cs + float(D[0]) * xd, rtol=1e-12, atol=1e-12)
    np.testing.assert_allclose(st_[0, 0, 0], cs[-1], rtol=1e-12)


def test_A_zero_general_shape_is_outer_product_sum(oracle_mod):
    rng = np.random.default_rng(4)
    x, dt, A, B, C, D = _rand_problem(rng, 2, 37, 4, 5, 2, 3)
    A[:] = 0
    y, st_ = _seq(oracle_mod, x, dt, A, B, C, D)
    Bh = np.repeat(B.astype(np.float64), 2, axis=2)
    Ch = np.repeat(C.astype(np.float64), 2, axis=2)
    Hs = np.cumsum(np.einsum("bth,bthp,bthn->bthpn", dt.astype(np.float64), x.astype(np.float64), Bh), axis=1)
    y_ref = np.einsum("bthpn,bthn->bthp", Hs, Ch) + D.astype(np.float64)[None, None, :, None] * x
    np.testing.assert_allclose(y, y_ref, rtol=1e-11, atol=1e-12)
    np.testing.assert_allclose(st_, Hs[:, -1], rtol=1e-11, atol=1e-12)


def test_geometric_closed_form(oracle_mod):
    """Constant dt and A, N=P=1, B=C=x=1: H_t = dt (1 - a^(t+1)) / (1 - a)."""
    T = 200
    dtv, Av, Dv = 0.05, -3.0, -0.25
    x = np.ones((1, T, 1, 1), np.float32)
    dt = np.full((1, T, 1), dtv, np.float32)
    A = np.array([Av], np.float32)
    B = np.ones((1, T, 1, 1), np.float32)
    C = np.ones((1, T, 1, 1), np.float32)
    D = np.array([Dv], np.float32)
    y, st_ = oracle_mod.prefill(x, dt, A, B, C, D)
    d = float(np.float32(dtv))
    a = math.exp(d * float(np.float32(Av)))
    t = np.arange(T)
    Ht = d * (1 - a ** (t + 1)) / (1 - a)
    np.testing.assert_allclose(y[0, :, 0], Ht + float(D[0]), rtol=1e-12)
    np.testing.assert_allclose(st_[0, 0, 0], Ht[-1], rtol=1e-12)


# ---------------------------------------------------------------- other forms
@pytest.mark.parametrize("Q", [1, 2, 3, 16, 64, 300])
def test_chunked_equals_sequential(oracle_mod, Q):
    from oracle import forms
    rng = np.random.default_rng(10 + Q)
    x, dt, A, B, C, D = _rand_problem(rng, 2, 300, 4, 6, 2, 5)
    init = rng.standard_normal((2 * 4, 6, 5))
    y, st_ = _seq(oracle_mod, x, dt, A, B, C, D, init=init)
    yc, sc = forms.chunked(x, dt, A, B, C, D, Q, init=init.reshape(2, 4, 6, 5))
    np.testing.assert_allclose(yc, y, rtol=1e-10, atol=1e-12)
    np.testing.assert_allclose(sc, st_, rtol=1e-10, atol=1e-12)


def test_quadratic_equals_sequential(oracle_mod):
    from oracle import forms
    rng = np.random.default_rng(11)
    x, dt, A, B, C, D = _rand_problem(rng, 1, 64, 3, 4, 1, 7)
    y, _ = _seq(oracle_mod, x, dt, A, B, C, D)
    yq = forms.quadratic(x, dt, A, B, C, D)
    np.testing.assert_allclose(yq, y, rtol=1e-10, atol=1e-12)


def test_quadratic_on_small_workload_shape(oracle_mod):
    """The fp32 single-layer workload's shape (T=256, H=4, P=N=64), quadratic form."""
    from oracle import forms
    s = gen.SSDShape(1, 256, 4, 64, 1, 64)
    inp = gen.prefill_inputs(s, seed=0)
    y, st_ = _seq(oracle_mod, inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D)
    yq = forms.quadratic(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D)
    np.testing.assert_allclose(yq, y, rtol=1e-9, atol=1e-12)


@settings(max_examples=25, deadline=None)
@given(T=st.integers(1, 120), Q=st.sampled_from([1, 2, 3, 16, 64]), P=st.integers(1, 9),
       N=st.integers(1, 9), G=st.sampled_from([1, 2]), seed=st.integers(0, 10 ** 6))
def test_chunked_equals_sequential_property(oracle_mod, T, Q, P, N, G, seed):
    from oracle import forms
    rng = np.random.default_rng(seed)
    H = 2 * G
    x, dt, A, B, C, D = _rand_problem(rng, 1, T, H, P, G, N)
    y, st_ = _seq(oracle_mod, x, dt, A, B, C, D)
    yc, sc = forms.chunked(x, dt, A, B, C, D, Q)
    np.testing.assert_allclose(yc, y, rtol=1e-9, atol=1e-12)
    np.testing.assert_allclose(sc, st_, rtol=1e-9, atol=1e-12)


# ---------------------------------------------------------------- identities
def test_C_zero_gives_skip_only(oracle_mod):
    rng = np.random.default_rng(5)
    x, dt, A, B, C, D = _rand_problem(rng, 2, 40, 4, 3, 2, 5)
    C[:] = 0
    y, _ = _seq(oracle_mod, x, dt, A, B, C, D)
    np.testing.assert_array_equal(y, D[None, None, :, None].astype(np.float64) * x)


def test_B_zero_only_decays_init(oracle_mod):
    rng = np.random.default_rng(6)
    x, dt, A, B, C, D = _rand_problem(rng, 1, 30, 2, 3, 1, 4)
    B[:] = 0
    init = rng.standard_normal((2, 3, 4))
    _, st_ = _seq(oracle_mod, x, dt, A, B, C, D, init=init)
    decay = np.exp((dt[0].astype(np.float64) * A[None, :]).sum(0))   # [H]
    np.testing.assert_allclose(st_[0], init * decay[:, None, None], rtol=1e-12)


def test_dt_zero_tokens_leave_state_unchanged(oracle_mod):
    rng = np.random.default_rng(7)
    x, dt, A, B, C, D = _rand_problem(rng, 1, 50, 2, 4, 1, 3)
    y1, s1 = _seq(oracle_mod, x[:, :20], dt[:, :20], A, B[:, :20], C[:, :20], D)
    dt2 = dt.copy()
    dt2[:, 20:] = 0
    y2, s2 = _seq(oracle_mod, x, dt2, A, B, C, D)
    np.testing.assert_array_equal(s2, s1)
    # y_t = C_t^T H + D x_t for the inert tokens
    Hs = s1[0]                                            # [H][P][N]
    y_ref = np.einsum("thn,hpn->thp", C[0, 20:].astype(np.float64).repeat(2, axis=1), Hs) \
        + D.astype(np.float64)[None, :, None] * x[0, 20:]
    np.testing.assert_allclose(y2[0, 20:], y_ref, rtol=1e-12, atol=1e-14)


def test_linear_in_x_and_init(oracle_mod):
    rng = np.random.default_rng(8)
    x, dt, A, B, C, D = _rand_problem(rng, 1, 64, 2, 4, 1, 6)
    x2 = rng.standard_normal(x.shape).astype(np.float32)
    i1 = rng.standard_normal((2, 4, 6))
    i2 = rng.standard_normal((2, 4, 6))
    ya, sa = _seq(oracle_mod, x, dt, A, B, C, D, init=i1)
    yb, sb = _seq(oracle_mod, x2, dt, A, B, C, D, init=i2)
    ys, ss = _seq(oracle_mod, (x.astype(np.float64) + x2).astype(np.float32), dt, A, B, C, D, init=i1 + i2)
    # x + x2 is rounded to fp32 for the input; compare against the exact sum's image
    xs = x.astype(np.float64) + x2
    lin_err = np.abs((xs - (x.astype(np.float64) + x2).astype(np.float32))).max()
    assert lin_err < 1e-6
    np.testing.assert_allclose(ys, ya + yb, rtol=1e-5, atol=1e-5)
    np.testing.assert_allclose(ss, sa + sb, rtol=1e-5, atol=1e-5)


def test_batch_permutation(oracle_mod):
    rng = np.random.default_rng(9)
    x, dt, A, B, C, D = _rand_problem(rng, 3, 25, 2, 3, 1, 4)
    perm = [2, 0, 1]
    y, s = _seq(oracle_mod, x, dt, A, B, C, D)
    yp, sp = _seq(oracle_mod, x[perm], dt[perm], A, B[perm], C[perm], D)
    np.testing.assert_array_equal(yp, y[perm])
    np.testing.assert_array_equal(sp, s[perm])


def test_transposed_state_layout_detected(oracle_mod):
    """The state is [p][n]: H[p][n] = dt x_p B_n for a single token from zero."""
    x = np.array([[[[1.0, 2.0]]]], np.float32)            # P = 2
    dt = np.array([[[1.0]]], np.float32)
    B = np.array([[[[3.0, 5.0, 7.0]]]], np.float32)       # N = 3
    C = np.zeros_like(B)
    _, s = oracle_mod.prefill(x, dt, np.array([-1.0], np.float32), B, C, np.zeros(1, np.float32))
    np.testing.assert_array_equal(s[0], [[3, 5, 7], [6, 10, 14]])


def test_group_mapping_is_contiguous_blocks(oracle_mod):
    """Head h reads group h // (H / G): with G = 2, H = 4, heads 0,1 -> group 0."""
    rng = np.random.default_rng(12)
    x, dt, A, B, C, D = _rand_problem(rng, 1, 10, 4, 2, 2, 3)
    y, _ = _seq(oracle_mod, x, dt, A, B, C, D)
    for h, g in [(0, 0), (1, 0), (2, 1), (3, 1)]:
        yh, _ = _seq(oracle_mod, x[:, :, h:h + 1], dt[:, :, h:h + 1], A[h:h + 1],
                     B[:, :, g:g + 1], C[:, :, g:g + 1], D[h:h + 1])
        np.testing.assert_array_equal(yh[:, :, 0], y[:, :, h])


# ---------------------------------------------------------------- cache / resume
def test_prefill_then_decode_equals_longer_prefill(oracle_mod):
    """prefill(T) followed by k decode steps == prefill(T + k) (the O(1) cache resumes)."""
    s = gen.SSDShape(1, 272, 4, 64, 1, 64)
    inp = gen.prefill_inputs(s, seed=0)
    T0 = 256
    y_full, s_full = oracle_mod.prefill(inp.x, inp.dt, inp.A, inp.B, inp.C, inp.D)
    _, st_ = oracle_mod.prefill(inp.x[:, :T0], inp.dt[:, :T0], inp.A, inp.B[:, :T0],
                                inp.C[:, :T0], inp.D)
    for k in range(T0, 272):
        yk = oracle_mod.decode_step(st_, inp.x[:, k], inp.dt[:, k], inp.A, inp.B[:, k],
                                    inp.C[:, k], inp.D)
        np.testing.assert_allclose(yk, y_full[:, k], rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(st_, s_full, rtol=1e-12, atol=1e-13)


def test_split_prefill_with_init(oracle_mod):
    rng = np.random.default_rng(13)
    x, dt, A, B, C, D = _rand_problem(rng, 2, 90, 2, 3, 1, 4)
    y, s = oracle_mod.prefill(x, dt, A, B, C, D)
    y1, s1 = oracle_mod.prefill(x[:, :33], dt[:, :33], A, B[:, :33], C[:, :33], D)
    y2, s2 = oracle_mod.prefill(x[:, 33:], dt[:, 33:], A, B[:, 33:], C[:, 33:], D, init=s1)
    np.testing.assert_allclose(np.concatenate([y1, y2], axis=1), y, rtol=1e-12, atol=1e-13)
    np.testing.assert_allclose(s2, s, rtol=1e-12, atol=1e-13)


def test_state_size_independent_of_T(oracle_mod):
    rng = np.random.default_rng(14)
    shapes = set()
    for T in [1, 7, 64, 333]:
        x, dt, A, B, C, D = _rand_problem(rng, 1, T, 2, 3, 1, 4)
        _, s = oracle_mod.prefill(x, dt, A, B, C, D)
        shapes.add(s.shape)
    assert shapes == {(2, 3, 4)}


def test_unit_subset_matches_full(oracle_mod):
    rng = np.random.default_rng(15)
    x, dt, A, B, C, D = _rand_problem(rng, 2, 20, 3, 2, 1, 3)
    y, s = oracle_mod.prefill(x, dt, A, B, C, D)
    units = [5, 0, 3]
    yu, su = oracle_mod.prefill(x, dt, A, B, C, D, units=units)
    np.testing.assert_array_equal(yu, y[units])
    np.testing.assert_array_equal(su, s[units])


def test_empty_sequence(oracle_mod):
    rng = np.random.default_rng(16)
    x, dt, A, B, C, D = _rand_problem(rng, 1, 0, 2, 3, 1, 4)
    init = rng.standard_normal((2, 3, 4))
    y, s = oracle_mod.prefill(x, dt, A, B, C, D, init=init)
    assert y.shape == (2, 0, 3)
    np.testing.assert_array_equal(s, init)


def test_softplus_dt_pins():
    """softplus at the points and identities that fix it: softplus(0) = ln 2,
    softplus(z) - softplus(-z) = z, softplus(z) -> z and -> exp(z) at the extremes; the
    bias is added per head (last axis)."""
    import math
    from oracle import softplus_dt
    assert softplus_dt(np.float32([0.0]))[0] == math.log(2.0)
    z = np.linspace(-30, 30, 121).astype(np.float32)
    np.testing.assert_allclose(softplus_dt(z) - softplus_dt(-z), z.astype(np.float64), rtol=0, atol=1e-12)
    assert softplus_dt(np.float32([60.0]))[0] == 60.0 + math.log1p(math.exp(-60.0))
    np.testing.assert_allclose(softplus_dt(np.float32([-40.0]))[0], math.exp(-40.0), rtol=1e-12)
    raw = np.zeros((2, 3, 4), dtype=np.float32)
    bias = np.float32([-1.0, 0.0, 1.0, 2.0])
    got = softplus_dt(raw, bias)
    np.testing.assert_allclose(got[1, 2], [math.log1p(math.exp(b)) for b in (-1.0, 0.0, 1.0, 2.0)], rtol=1e-15)
