"""The Python binding's argument checks (CPU only, no library call).

The C ABI receives bare pointers, so a tensor of the wrong size would be read or written out
of bounds on the device.  The binding therefore checks every tensor's shape against the
layouts in include/ssd.h before anything else.  These tests drive it with storage-less tensors:
a wrong shape must be reported as such; a right one must get past the shape checks and
stop at the CUDA-tensor check, which comes before any library call.
"""
import pytest
import torch

from state_space_model_05_b200 import binding
import state_space_model_05_b200 as ssd

f32, bf = torch.float32, torch.bfloat16


@pytest.fixture(autouse=True)
def no_library(monkeypatch, tmp_path):
    """Any library call would raise RuntimeError: the checks must all come first."""
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)


def z(*shape, dtype=f32):
    """A tensor of that shape with no storage (the checks read shapes, devices and dtypes only)."""
    return torch.empty(shape, dtype=dtype, device="meta")


def prefill_args(b=2, T=300, H=4, P=64, G=1, N=128, dtype=bf):
    return dict(x=z(b, T, H, P, dtype=dtype), dt=z(b, T, H), A=z(H), B=z(b, T, G, N, dtype=dtype),
                C=z(b, T, G, N, dtype=dtype), D=z(H))


def call_prefill(a, **kw):
    return ssd.ssd_prefill(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], 256, **kw)


def shapes_accepted(fn):
    """Run ``fn``; the shape checks passed if it stops at the CUDA-tensor check."""
    with pytest.raises(ValueError, match="must be a CUDA tensor"):
        fn()


@pytest.mark.parametrize("shape", [(8, 2048, 24, 64, 1, 128), (4, 16384, 80, 64, 1, 128),
                                   (1, 256, 4, 64, 1, 64), (2, 0, 3, 8, 1, 16), (2, 300, 8, 64, 2, 128)])
def test_prefill_valid_shapes_pass(shape):
    b, T, H, P, G, N = shape
    a = prefill_args(b, T, H, P, G, N)
    st = z(b, H, P, N)
    shapes_accepted(lambda: call_prefill(a))
    shapes_accepted(lambda: call_prefill(a, init_state=st, final_state=st, y=z(b, T, H, P, dtype=bf)))
    shapes_accepted(lambda: call_prefill(a, dt_softplus=True, dt_bias=z(H)))
    shapes_accepted(lambda: call_prefill(a, dt_softplus=True))          # bias is optional


@pytest.mark.parametrize("field,bad", [("dt", (2, 300, 5)), ("dt", (2, 299, 4)), ("A", (5,)), ("D", (4, 1)),
                                       ("B", (2, 300, 128)), ("C", (2, 300, 1, 64)), ("C", (1, 300, 1, 128)),
                                       ("x", (2, 300, 4))])
def test_prefill_wrong_shape_is_refused(field, bad):
    a = prefill_args()
    a[field] = z(*bad, dtype=a[field].dtype)
    with pytest.raises(ValueError, match="shape"):
        call_prefill(a)


@pytest.mark.parametrize("kw", [dict(init_state=z(2, 4, 64, 64)), dict(final_state=z(8, 64, 128)),
                                dict(y=z(2, 300, 4, 32, dtype=bf)), dict(dt_softplus=True, dt_bias=z(2, 4))])
def test_prefill_wrong_optional_shape_is_refused(kw):
    with pytest.raises(ValueError, match="has shape"):
        call_prefill(prefill_args(), **kw)


def test_varlen_shapes():
    total, H, P, G, N = 600, 8, 64, 2, 128
    x, dt, B = z(total, H, P, dtype=bf), z(total, H), z(total, G, N, dtype=bf)
    cu = torch.tensor([0, 300, 600], dtype=torch.int32)
    st = z(2, H, P, N)
    call = lambda **kw: ssd.ssd_prefill_varlen(kw.get("x", x), kw.get("dt", dt), z(H), kw.get("B", B), B, z(H),
                                               kw.get("cu", cu), 256, init_states=kw.get("init"),
                                               final_states=kw.get("final"))
    shapes_accepted(lambda: call())
    shapes_accepted(lambda: call(init=st, final=st))
    for kw in (dict(dt=z(total, H + 1)), dict(B=z(total, N, dtype=bf)), dict(init=z(3, H, P, N)),
               dict(final=z(2, H, P, N + 8)), dict(x=z(1, total, H, P, dtype=bf)), dict(cu=cu.reshape(1, 3))):
        with pytest.raises(ValueError, match="shape"):
            call(**kw)


def test_decode_shapes():
    b, H, P, G, N = 64, 80, 64, 1, 128
    state, x, dt, B = z(b, H, P, N), z(b, H, P), z(b, H), z(b, G, N)
    call = lambda **kw: ssd.ssd_decode_step(kw.get("state", state), kw.get("x", x), kw.get("dt", dt), z(H),
                                            kw.get("B", B), B, z(H), y_t=kw.get("y"))
    shapes_accepted(lambda: call())
    shapes_accepted(lambda: call(y=z(b, H, P)))
    for kw in (dict(state=z(b, H, N, P)), dict(state=z(b - 1, H, P, N)), dict(dt=z(b, H, 1)),
               dict(B=z(b, 2, N)), dict(y=z(b, H, P + 1)), dict(x=z(b, H * P))):
        with pytest.raises(ValueError, match="shape"):
            call(**kw)


def test_gdn_shapes():
    b, hqk, hv, dk, dv = 2, 16, 32, 128, 64
    state, q, v, g = z(b, hv, dk, dv), z(b, hqk, dk), z(b, hv, dv), z(b, hv)
    call = lambda **kw: ssd.ssd_gdn_decode_step(kw.get("state", state), q, kw.get("k", q), v, kw.get("g", g), g,
                                                out=kw.get("out"))
    shapes_accepted(lambda: call())
    shapes_accepted(lambda: ssd.ssd_gdn_decode_step(z(0, 32, 128, 128), z(0, 16, 128), z(0, 16, 128),
                                                    z(0, 32, 128), z(0, 32), z(0, 32)))
    for kw in (dict(state=z(b, hv, dv, dk)), dict(k=z(b, hqk, dk + 8)), dict(g=z(b, hqk)), dict(out=z(b, hv, dk))):
        with pytest.raises(ValueError, match="shape"):
            call(**kw)
