"""ctypes binding of the SSD C ABI (``include/ssd.h``).

Argument marshalling only: tensors are passed as device pointers together with
the current CUDA stream; every step of the computation runs in the CUDA library.
There is no fallback -- if ``libssd.so`` is missing or a call fails, an exception
is raised.
"""
from __future__ import annotations

import ctypes
import os

import torch

HERE = os.path.dirname(os.path.abspath(__file__))
LIB_PATH = os.path.join(HERE, "libssd.so")

SSD_OK = 0
SSD_ERR_NULL = 1
SSD_ERR_ALIGN = 4
SSD_ERR_TIMEOUT = 7
SSD_F32 = 0
SSD_BF16 = 1

STATUS_NAMES = {0: "SSD_OK", 1: "SSD_ERR_NULL", 2: "SSD_ERR_SHAPE", 3: "SSD_ERR_DTYPE",
                4: "SSD_ERR_ALIGN", 5: "SSD_ERR_UNSUPPORTED", 6: "SSD_ERR_CUDA",
                7: "SSD_ERR_TIMEOUT", 8: "SSD_ERR_WORKSPACE"}

# exported symbols and their ctypes signatures, as declared in include/ssd.h
_P, _I, _Z = ctypes.c_void_p, ctypes.c_int, ctypes.c_size_t
SIGNATURES = {
    "ssd_abi_version": ([], _I),
    "ssd_status_string": ([_I], ctypes.c_char_p),
    "ssd_prefill_workspace_bytes": ([_I, _I, _I, _I, _I, _I, _I, _I], _Z),
    "ssd_prefill": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _Z, _P], _I),
    "ssd_decode_step": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P], _I),
    "ssd_decode_steps": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _P, _P], _I),
    "ssd_decode_step_layers": ([_P, _I, _I, _I, _I, _I, _I, _I, _P], _I),
    "ssd_decode_steps_layers": ([_P, _I, _I, _I, _I, _I, _I, _I, _I, _P], _I),
    "ssd_gdn_decode_step": ([_P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P], _I),
    "ssd_prefill_varlen_workspace_bytes": ([_I, _I, _I, _I, _I, _I, _I, _I], _Z),
    "ssd_prefill_varlen": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _Z, _P], _I),
    "ssd_prefill_dtraw": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P, _Z, _P], _I),
    "ssd_decode_step_dtraw": ([_P, _P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _P, _P], _I),
    "ssd_prefill_noalloc": ([_P, _P, _P, _P, _P, _P, _P, _I, _I, _I, _I, _I, _I, _I, _I, _P, _P, _P], _I),
    "ssd_device_status": ([_P], _I),
    "ssd_set_prefill_path": ([_I], _I),
    "ssd_get_prefill_path": ([], _I),
    "ssd_selftest_bounded_waits": ([_P, _P], _I),
    "ssd_profile_enable": ([_I], None),
    "ssd_profile_reset": ([], None),
    "ssd_profile_read": ([_I, ctypes.POINTER(ctypes.c_char_p), ctypes.POINTER(ctypes.c_double),
                          ctypes.POINTER(ctypes.c_longlong)], _I),
}

_lib = None


class SSDError(RuntimeError):
    def __init__(self, status: int, what: str):
        self.status = status
        super().__init__(f"{what}: {STATUS_NAMES.get(status, status)} ({_status_text(status)})")


def lib() -> ctypes.CDLL:
    """The loaded C library (raises if the CUDA extension has not been built)."""
    global _lib
    if _lib is None:
        if not os.path.exists(LIB_PATH):
            raise RuntimeError(f"SSD CUDA library not built: {LIB_PATH} is missing "
                               "(run `python -m state_space_model_05_b200.build`)")
        l = ctypes.CDLL(LIB_PATH)
        for name, (args, res) in SIGNATURES.items():
            fn = getattr(l, name)
            fn.argtypes = args
            fn.restype = res
        _lib = l
    return _lib


def _status_text(status: int) -> str:
    try:
        return lib().ssd_status_string(status).decode()
    except Exception:  # noqa: BLE001 - only used for messages
        return "?"


def _check(status: int, what: str):
    if status != SSD_OK:
        raise SSDError(status, what)


def _dtype_code(t: torch.Tensor) -> int:
    if t.dtype == torch.float32:
        return SSD_F32
    if t.dtype == torch.bfloat16:
        return SSD_BF16
    raise TypeError(f"unsupported dtype {t.dtype} (float32 or bfloat16)")


def _ptr(t):
    return None if t is None else ctypes.c_void_p(t.data_ptr())


def _stream(stream=None):
    s = torch.cuda.current_stream() if stream is None else stream
    return ctypes.c_void_p(s.cuda_stream)


def _need(t: torch.Tensor, name: str, dtype=None):
    if not t.is_cuda:
        raise ValueError(f"{name} must be a CUDA tensor")
    if not t.is_contiguous():
        raise ValueError(f"{name} must be contiguous")
    if dtype is not None and t.dtype != dtype:
        raise TypeError(f"{name} must be {dtype}")


def _rank(t: torch.Tensor, name: str, layout: str):
    """Raise unless ``t`` has one axis per name in ``layout`` (e.g. "[batch][seqlen][nheads]")."""
    if t.dim() != layout.count("["):
        raise ValueError(f"{name} must be {layout}, got shape {tuple(t.shape)}")


def _check_args(ref: torch.Tensor, specs):
    """Validate the tensors of one call before anything reaches the library, which sees only
    pointers and so cannot tell a short buffer from a right one.  ``specs`` holds
    (tensor or None, name, expected shape, dtype or None); every tensor given must have that
    shape, live on ``ref``'s device, be a contiguous CUDA tensor and (if stated) have that
    dtype.  ``ref`` must be on the current device, whose stream the library launches on."""
    for t, name, shape, _ in specs:
        if t is not None and tuple(t.shape) != tuple(shape):
            raise ValueError(f"{name} has shape {tuple(t.shape)}, expected {tuple(shape)}")
    for t, name, _, dtype in specs:
        if t is None:
            continue
        _need(t, name, dtype)
        if t.device != ref.device:
            raise ValueError(f"{name} is on {t.device}, expected {ref.device}")
    if ref.device.index != torch.cuda.current_device():
        raise ValueError(f"tensors are on {ref.device} but the current device is "
                         f"cuda:{torch.cuda.current_device()}")


def ssd_prefill_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len, dtype_code):
    return int(lib().ssd_prefill_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate,
                                                 chunk_len, dtype_code))


PREFILL_PATHS = {"auto": 0, "fused": 1, "two_pass": 2}


def ssd_set_prefill_path(path: str) -> str:
    """Select the tensor-core prefill kernels ("auto", "fused" or "two_pass"; see
    ``include/ssd.h``); returns the previous setting."""
    prev = ssd_get_prefill_path()
    _check(lib().ssd_set_prefill_path(PREFILL_PATHS[path]), "ssd_set_prefill_path")
    return prev


def ssd_get_prefill_path() -> str:
    code = int(lib().ssd_get_prefill_path())
    return next(k for k, v in PREFILL_PATHS.items() if v == code)


def ssd_prefill(x, dt, A, B, C, D, chunk_len, init_state=None, y=None, final_state=None,
                workspace=None, stream=None, dt_softplus=False, dt_bias=None):
    """Chunked SSD prefill.  Shapes as in ``include/ssd.h``; returns ``(y, final_state)``.
    With ``dt_softplus`` the kernels use softplus(dt + dt_bias) (ssd_prefill_dtraw)."""
    _rank(x, "x", "[batch][seqlen][nheads][headdim]")
    _rank(B, "B", "[batch][seqlen][ngroups][dstate]")
    batch, seqlen, nheads, headdim = x.shape
    ngroups, dstate = B.shape[2], B.shape[3]
    f32, state_shape = torch.float32, (batch, nheads, headdim, dstate)
    _check_args(x, ((x, "x", x.shape, x.dtype), (dt, "dt", (batch, seqlen, nheads), f32),
                    (A, "A", (nheads,), f32), (B, "B", B.shape, x.dtype),
                    (C, "C", B.shape, x.dtype), (D, "D", (nheads,), f32),
                    (init_state, "init_state", state_shape, f32), (y, "y", x.shape, x.dtype),
                    (final_state, "final_state", state_shape, f32),
                    (dt_bias if dt_softplus else None, "dt_bias", (nheads,), f32),
                    (workspace, "workspace", workspace.shape if workspace is not None else (), None)))
    code = _dtype_code(x)
    if y is None:
        y = torch.empty_like(x)
    if final_state is None:
        final_state = torch.empty(state_shape, device=x.device, dtype=f32)
    need = ssd_prefill_workspace_bytes(batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len, code)
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=x.device, dtype=torch.uint8)
    if dt_softplus:
        st = lib().ssd_prefill_dtraw(_ptr(x), _ptr(dt), _ptr(dt_bias), _ptr(A), _ptr(B), _ptr(C), _ptr(D),
                                     _ptr(init_state), batch, seqlen, nheads, headdim, ngroups, dstate,
                                     chunk_len, code, _ptr(y), _ptr(final_state), _ptr(workspace),
                                     workspace.numel(), _stream(stream))
        _check(st, "ssd_prefill_dtraw")
        return y, final_state
    st = lib().ssd_prefill(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_state),
                           batch, seqlen, nheads, headdim, ngroups, dstate, chunk_len, code,
                           _ptr(y), _ptr(final_state), _ptr(workspace), workspace.numel(),
                           _stream(stream))
    _check(st, "ssd_prefill")
    return y, final_state


def ssd_prefill_varlen(x, dt, A, B, C, D, cu_seqlens, chunk_len, init_states=None, y=None,
                       final_states=None, workspace=None, stream=None):
    """Packed variable-length prefill.  x [T][H][P], dt [T][H], B/C [T][G][N] (the batch-1
    layouts without the batch axis), cu_seqlens a CUDA int32 tensor of nseq + 1 offsets.
    Returns ``(y, final_states)``, final_states [nseq][H][P][N]."""
    _rank(x, "x", "[tokens][nheads][headdim]")
    _rank(B, "B", "[tokens][ngroups][dstate]")
    _rank(cu_seqlens, "cu_seqlens", "[nseq + 1]")
    total, nheads, headdim = x.shape
    ngroups, dstate = B.shape[1], B.shape[2]
    nseq = cu_seqlens.numel() - 1
    f32, state_shape = torch.float32, (nseq, nheads, headdim, dstate)
    _check_args(x, ((x, "x", x.shape, x.dtype), (dt, "dt", (total, nheads), f32), (A, "A", (nheads,), f32),
                    (B, "B", B.shape, x.dtype), (C, "C", B.shape, x.dtype), (D, "D", (nheads,), f32),
                    (cu_seqlens, "cu_seqlens", cu_seqlens.shape, torch.int32),
                    (init_states, "init_states", state_shape, f32), (y, "y", x.shape, x.dtype),
                    (final_states, "final_states", state_shape, f32),
                    (workspace, "workspace", workspace.shape if workspace is not None else (), None)))
    code = _dtype_code(x)
    if y is None:
        y = torch.empty_like(x)
    if final_states is None:
        final_states = torch.empty(state_shape, device=x.device, dtype=f32)
    need = int(lib().ssd_prefill_varlen_workspace_bytes(nseq, total, nheads, headdim, ngroups, dstate,
                                                        chunk_len, code))
    if workspace is None:
        workspace = torch.empty(max(need, 1), device=x.device, dtype=torch.uint8)
    st = lib().ssd_prefill_varlen(_ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), _ptr(init_states),
                                  _ptr(cu_seqlens), nseq, total, nheads, headdim, ngroups, dstate, chunk_len,
                                  code, _ptr(y), _ptr(final_states), _ptr(workspace), workspace.numel(),
                                  _stream(stream))
    _check(st, "ssd_prefill_varlen")
    return y, final_states


def ssd_decode_step(state, x_t, dt_t, A, B_t, C_t, D, y_t=None, stream=None, dt_softplus=False,
                    dt_bias=None):
    """One decode step; ``state`` [b][H][P][N] fp32 is updated in place.  Returns ``y_t``.
    With ``dt_softplus`` the kernel uses softplus(dt_t + dt_bias) (ssd_decode_step_dtraw)."""
    _rank(x_t, "x_t", "[batch][nheads][headdim]")
    _rank(B_t, "B_t", "[batch][ngroups][dstate]")
    batch, nheads, headdim = x_t.shape
    ngroups, dstate = B_t.shape[1], B_t.shape[2]
    f32 = torch.float32
    _check_args(x_t, ((state, "state", (batch, nheads, headdim, dstate), f32), (x_t, "x_t", x_t.shape, x_t.dtype),
                      (dt_t, "dt_t", (batch, nheads), f32), (A, "A", (nheads,), f32),
                      (B_t, "B_t", B_t.shape, x_t.dtype), (C_t, "C_t", B_t.shape, x_t.dtype),
                      (D, "D", (nheads,), f32), (y_t, "y_t", x_t.shape, x_t.dtype),
                      (dt_bias if dt_softplus else None, "dt_bias", (nheads,), f32)))
    if y_t is None:
        y_t = torch.empty_like(x_t)
    if dt_softplus:
        st = lib().ssd_decode_step_dtraw(_ptr(state), _ptr(x_t), _ptr(dt_t), _ptr(dt_bias), _ptr(A), _ptr(B_t),
                                         _ptr(C_t), _ptr(D), batch, nheads, headdim, ngroups, dstate,
                                         _dtype_code(x_t), _ptr(y_t), _stream(stream))
        _check(st, "ssd_decode_step_dtraw")
        return y_t
    st = lib().ssd_decode_step(_ptr(state), _ptr(x_t), _ptr(dt_t), _ptr(A), _ptr(B_t), _ptr(C_t),
                               _ptr(D), batch, nheads, headdim, ngroups, dstate, _dtype_code(x_t),
                               _ptr(y_t), _stream(stream))
    _check(st, "ssd_decode_step")
    return y_t


def ssd_decode_steps(state, x, dt, A, B, C, D, y=None, stream=None):
    """``steps`` decode steps in one launch; ``state`` [b][H][P][N] fp32 is updated in place.
    x [steps][b][H][P], dt [steps][b][H], B/C [steps][b][G][N].  Returns y [steps][b][H][P]."""
    _rank(x, "x", "[steps][batch][nheads][headdim]")
    _rank(B, "B", "[steps][batch][ngroups][dstate]")
    steps, batch, nheads, headdim = x.shape
    ngroups, dstate = B.shape[2], B.shape[3]
    f32 = torch.float32
    _check_args(x, ((state, "state", (batch, nheads, headdim, dstate), f32), (x, "x", x.shape, x.dtype),
                    (dt, "dt", (steps, batch, nheads), f32), (A, "A", (nheads,), f32),
                    (B, "B", B.shape, x.dtype), (C, "C", B.shape, x.dtype), (D, "D", (nheads,), f32),
                    (y, "y", x.shape, x.dtype)))
    if y is None:
        y = torch.empty_like(x)
    st = lib().ssd_decode_steps(_ptr(state), _ptr(x), _ptr(dt), _ptr(A), _ptr(B), _ptr(C), _ptr(D), steps,
                                batch, nheads, headdim, ngroups, dstate, _dtype_code(x), _ptr(y), _stream(stream))
    _check(st, "ssd_decode_steps")
    return y


# field order of ssd_decode_layer_t
LAYER_FIELDS = ("state", "x_t", "dt_t", "A", "B_t", "C_t", "D", "y_t")


def decode_layer_table(layers, device=None):
    """Device array of ssd_decode_layer_t (int64 [n_layers][8]) from a list of dicts of
    tensors keyed by LAYER_FIELDS (their data pointers, in field order)."""
    rows = [[int(layer[f].data_ptr()) for f in LAYER_FIELDS] for layer in layers]
    dev = device or layers[0]["state"].device
    return torch.tensor(rows, dtype=torch.int64, device=dev).reshape(len(rows), len(LAYER_FIELDS))


def ssd_decode_step_layers(table, batch, nheads, headdim, ngroups, dstate, dtype, stream=None):
    """One decode step of every layer in ``table`` (from decode_layer_table), one launch."""
    if not table.is_cuda or table.dtype != torch.int64 or table.dim() != 2 or table.shape[1] != len(LAYER_FIELDS):
        raise ValueError("table must be a CUDA int64 [n_layers][8] tensor")
    code = SSD_BF16 if dtype in (torch.bfloat16, SSD_BF16) else SSD_F32
    st = lib().ssd_decode_step_layers(_ptr(table), table.shape[0], batch, nheads, headdim, ngroups,
                                      dstate, code, _stream(stream))
    _check(st, "ssd_decode_step_layers")


def ssd_decode_steps_layers(table, steps, batch, nheads, headdim, ngroups, dstate, dtype, stream=None):
    """``steps`` decode steps of every layer in ``table`` (from decode_layer_table, whose
    per-step entries point at each layer's [steps][...] arrays), one launch."""
    if not table.is_cuda or table.dtype != torch.int64 or table.dim() != 2 or table.shape[1] != len(LAYER_FIELDS):
        raise ValueError("table must be a CUDA int64 [n_layers][8] tensor")
    code = SSD_BF16 if dtype in (torch.bfloat16, SSD_BF16) else SSD_F32
    st = lib().ssd_decode_steps_layers(_ptr(table), table.shape[0], steps, batch, nheads, headdim, ngroups,
                                       dstate, code, _stream(stream))
    _check(st, "ssd_decode_steps_layers")


def ssd_gdn_decode_step(state, q, k, v, gate, beta, out=None, stream=None):
    """One Gated DeltaNet decode step; ``state`` [b][hv][dk][dv] fp32 is updated in place.
    q, k [b][hqk][dk]; v [b][hv][dv] (fp32 or bf16, all alike); gate, beta [b][hv] fp32.
    Returns ``out`` [b][hv][dv]."""
    _rank(q, "q", "[batch][heads_qk][dk]")
    _rank(v, "v", "[batch][heads_v][dv]")
    batch, hqk, dk = q.shape
    hv, dv = v.shape[1], v.shape[2]
    f32 = torch.float32
    _check_args(q, ((state, "state", (batch, hv, dk, dv), f32), (q, "q", q.shape, q.dtype),
                    (k, "k", q.shape, q.dtype), (v, "v", (batch, hv, dv), q.dtype),
                    (gate, "gate", (batch, hv), f32), (beta, "beta", (batch, hv), f32),
                    (out, "out", (batch, hv, dv), q.dtype)))
    if out is None:
        out = torch.empty_like(v)
    st = lib().ssd_gdn_decode_step(_ptr(state), _ptr(q), _ptr(k), _ptr(v), _ptr(gate), _ptr(beta), batch,
                                   hqk, hv, dk, dv, _dtype_code(q), _ptr(out), _stream(stream))
    _check(st, "ssd_gdn_decode_step")
    return out


def ssd_device_status(stream=None) -> int:
    """Synchronise the stream and return (and clear) the device error word."""
    return int(lib().ssd_device_status(_stream(stream)))


def ssd_profile_enable(on: bool = True):
    lib().ssd_profile_enable(1 if on else 0)


def ssd_profile_reset():
    lib().ssd_profile_reset()


def ssd_profile_read() -> dict:
    """{kernel name: (total_ms, launches)} since the last reset (synchronises)."""
    n = 16
    names = (ctypes.c_char_p * n)()
    ms = (ctypes.c_double * n)()
    cnt = (ctypes.c_longlong * n)()
    k = lib().ssd_profile_read(n, names, ms, cnt)
    if k < 0:
        raise SSDError(6, "ssd_profile_read")
    return {names[i].decode(): (ms[i], cnt[i]) for i in range(k)}
