"""C ABI checks that need no GPU: the library loads, exports every function that
include/ssd.h declares, and rejects bad arguments on the host before any launch."""
import ctypes
import os
import re

import pytest

from state_space_model_05_b200 import binding
from state_space_model_05_b200.build import build

ROOT = os.path.dirname(os.path.dirname(os.path.abspath(__file__)))
HEADER = os.path.join(ROOT, "include", "ssd.h")


@pytest.fixture(scope="module")
def lib():
    build()
    return binding.lib()


def declared_functions():
    text = open(HEADER).read()
    text = re.sub(r"/\*.*?\*/", "", text, flags=re.S)
    return sorted(set(re.findall(r"\b(ssd_[a-z_]+)\s*\(", text)))


def test_exports_every_declared_function(lib):
    names = declared_functions()
    assert "ssd_prefill" in names and "ssd_decode_step" in names
    for n in names:
        assert hasattr(lib, n), f"{n} declared in ssd.h but not exported"
    assert set(names) == set(binding.SIGNATURES), "binding signatures out of sync with ssd.h"


def test_status_strings(lib):
    for code in range(0, 9):
        s = lib.ssd_status_string(code)
        assert s and s.decode() != "unknown status"
    assert lib.ssd_status_string(99).decode() == "unknown status"
    assert lib.ssd_abi_version() == 101


def _ws(*a):
    return binding.ssd_prefill_workspace_bytes(*a)


def test_workspace_bytes(lib):
    up = lambda v: (v + 255) // 256 * 256
    b, T, H, P, G, N, Q = 2, 300, 4, 64, 1, 128, 128
    c = 3
    # CUDA-core path: lam [b][H][c][2][Q] (hi and lo parts) + states [b][H][c][P][N]
    lam = b * H * c * 2 * Q * 4
    st = b * H * c * P * N * 4
    assert _ws(b, T, H, P, G, N, Q, binding.SSD_F32) == up(lam) + up(st)
    # tensor-core path (bf16, P 64, N 128, Q 128/256), sized by 128-token blocks: per block
    # Lam, dt and two column-factor rows; then either the two-pass kernels' chunk-state
    # weights and block decay and bf16 block-start-state images, or the fused kernels' bf16
    # G = C B^T per (b, g, block) with a two-head fp32 hand-off state and a flag per CTA
    # boundary (head pairs, at most 256 CTAs), whichever is larger; then the fp16 copy of B
    def tc_bytes(T):
        nb = -(-T // 128)
        fac = b * H * nb * 4 * 128 * 4           # Lam, dt, two column-factor rows
        wts = b * H * nb * (128 + 4) * 4          # chunk-state weights + block decay
        two_pass = up(wts) + up(b * H * nb * 16384)
        slots = min(b * G * (H // G // 2), 256) + 1
        fused = up(b * G * nb * 128 * 128 * 2) + up(slots * 2 * P * N * 4) + up(slots * 4)
        return up(fac) + max(two_pass, fused) + up(b * T * G * N * 2)
    assert _ws(b, T, H, P, G, N, Q, binding.SSD_BF16) == tc_bytes(T)
    assert _ws(b, T, H, P, G, N, 256, binding.SSD_BF16) == tc_bytes(T)
    # bf16 with other shapes uses the CUDA-core layout
    assert _ws(b, T, H, P, G, N, 64, binding.SSD_BF16) == up(b * H * 5 * 2 * 64 * 4) + up(b * H * 5 * P * N * 4)
    assert _ws(b, 0, H, P, G, N, Q, binding.SSD_F32) == 0
    assert _ws(b, T, H, 63, G, N, Q, binding.SSD_F32) == 0          # headdim not a multiple of 8
    assert _ws(b, T, 3, P, 2, N, Q, binding.SSD_F32) == 0           # nheads % ngroups
    assert _ws(b, T, H, P, G, N, 0, binding.SSD_F32) == 0
    assert _ws(b, T, H, P, G, N, Q, 7) == 0                         # bad dtype


FAKE = 0x10000  # 16-byte aligned dummy address; never dereferenced (calls fail validation first)


def _prefill(lib, **kw):
    a = dict(x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=FAKE, init=None, batch=1, seqlen=16,
             nheads=2, headdim=64, ngroups=1, dstate=128, chunk_len=16, dtype=binding.SSD_F32,
             y=FAKE, final=FAKE, ws=FAKE, ws_bytes=1 << 40, stream=None)
    a.update(kw)
    return lib.ssd_prefill(a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"], a["init"], a["batch"],
                           a["seqlen"], a["nheads"], a["headdim"], a["ngroups"], a["dstate"],
                           a["chunk_len"], a["dtype"], a["y"], a["final"], a["ws"], a["ws_bytes"],
                           a["stream"])


def test_prefill_validation(lib):
    E = binding
    assert _prefill(lib, nheads=3, ngroups=2) == 2
    assert _prefill(lib, headdim=12) == 2
    assert _prefill(lib, dstate=0) == 2
    assert _prefill(lib, seqlen=-1) == 2
    assert _prefill(lib, chunk_len=0) == 2
    assert _prefill(lib, chunk_len=512) == 5
    assert _prefill(lib, headdim=256) == 5
    assert _prefill(lib, dtype=5) == 3
    assert _prefill(lib, x=None) == 1
    assert _prefill(lib, final=None) == 1
    assert _prefill(lib, y=FAKE + 4) == 4
    assert _prefill(lib, init=FAKE + 8) == 4
    assert _prefill(lib, ws_bytes=16) == 8
    assert _prefill(lib, ws=None) == 8
    assert _prefill(lib, batch=0) == 0          # nothing to do, nothing launched


def _decode(lib, **kw):
    a = dict(state=FAKE, x=FAKE, dt=FAKE, A=FAKE, B=FAKE, C=FAKE, D=FAKE, batch=2, nheads=4,
             headdim=64, ngroups=1, dstate=128, dtype=binding.SSD_F32, y=FAKE, stream=None)
    a.update(kw)
    return lib.ssd_decode_step(a["state"], a["x"], a["dt"], a["A"], a["B"], a["C"], a["D"],
                               a["batch"], a["nheads"], a["headdim"], a["ngroups"], a["dstate"],
                               a["dtype"], a["y"], a["stream"])


def test_decode_validation(lib):
    assert _decode(lib, nheads=5, ngroups=2) == 2
    assert _decode(lib, dstate=1024) == 5
    assert _decode(lib, dstate=20) == 2
    assert _decode(lib, state=None) == 1
    assert _decode(lib, y=None) == 1
    assert _decode(lib, B=FAKE + 2) == 4
    assert _decode(lib, dtype=9) == 3
    assert _decode(lib, batch=-1) == 2
    assert _decode(lib, batch=0) == 0


def test_decode_steps_validation(lib):
    """Sizes and pointers are checked on the host before any launch."""
    f = lib.ssd_decode_steps
    args = lambda steps=3, nh=8, ng=1, ds=128, st=FAKE, y=FAKE, B=FAKE, dtype=binding.SSD_F32: (
        st, FAKE, FAKE, FAKE, B, FAKE, FAKE, steps, 2, nh, 64, ng, ds, dtype, y, None)
    assert f(*args(steps=-1)) == 2                   # negative step count
    assert f(*args(nh=6, ng=4)) == 2                 # nheads % ngroups
    assert f(*args(ds=1024)) == 5                    # dstate > 512
    assert f(*args(st=None)) == 1
    assert f(*args(y=None)) == 1
    assert f(*args(B=FAKE + 4)) == 4                 # misaligned
    assert f(*args(dtype=9)) == 3
    assert f(*args(steps=0, st=None)) == 0           # nothing to do


def test_decode_layers_validation(lib):
    """Sizes are checked on the host before any launch; the table is read only by the kernel."""
    f = lib.ssd_decode_step_layers
    assert f(FAKE, 4, 2, 6, 64, 4, 128, binding.SSD_F32, None) == 2      # nheads % ngroups
    assert f(FAKE, 4, 2, 8, 64, 4, 1024, binding.SSD_F32, None) == 5     # dstate > 512
    assert f(FAKE, 4, 2, 8, 64, 4, 128, 7, None) == 3                    # dtype
    assert f(FAKE, -1, 2, 8, 64, 4, 128, binding.SSD_F32, None) == 2     # n_layers
    assert f(None, 4, 2, 8, 64, 4, 128, binding.SSD_F32, None) == 1      # NULL table
    assert f(FAKE + 4, 4, 2, 8, 64, 4, 128, binding.SSD_F32, None) == 4  # misaligned table
    assert f(None, 0, 2, 8, 64, 4, 128, binding.SSD_F32, None) == 0      # nothing to do
    assert f(None, 4, 0, 8, 64, 4, 128, binding.SSD_F32, None) == 0


def test_decode_steps_layers_validation(lib):
    """The multi-step stack call validates sizes on the host before any launch, like the
    one-step stack call, and also rejects a negative step count."""
    f = lib.ssd_decode_steps_layers
    F32 = binding.SSD_F32
    assert f(FAKE, 4, 3, 2, 6, 64, 4, 128, F32, None) == 2       # nheads % ngroups
    assert f(FAKE, 4, 3, 2, 8, 64, 4, 1024, F32, None) == 5      # dstate > 512
    assert f(FAKE, 4, 3, 2, 8, 64, 4, 128, 7, None) == 3         # dtype
    assert f(FAKE, -1, 3, 2, 8, 64, 4, 128, F32, None) == 2      # n_layers < 0
    assert f(FAKE, 65536, 3, 2, 8, 64, 4, 128, F32, None) == 2   # n_layers > 65535
    assert f(FAKE, 4, -1, 2, 8, 64, 4, 128, F32, None) == 2      # steps < 0
    assert f(None, 4, 3, 2, 8, 64, 4, 128, F32, None) == 1       # NULL table
    assert f(FAKE + 4, 4, 3, 2, 8, 64, 4, 128, F32, None) == 4   # misaligned table
    assert f(None, 0, 3, 2, 8, 64, 4, 128, F32, None) == 0       # nothing to do
    assert f(None, 4, 0, 2, 8, 64, 4, 128, F32, None) == 0
    assert f(None, 4, 3, 0, 8, 64, 4, 128, F32, None) == 0


def test_dtraw_validation(lib):
    """The raw-dt variants validate like the plain calls, and reject a misaligned bias
    (every call here fails validation before any launch)."""
    F = FAKE
    f = lib.ssd_decode_step_dtraw
    assert f(F, F, F, F + 4, F, F, F, F, 2, 8, 64, 4, 128, binding.SSD_F32, F, None) == 4
    assert f(F, F, F, None, F, F, F, F, 2, 6, 64, 4, 128, binding.SSD_F32, F, None) == 2
    p = lib.ssd_prefill_dtraw
    args = [F, F, F + 4, F, F, F, F, None, 2, 300, 4, 64, 1, 128, 128, binding.SSD_BF16, F, F, F, 1 << 30, None]
    assert p(*args) == 4                                   # misaligned bias
    args[2] = F
    args[9] = -1
    assert p(*args) == 2                                   # bad seqlen


def test_varlen_validation(lib):
    """Workspace sizes of both paths; every call below fails validation before any launch
    (a zero workspace where the sizes themselves are valid)."""
    F = FAKE
    ws = lib.ssd_prefill_varlen_workspace_bytes
    up = lambda v: (v + 255) // 256 * 256
    nseq, T, H = 3, 1000, 4
    nb = T // 128 + nseq                             # tensor-core block bound: floor(T / 128) + nseq
    main = (up(H * nb * 4 * 128 * 4) + up(H * nb * 132 * 4) + up(H * nb * 16384) + up(T * 128 * 2))
    assert ws(nseq, T, H, 64, 1, 128, 256, binding.SSD_BF16) == main + up((nseq + 1) * 4) + up(nb * 4)
    assert ws(nseq, 0, H, 64, 1, 128, 256, binding.SSD_BF16) == 0
    nc = T // 64 + nseq                              # CUDA-core chunks of 64: lam + per-chunk fp32 states
    simt = up(H * nc * 2 * 64 * 4) + up(H * nc * 64 * 128 * 4)
    assert ws(nseq, T, H, 64, 1, 128, 64, binding.SSD_F32) == simt + up((nseq + 1) * 4) + up(nc * 4)
    f = lib.ssd_prefill_varlen
    args = lambda **kw: [F, F, F, F, F, F, None, kw.get("cu", F), kw.get("nseq", 3), kw.get("T", 1000), 4,
                         kw.get("P", 64), 1, 128, kw.get("Q", 256), kw.get("dtype", binding.SSD_BF16), F, F, F,
                         kw.get("wsb", 0), None]
    assert f(*args()) == 8                           # workspace too small (checked before any launch)
    assert f(*args(dtype=binding.SSD_F32)) == 8      # CUDA-core path, same check
    assert f(*args(Q=512)) == 5
    assert f(*args(P=12)) == 2
    assert f(*args(dtype=7)) == 3
    assert f(*args(nseq=0)) == 2
    assert f(*args(T=-1)) == 2
    assert f(*args(cu=None)) == 1
    assert f(*args(cu=F + 2)) == 4


def test_gdn_validation(lib):
    f = lib.ssd_gdn_decode_step
    F = FAKE
    args = lambda **kw: [kw.get("state", F), F, F, F, F, F, kw.get("batch", 2), kw.get("hqk", 16),
                         kw.get("hv", 32), kw.get("dk", 128), kw.get("dv", 128), kw.get("dtype", binding.SSD_F32),
                         kw.get("out", F), None]
    assert f(*args(hv=24, hqk=16)) == 2        # value heads not a multiple of query/key heads
    assert f(*args(dk=12)) == 2                # dk not a multiple of 8
    assert f(*args(dv=6)) == 2                 # dv not a multiple of 4
    assert f(*args(dk=256)) == 5               # beyond the supported state
    assert f(*args(dv=256)) == 5
    assert f(*args(dtype=4)) == 3
    assert f(*args(state=None)) == 1
    assert f(*args(out=F + 8)) == 4
    assert f(*args(batch=-1)) == 2
    assert f(*args(batch=0, state=None)) == 0  # nothing to do


def test_binding_fails_loudly_without_library(monkeypatch, tmp_path):
    monkeypatch.setattr(binding, "LIB_PATH", str(tmp_path / "missing.so"))
    monkeypatch.setattr(binding, "_lib", None)
    with pytest.raises(RuntimeError, match="not built"):
        binding.lib()


def test_selftest_rejects_null_scratch(lib):
    assert lib.ssd_selftest_bounded_waits(None, None) == 1


def test_prefill_path_setting(lib):
    """The tensor-core path selector: known values round-trip, others are refused."""
    prev = lib.ssd_get_prefill_path()
    try:
        for v in (1, 2, 0):
            assert lib.ssd_set_prefill_path(v) == 0
            assert lib.ssd_get_prefill_path() == v
        assert lib.ssd_set_prefill_path(3) == 2
        assert lib.ssd_set_prefill_path(-1) == 2
        assert lib.ssd_get_prefill_path() == 0
        assert binding.ssd_set_prefill_path("two_pass") == "auto"
        assert binding.ssd_get_prefill_path() == "two_pass"
    finally:
        lib.ssd_set_prefill_path(prev)
