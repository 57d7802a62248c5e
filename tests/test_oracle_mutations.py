"""Plant plausible mistakes in a copy of the oracle and check that the pins catch each.

The mistakes are planted in a temporary copy of the oracle's C source, compiled
on the CPU; the committed oracle is untouched.  Every mutant must fail at least
one of the pins below (hand-worked case, separately written chunked form,
prefill/decode resume, group mapping).  Ten mutants change the recurrence wherever
it is written; six more change the decode step alone, with the prefill correct.
"""
import json
import math
import os
import re
import subprocess

import numpy as np
import pytest

import oracle
from oracle import forms

HERE = os.path.dirname(os.path.abspath(__file__))
SRC = os.path.join(os.path.dirname(HERE), "oracle", "ssd_oracle.c")
GOLDEN = os.path.join(HERE, "golden", "ssd_tiny_hand.json")

UPDATE = r"Hp\[n\] = a \* Hp\[n\] \+ dx \* \(double\)Bt\[n\];"
MUTANTS = {
    "no_decay": (UPDATE, "Hp[n] = Hp[n] + dx * (double)Bt[n];"),
    "exp_sign": (r"exp\(dtv \* \(double\)A\[h\]\)", "exp(-dtv * (double)A[h])"),
    "y_before_update": (r"(Hp\[n\] = a \* Hp\[n\] \+ dx \* \(double\)Bt\[n\];)(\s*)(acc \+= \(double\)Ct\[n\] \* Hp\[n\];)",
                        r"\3\2\1"),
    "no_skip": (r" \+ \(double\)D\[h\] \* \(double\)xt\[p\]", ""),
    "B_for_C": (r"acc \+= \(double\)Ct\[n\]", "acc += (double)Bt[n]"),
    "group_modulo": (r"g = h / heads_per_group", "g = h % ngroups"),
    "no_dt_on_input": (r"const double dx = dtv \* \(double\)xt\[p\];", "const double dx = (double)xt[p];"),
    "dt_off_by_one": (r"dt\[tok \* nheads \+ h\]", "dt[(t > 0 ? tok - 1 : tok) * nheads + h]"),
    "init_ignored": (r"if \(init\)", "if (0)"),
    "decay_squared": (r"Hp\[n\] = a \* Hp\[n\]", "Hp[n] = a * a * Hp[n]"),
}
# the same kinds of mistake planted in the decode step alone (the prefill left correct): the
# resume pin, prefill(T0) followed by decode steps against prefill(T), must catch each
DECODE_MUTANTS = {
    "decode_no_decay": MUTANTS["no_decay"],
    "decode_exp_sign": MUTANTS["exp_sign"],
    "decode_y_before_update": MUTANTS["y_before_update"],
    "decode_no_skip": MUTANTS["no_skip"],
    "decode_group_modulo": MUTANTS["group_modulo"],
    "decode_B_ignores_batch": (r"B_t \+ \(\(size_t\)b \* ngroups \+ g\) \* dstate", "B_t + (size_t)g * dstate"),
}
DECODE_ENTRY = "int ssd_oracle_decode_step("


def _build_mutant(tmp_path, name):
    src = open(SRC).read()
    if name in DECODE_MUTANTS:
        pat, rep = DECODE_MUTANTS[name]
        cut = src.index(DECODE_ENTRY)
        tail, n = re.subn(pat, rep, src[cut:])
        mutated = src[:cut] + tail
    else:
        pat, rep = MUTANTS[name]
        mutated, n = re.subn(pat, rep, src)
    assert n >= 1, f"mutation {name} did not apply"
    c = tmp_path / f"{name}.c"
    so = tmp_path / f"lib_{name}.so"
    c.write_text(mutated)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", "-o", str(so), str(c), "-lm"])
    return oracle.bind(str(so))


def _close(a, b, tol=1e-9):
    return np.allclose(a, b, rtol=tol, atol=1e-12)


def _pins_pass(lib) -> bool:
    g = json.load(open(GOLDEN))
    inp = {k: np.array(v, dtype=np.float32) for k, v in g["inputs"].items()}
    ev = lambda s: float(eval(s, {"__builtins__": {}}, {"exp": math.exp}))
    for c in g["cases"]:
        init = None if c["init"] is None else np.array(c["init"], dtype=np.float64)[None]
        y, s = oracle.prefill(inp["x"], inp["dt"], inp["A"], inp["B"], inp["C"], inp["D"],
                              init=init, lib=lib)
        if not _close(y[0], [[ev(v) for v in r] for r in c["y"]], 1e-13):
            return False
        if not _close(s[0], [[ev(v) for v in r] for r in c["state"]], 1e-13):
            return False
    rng = np.random.default_rng(1)
    b, T, H, P, G, N = 2, 70, 4, 3, 2, 5
    x = rng.standard_normal((b, T, H, P)).astype(np.float32)
    dt = np.exp(rng.uniform(np.log(1e-3), np.log(0.3), (b, T, H))).astype(np.float32)
    A = (-np.exp(rng.uniform(0, np.log(16), H))).astype(np.float32)
    B = (rng.standard_normal((b, T, G, N)) / np.sqrt(N)).astype(np.float32)
    C = (rng.standard_normal((b, T, G, N)) / np.sqrt(N)).astype(np.float32)
    D = rng.standard_normal(H).astype(np.float32)
    init = rng.standard_normal((b * H, P, N))
    y, s = oracle.prefill(x, dt, A, B, C, D, init=init, lib=lib)
    yc, sc = forms.chunked(x, dt, A, B, C, D, 16, init=init.reshape(b, H, P, N))
    if not _close(oracle.units_to_bthp(y, b, H), yc) or not _close(s.reshape(b, H, P, N), sc):
        return False
    # resume: prefill(T0) + decode steps == prefill(T)
    T0 = 60
    _, st = oracle.prefill(x[:, :T0], dt[:, :T0], A, B[:, :T0], C[:, :T0], D, lib=lib)
    y_full, s_full = oracle.prefill(x, dt, A, B, C, D, lib=lib)
    for k in range(T0, T):
        yk = oracle.decode_step(st, x[:, k], dt[:, k], A, B[:, k], C[:, k], D, lib=lib)
        if not _close(yk, y_full[:, k]):
            return False
    return _close(st, s_full)


def test_unmutated_copy_passes(tmp_path):
    so = tmp_path / "lib_clean.so"
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC",
                           "-shared", "-o", str(so), SRC, "-lm"])
    assert _pins_pass(oracle.bind(str(so)))


@pytest.mark.parametrize("name", sorted(MUTANTS) + sorted(DECODE_MUTANTS))
def test_mutant_is_caught(tmp_path, name):
    lib = _build_mutant(tmp_path, name)
    assert not _pins_pass(lib), f"planted mistake '{name}' passed every pin"
