"""Pins of the fp64 Gated DeltaNet decode oracle against what the page and the algebra fix:
a hand-worked case, closed forms for gate/beta at their extremes, the page's two-pass
identity, and the value-head -> query/key-head grouping.  Planted mistakes in a copy of the
C source must each fail one of them."""
import json
import os
import re
import subprocess

import numpy as np
import pytest

from oracle import gdn

HERE = os.path.dirname(os.path.abspath(__file__))
GOLDEN = os.path.join(HERE, "golden", "gdn_tiny_hand.json")
SRC = os.path.join(os.path.dirname(HERE), "oracle", "gdn_oracle.c")


def _rand(seed, b=2, hqk=2, hv=4, dk=8, dv=6):
    r = np.random.default_rng(seed)
    q = r.standard_normal((b, hqk, dk)).astype(np.float32)
    k = r.standard_normal((b, hqk, dk)).astype(np.float32)
    k /= np.linalg.norm(k, axis=-1, keepdims=True)
    v = r.standard_normal((b, hv, dv)).astype(np.float32)
    gate = r.uniform(0.5, 1.0, (b, hv)).astype(np.float32)
    beta = r.uniform(0.0, 1.0, (b, hv)).astype(np.float32)
    S = r.standard_normal((b, hv, dk, dv))
    return S, q, k, v, gate, beta


def _expand(a, hv):
    """query/key heads repeated for each value head of their group"""
    return np.repeat(a, hv // a.shape[1], axis=1)


def _hand(lib=None):
    g = json.load(open(GOLDEN))
    i = g["inputs"]
    S = np.array(i["S"], dtype=np.float64)[None, None]
    f = lambda a: np.array(a, dtype=np.float32)[None, None]
    o = gdn.decode_step(S, f(i["q"]), f(i["k"]), f(i["v"]), np.float32([[i["gate"]]]),
                        np.float32([[i["beta"]]]), lib=lib)
    return S[0, 0], o[0, 0], g["expected"]


def test_hand_worked_case():
    S, o, want = _hand()
    np.testing.assert_allclose(S, want["S"], rtol=0, atol=1e-15)
    np.testing.assert_allclose(o, want["o"], rtol=0, atol=1e-15)


def _closed_forms(lib=None):
    S0, q, k, v, gate, beta = _rand(1)
    hv = v.shape[1]
    qe, ke = _expand(q, hv).astype(np.float64), _expand(k, hv).astype(np.float64)
    ok = True
    # gate 1, beta 0: the state is unchanged and the output is S^T q
    S = S0.copy()
    o = gdn.decode_step(S, q, k, v, np.ones_like(gate), np.zeros_like(beta), lib=lib)
    ok &= np.allclose(S, S0, rtol=0, atol=0)
    ok &= np.allclose(o, np.einsum("bhij,bhi->bhj", S0, qe), rtol=1e-12, atol=1e-12)
    # gate 0: the state becomes beta k v^T and the output beta (q.k) v
    S = S0.copy()
    o = gdn.decode_step(S, q, k, v, np.zeros_like(gate), beta, lib=lib)
    bv = beta[..., None].astype(np.float64) * v
    ok &= np.allclose(S, np.einsum("bhi,bhj->bhij", ke, bv), rtol=1e-12, atol=1e-12)
    ok &= np.allclose(o, np.einsum("bhi,bhi->bh", qe, ke)[..., None] * bv, rtol=1e-12, atol=1e-12)
    # gate 1, beta 1, k a unit vector e_i: row i of the state is overwritten with v exactly
    dk = k.shape[-1]
    kk = np.zeros_like(k)
    kk[..., 3] = 1.0
    S = S0.copy()
    gdn.decode_step(S, q, kk, v, np.ones_like(gate), np.ones_like(beta), lib=lib)
    want = S0.copy()
    want[:, :, 3, :] = v
    ok &= np.allclose(S, want, rtol=0, atol=1e-15)
    return ok


def test_closed_forms():
    assert _closed_forms()


def _identity(lib=None):
    """The page's rewrite: S_t^T q = g S_{t-1}^T q + (q^T k) dv, with dv = beta (v - g S_{t-1}^T k)."""
    S0, q, k, v, gate, beta = _rand(2)
    hv = v.shape[1]
    qe, ke = _expand(q, hv).astype(np.float64), _expand(k, hv).astype(np.float64)
    g, bt = gate[..., None].astype(np.float64), beta[..., None].astype(np.float64)
    S = S0.copy()
    o = gdn.decode_step(S, q, k, v, gate, beta, lib=lib)
    dv = bt * (v - g * np.einsum("bhij,bhi->bhj", S0, ke))
    o2 = g * np.einsum("bhij,bhi->bhj", S0, qe) + np.einsum("bhi,bhi->bh", qe, ke)[..., None] * dv
    S2 = g[..., None] * S0 + np.einsum("bhi,bhj->bhij", ke, dv)
    return np.allclose(o, o2, rtol=1e-10, atol=1e-12) and np.allclose(S, S2, rtol=1e-10, atol=1e-12)


def test_two_pass_identity():
    assert _identity()


def _grouping(lib=None):
    """Value heads 2j and 2j+1 share query/key head j: same result as repeating q and k."""
    S0, q, k, v, gate, beta = _rand(3)
    hv = v.shape[1]
    S1, S2 = S0.copy(), S0.copy()
    o1 = gdn.decode_step(S1, q, k, v, gate, beta, lib=lib)
    o2 = gdn.decode_step(S2, _expand(q, hv), _expand(k, hv), v, gate, beta, lib=lib)
    return np.array_equal(o1, o2) and np.array_equal(S1, S2)


def test_head_grouping():
    assert _grouping()


def test_multi_step_stays_bounded():
    """beta in [0, 1], gate <= 1 and unit keys: the state norm stays bounded over many steps."""
    S, q, k, v, gate, beta = _rand(4)
    for t in range(200):
        _, q, k, v, gate, beta = _rand(100 + t)
        gdn.decode_step(S, q, k, v, gate, beta)
    assert np.isfinite(S).all() and np.abs(S).max() < 50


MUTANTS = {
    "retrieve_after_update": (r"(const double corr = .*?;)\s*(for \(int i = 0; i < dk; \+\+i\)\s*S\[\(size_t\)i \* dv \+ j\] = g \* S\[\(size_t\)i \* dv \+ j\] \+ \(double\)kh\[i\] \* corr;)",
                              r"for (int i = 0; i < dk; ++i) S[(size_t)i * dv + j] = g * S[(size_t)i * dv + j];\n            r = 0.0; for (int i = 0; i < dk; ++i) r += S[(size_t)i * dv + j] * (double)kh[i];\n            \1\n            for (int i = 0; i < dk; ++i) S[(size_t)i * dv + j] += (double)kh[i] * corr;"),
    "no_gate_in_correction": (r"bt \* \(\(double\)vh\[j\] - g \* r\)", "bt * ((double)vh[j] - r)"),
    "no_beta": (r"const double corr = bt \* ", "const double corr = "),
    "output_from_old_state": (r"(for \(int i = 0; i < dk; \+\+i\)\s*S\[\(size_t\)i \* dv \+ j\] = g \* [^;]*;)(\s*)(double acc = 0\.0;[^\n]*\n\s*for \(int i = 0; i < dk; \+\+i\) acc \+= [^;]*;)",
                              r"\3\2\1"),
    "group_modulo": (r"hk = h / group", "hk = h % hqk"),
    "state_not_gated": (r"S\[\(size_t\)i \* dv \+ j\] = g \* S\[\(size_t\)i \* dv \+ j\] \+", "S[(size_t)i * dv + j] = S[(size_t)i * dv + j] +"),
    "sign_of_correction": (r"\+ \(double\)kh\[i\] \* corr", "- (double)kh[i] * corr"),
}


def _mutant(tmp_path, name):
    pat, rep = MUTANTS[name]
    src = open(SRC).read()
    out, n = re.subn(pat, rep, src, flags=re.S)
    assert n >= 1, f"mutation {name} did not apply"
    c, so = tmp_path / f"{name}.c", tmp_path / f"lib{name}.so"
    c.write_text(out)
    subprocess.check_call(["gcc", "-O2", "-std=c11", "-ffp-contract=off", "-fopenmp", "-fPIC", "-shared",
                           "-o", str(so), str(c), "-lm"])
    return gdn.bind(str(so))


@pytest.mark.parametrize("name", sorted(MUTANTS))
def test_pins_catch_planted_mistake(tmp_path, name):
    lib = _mutant(tmp_path, name)
    S, o, want = _hand(lib)
    hand_ok = np.allclose(S, want["S"], atol=1e-12) and np.allclose(o, want["o"], atol=1e-12)
    assert not (hand_ok and _closed_forms(lib) and _identity(lib) and _grouping(lib)), \
        f"mutant {name} passed every pin"
